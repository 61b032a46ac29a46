// bwd_bf16.cuh — backward pass of exact attention on the 5th-generation tensor cores.
//
// "Autoatención, kernels CUDA y FlashAttention" §3 ("Recálculo durante la
// retropropagación") and "FlashAttention" (paweldubiel.com notes, "Mecanismo y
// detalles"): the forward pass keeps only small per-row normalisation statistics (here
// lse = m + ln l) and the backward pass recomputes the attention tiles on chip instead
// of reading an N x N matrix back from memory.  The gradients themselves are not on the
// pages; they are those of the definition O = softmax(S) V, S = scale Q K^T:
//     P = exp(S - lse),  dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
//     dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels:
//   1. fa_bwd_preprocess_kernel: D_i, lse in base 2 (padded to whole 128-row tiles with
//      +inf, so padded rows get P = 0), and zeroes the fp32 dQ accumulator.
//   2. fa_bwd_bf16_kernel: one CTA per (128-key tile j, batch, key/value head).  It keeps
//      K_j, V_j in shared memory and walks the G query heads of its group and their
//      query tiles i (causal: only tiles at or below the diagonal).  Each step is split
//      into query halves A (rows 0-63) and B (64-127) so the softmax-gradient of one half
//      overlaps the tensor-core work of the other:
//        warp 0      TMA producer: K_j, V_j once; Q_i, dO_i, lse_i, D_i per step (2 stages)
//        warp 1      MMA issuer (one thread): per half, S^T = K_j Q_h^T and dP^T = V_j dO_h^T
//                    into TMEM; per half, dV += P^T dO_h and dK += dS^T Q_h with P^T, dS^T
//                    read from TMEM; then dQ_i = dS K_j with dS read from shared memory.
//        warps 4-11  one thread per key (TMEM lane), both warpgroups on half A and then
//                    on half B (32 columns each): P^T and dS^T from S^T, dP^T, lse, D;
//                    P^T and dS^T (bf16) go back over S^T and dP^T in TMEM, dS^T also to
//                    shared memory (swizzled, query-major) for the dQ MMA.  At the end
//                    warps 4-7 write dK_j and warps 8-11 dV_j.
//        warps 12-15 one thread per query row: read dQ_i from TMEM and add it into the fp32
//                    accumulator with vector reductions (red.global.add.v4.f32).
//   3. fa_bwd_finalize_kernel: fp32 dQ accumulator -> bf16 dq (only for bf16 gradients;
//      fp32 gradients accumulate straight into dq).
//
// The scale is folded into dS before it is rounded to bf16 (the preprocess stores
// D_i * scale), so dK and dQ need no further scaling.  TMEM (512 columns): S^T [0,128),
// dP^T [128,256), dV, dK (D columns each), and dQ: at D = 64 one buffer of 64 columns
// followed by K_j and V_j as bf16 A operands (32 columns each), so that S^T and dP^T are
// TS MMAs that read only Q and dO from shared memory; at D = 128 dQ takes the dP^T
// columns, which are free once dK has consumed dS^T, and S^T and dP^T read K_j and V_j
// from shared memory.
#pragma once
#include "common.cuh"

namespace fa {

// FA_BWD_B_FIRST 1: half B's next S^T / dP^T are issued before the step's dQ MMA; 0: after
// it (measured on B200, training workload backward: 1.088 vs 1.077 ms).
#ifndef FA_BWD_B_FIRST
#define FA_BWD_B_FIRST 0
#endif

template <int D>
struct BwdCfg {
  static constexpr int BM = 128;  // query rows per step
  static constexpr int BN = 128;  // keys per CTA
  static constexpr int KB = D / 64;
  static constexpr int TILE = 128 * D * 2;  // one [128 x D] bf16 tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;           // + stage * TILE
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;      // + stage * TILE
  // d = 64 issues the next step's half-A scores before the current step's dQ MMA, so
  // the dS tile that dQ reads is double-buffered; d = 128 has no room and keeps one.
  static constexpr bool EARLY = (D == 64);
  static constexpr int DS_BUF = EARLY ? 2 : 1;
  static constexpr int OFF_DS = OFF_DO + 2 * TILE;     // DS_BUF x [2 query chunks][128 keys][128 B]
  static constexpr int OFF_STAT = OFF_DS + DS_BUF * 128 * 128 * 2;  // per stage: lse2[128], D[128]
  // d = 64 adds dQ into the fp32 accumulator with TMA reduce-adds from per-warp staging
  // (4 drain warps x 32 rows x 64 fp32, 128-byte swizzle); d = 128 has no room left and
  // uses vector reductions from registers
  static constexpr bool DQ_TMA = (D == 64);
  static constexpr int OFF_DQS = OFF_STAT + 2 * 2 * 512;
  static constexpr int OFF_BAR = OFF_DQS + (DQ_TMA ? 4 * 32 * 64 * 4 : 0);
  // D = 128 fills the 227 KB limit exactly, leaving no room to re-align the base: that
  // variant relies on the dynamic shared memory starting 1024-byte aligned and checks it.
  static constexpr int SLACK = (D == 128) ? 0 : 1024;
  static constexpr int SMEM = OFF_BAR + 256 + SLACK;
  static constexpr int WG_DRAIN = 12;  // first dQ drain warp
  static constexpr int THREADS = 512;  // producer, MMA, 2 idle, 8 softmax-gradient, 4 dQ drain
  // epilogue staging (the Q / dO stages, free by then): per softmax warp, its 32 key rows
  // of dK or dV as D / 32 swizzled boxes of 32 rows x 128 bytes (fp32; bf16 uses half)
  static constexpr int STG_WARP = (D / 32) * 4096;
  static_assert(8 * STG_WARP <= 4 * TILE, "epilogue staging must fit the Q and dO stages");
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  // D = 64: K_j and V_j live in TMEM as the A operands of S^T and dP^T (TS MMAs); each
  // SS MMA of N = 64 would read 6 KB of shared memory for 0.26 MFLOP, the TS form reads 2 KB
  static constexpr bool KV_TMEM = (D == 64);
  static constexpr uint32_t COL_KA = 448, COL_VA = 480;  // D = 64 only: 32 columns each
  static constexpr int NQB = 1;                          // dQ TMEM buffers
  __host__ __device__ static constexpr uint32_t col_dq(int) { return D == 64 ? 384u : COL_DP; }
};

struct BwdParams {
  float* dq_acc;          // fp32 [B,Hq,Nq,D] (the caller's dq when gradients are fp32)
  const float* lse2;      // [B*Hq][Nq_pad] lse * log2(e), +inf past Nq
  const float* dstat;     // [B*Hq][Nq_pad] D_i * scale, 0 past Nq
  void* dk;
  void* dv;
  int grad_bf16;
  int dout;               // row width of dq, dk, dv and the accumulator (D, or 96 on the D = 128 kernel)
  int Hq, Hkv, Nq, Nkv, Nq_pad;
  float scale;
  float scale_log2;
  uint64_t wait_ns;
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t kv_tmem;  // D = 64: K_j and V_j copied into TMEM (8 softmax-gradient warps arrive)
  uint64_t qdo_full[2];
  uint64_t qdo_empty[2];
  uint64_t sdp_full[2];  // per query half
  uint64_t ds_ready[2];  // per query half
  uint64_t dq_full[2];
  uint64_t dq_free[2];
  uint64_t dkdv_full;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// ------------------------------------------------------------------------------ 1
// D_i * scale with D_i = sum_c dO_ic O_ic per query row; lse2 = lse * log2(e); both
// padded to Nq_pad.  8 threads per row, each covering D/8 consecutive elements.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_preprocess_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dO,
                                                                 const float* lse, float* lse2, float* dstat,
                                                                 float* dq_zero, long total_rows_pad, int Nq,
                                                                 int Nq_pad, long dq_elems, float scale) {
  const long gt = long(blockIdx.x) * blockDim.x + threadIdx.x;
  const long row = gt >> 3;  // padded row index
  const int part = int(gt & 7);
  if (row < total_rows_pad) {
    const long bh = row / Nq_pad;
    const int q = int(row % Nq_pad);
    float acc = 0.f;
    if (q < Nq) {
      const size_t base = (size_t(bh) * Nq + q) * D + part * (D / 8);
      if constexpr ((D / 8) % 8 == 0) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const uint4 a = *reinterpret_cast<const uint4*>(o + base + c * 8);
          const uint4 g = *reinterpret_cast<const uint4*>(dO + base + c * 8);
          const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fa = __bfloat1622float2(a2[e]), fg = __bfloat1622float2(g2[e]);
            acc = fmaf(fa.x, fg.x, acc);
            acc = fmaf(fa.y, fg.y, acc);
          }
        }
      } else {  // D = 96: 12 elements per thread, 8-byte loads
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const uint2 a = *reinterpret_cast<const uint2*>(o + base + c * 4);
          const uint2 g = *reinterpret_cast<const uint2*>(dO + base + c * 4);
          const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float2 fa = __bfloat1622float2(a2[e]), fg = __bfloat1622float2(g2[e]);
            acc = fmaf(fa.x, fg.x, acc);
            acc = fmaf(fa.y, fg.y, acc);
          }
        }
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (part == 0) {
      dstat[row] = q < Nq ? acc * scale : 0.f;
      lse2[row] = q < Nq ? lse[size_t(bh) * Nq + q] * 1.4426950408889634f : INFINITY;
    }
  }
  // zero the fp32 dQ accumulator (grid-stride, float4)
  const long n4 = dq_elems / 4;
  for (long i = gt; i < n4; i += long(gridDim.x) * blockDim.x)
    reinterpret_cast<float4*>(dq_zero)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------------------ 3
__global__ void __launch_bounds__(256) fa_bwd_finalize_kernel(const float* acc, __nv_bfloat16* dq, long n) {
  const long i = (long(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i < n) {
    const float4 v = *reinterpret_cast<const float4*>(acc + i);
    uint2 pk;
    pk.x = pack_bf16x2(v.x, v.y);
    pk.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(dq + i) = pk;
  }
}

// ------------------------------------------------------------------------------ 2
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    fa_bwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                       const __grid_constant__ CUtensorMap tmDV, const BwdParams p) {
  // tmO maps dO (same geometry as Q); tmDQ maps the fp32 dQ accumulator (32 x 32 boxes);
  // tmDK, tmDV map dk, dv: fp32 with 32 x 32 boxes or bf16 with 64 x 32 boxes (128-byte swizzle)
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  if (C::SLACK == 0 && (smem_u32(smem_raw) & 1023u) != 0) {  // uniform across the CTA
    if (threadIdx.x == 0) set_status(FA_ERR_UNSUPPORTED, 299);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = warp_id(), lane = lane_id();
  const int nj = (p.Nkv + C::BN - 1) / C::BN;
  int j, bk;  // key tile, (batch, kv head)
  bwd_tile_order(blockIdx.x, nj, gridDim.x / nj, j, bk);
  const int b = bk / p.Hkv, hk = bk % p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int off = p.Nkv - p.Nq;
  const int k0 = j * C::BN;
  // first query tile with a row that may see key k0 (row + off >= k0)
  const int i_begin = CAUSAL ? max(0, k0 - off) / C::BM : 0;
  const int n_qt = (p.Nq + C::BM - 1) / C::BM;
  const int n_i = max(0, n_qt - i_begin);
  const int n_steps = G * n_i;  // step s: head h = hk*G + s / n_i, tile i = i_begin + s % n_i

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_tmem, 8);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->qdo_full[s], 1);
      mbar_init(&bars->qdo_empty[s], 1);
      mbar_init(&bars->dq_full[s], 1);
      mbar_init(&bars->dq_free[s], 4);
      mbar_init(&bars->sdp_full[s], 1);
      mbar_init(&bars->ds_ready[s], 8);
    }
    mbar_init(&bars->dkdv_full, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && n_steps > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmO);
      mbar_arrive_expect_tx(&bars->kv_full, 2 * C::TILE);
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_3d(smem + C::OFF_K + kb * 128 * 128, &tmK, &bars->kv_full, kb * 64, k0, bk);
        tma_load_3d(smem + C::OFF_V + kb * 128 * 128, &tmV, &bars->kv_full, kb * 64, k0, bk);
      }
      for (int s = 0; s < n_steps; ++s) {
        const int st = s & 1;
        if (s >= 2 && !mbar_wait(&bars->qdo_empty[st], ((s >> 1) - 1) & 1, p.wait_ns, abort_flag, 200)) break;
        const int h = hk * G + s / n_i, i = i_begin + s % n_i;
        const int bh = b * p.Hq + h;
        mbar_arrive_expect_tx(&bars->qdo_full[st], 2 * C::TILE + 1024);
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_3d(smem + C::OFF_Q + st * C::TILE + kb * 128 * 128, &tmQ, &bars->qdo_full[st], kb * 64,
                      i * C::BM, bh);
          tma_load_3d(smem + C::OFF_DO + st * C::TILE + kb * 128 * 128, &tmO, &bars->qdo_full[st], kb * 64,
                      i * C::BM, bh);
        }
        const size_t srow = size_t(bh) * p.Nq_pad + size_t(i) * C::BM;
        bulk_load(smem + C::OFF_STAT + st * 1024, p.lse2 + srow, 512, &bars->qdo_full[st]);
        bulk_load(smem + C::OFF_STAT + st * 1024 + 512, p.dstat + srow, 512, &bars->qdo_full[st]);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Each step is split into query halves A (rows 0-63) and B (64-127): S^T and dP^T of
    // half B run on the tensor core while half A's softmax-gradient is computed, and
    // half A's dV/dK MMAs run while half B's is.  The whole warp runs this role (so the
    // descriptors stay warp-uniform); the elected lane issues the MMAs and commits.
    if (n_steps > 0) {
      const uint32_t leader = elect_one();
      constexpr uint32_t idKK = idesc_bf16_f32(128, 64, 0);             // S^T, dP^T halves: N = 64
      constexpr uint32_t idTS = idesc_bf16_f32(128, D, 1);              // dV, dK: B (dO, Q) MN-major
      constexpr uint32_t idQ = idesc_bf16_f32(128, D, 1) | (1u << 15);  // dQ: A (dS), B (K) MN-major
      // base descriptors (128-byte swizzle): K-major operands step 32 B per k-step inside a
      // 64-column block and 16 KB per block; MN-major ones have 128-row (16 KB) blocks
      const uint64_t dK = sdesc_sw128(sbase + C::OFF_K, 16, 1024), dV = sdesc_sw128(sbase + C::OFF_V, 16, 1024);
      const uint64_t dQk = sdesc_sw128(sbase + C::OFF_Q, 16, 1024), dOk = sdesc_sw128(sbase + C::OFF_DO, 16, 1024);
      const uint64_t dQm = sdesc_sw128(sbase + C::OFF_Q, 128 * 128, 1024);
      const uint64_t dOm = sdesc_sw128(sbase + C::OFF_DO, 128 * 128, 1024);
      const uint64_t dSm = sdesc_sw128(sbase + C::OFF_DS, 128 * 128, 1024);
      const uint64_t dKm = sdesc_sw128(sbase + C::OFF_K, 128 * 128, 1024);
      // S^T and dP^T of query half hf of step s (commit sdp_full[hf])
      auto issue_sdp = [&](int s, int hf) {
        const uint32_t qo = (s & 1) * C::TILE + hf * 64 * 128;  // rows [64 hf, 64 hf + 64) of Q, dO
        // K_j, V_j as A from TMEM (D = 64: 8 columns = 16 bf16 per k-step) or shared memory
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * 128 * 128 + (ks & 3) * 32;
          if constexpr (C::KV_TMEM)
            mma_ts_p(tmem + C::COL_S + 64 * hf, tmem + C::COL_KA + ks * 8, desc_add(dQk, qo + koff), idKK, ks > 0,
                     leader);
          else
            mma_ss_p(tmem + C::COL_S + 64 * hf, desc_add(dK, koff), desc_add(dQk, qo + koff), idKK, ks > 0, leader);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * 128 * 128 + (ks & 3) * 32;
          if constexpr (C::KV_TMEM)
            mma_ts_p(tmem + C::COL_DP + 64 * hf, tmem + C::COL_VA + ks * 8, desc_add(dOk, qo + koff), idKK, ks > 0,
                     leader);
          else
            mma_ss_p(tmem + C::COL_DP + 64 * hf, desc_add(dV, koff), desc_add(dOk, qo + koff), idKK, ks > 0, leader);
        }
        mma_commit_p(&bars->sdp_full[hf], leader);
      };
      // dV += P^T dO ; dK += dS^T Q for query half hf of step s (K dimension = 64 queries)
      auto issue_dvdk = [&](int s, int hf) {
        const uint32_t so = (s & 1) * C::TILE;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t acc = (s > 0 || hf > 0 || ks > 0) ? 1u : 0u;
          const uint32_t roff = (hf * 4 + ks) * 2048;  // 16 query rows per k-step
          const uint32_t pcol = 64 * hf + (ks >> 1) * 32 + (ks & 1) * 8;  // packed P / dS of queries 16ks..
          mma_ts_p(tmem + C::COL_DV, tmem + C::COL_S + pcol, desc_add(dOm, so + roff), idTS, acc, leader);
          mma_ts_p(tmem + C::COL_DK, tmem + C::COL_DP + pcol, desc_add(dQm, so + roff), idTS, acc, leader);
        }
      };
      // dQ_i = dS K_j (M = queries, K dimension = the 128 keys); then release Q_i, dO_i
      auto issue_dq = [&](int s) -> bool {
        const int qb = 0;
        if constexpr (C::EARLY) {  // (D = 128 waits for the drain before the step's dP^T)
          if (s >= 1 && !warp_wait(&bars->dq_free[0], (s - 1) & 1, p.wait_ns, abort_flag, 214)) return false;
        }
        const uint32_t dso = (s % C::DS_BUF) * (128 * 128 * 2);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss_p(tmem + C::col_dq(qb), desc_add(dSm, dso + ks * 2048), desc_add(dKm, ks * 2048), idQ, ks > 0, leader);
        mma_commit_p(&bars->dq_full[qb], leader);
        mma_commit_p(&bars->qdo_empty[s & 1], leader);
        return true;
      };
      auto wait_qdo = [&](int s) { return warp_wait(&bars->qdo_full[s & 1], (s >> 1) & 1, p.wait_ns, abort_flag, 211); };
      auto wait_ds = [&](int s, int hf) { return warp_wait(&bars->ds_ready[hf], s & 1, p.wait_ns, abort_flag, 213); };

      bool ok = C::KV_TMEM ? warp_wait(&bars->kv_tmem, 0, p.wait_ns, abort_flag, 210)
                           : warp_wait(&bars->kv_full, 0, p.wait_ns, abort_flag, 210);
      if constexpr (C::EARLY) {
        // half A of step s+1 enters the tensor core as soon as half A of step s is
        // consumed (and half B's as soon as half B's), so the warpgroups of the two halves
        // run staggered by half a step
        if (ok && (ok = wait_qdo(0))) {
          tc_fence_after();
          issue_sdp(0, 0);
          issue_sdp(0, 1);
        }
        for (int s = 0; s < n_steps && ok; ++s) {
          if (!(ok = wait_ds(s, 0))) break;
          tc_fence_after();
          issue_dvdk(s, 0);
          if (s + 1 < n_steps) {
            if (!(ok = wait_qdo(s + 1))) break;
            tc_fence_after();
            issue_sdp(s + 1, 0);
          }
          if (!(ok = wait_ds(s, 1))) break;
          tc_fence_after();
          issue_dvdk(s, 1);
          if (FA_BWD_B_FIRST) {
            // half B's next scores go before this step's dQ, which no softmax warp waits for
            if (s + 1 < n_steps) issue_sdp(s + 1, 1);
            if (!(ok = issue_dq(s))) break;
          } else {
            if (!(ok = issue_dq(s))) break;
            if (s + 1 < n_steps) issue_sdp(s + 1, 1);
          }
        }
      } else {
        for (int s = 0; s < n_steps && ok; ++s) {
          if (!(ok = wait_qdo(s))) break;
          if (s > 0 && !(ok = warp_wait(&bars->dq_free[0], (s - 1) & 1, p.wait_ns, abort_flag, 212))) break;
          tc_fence_after();  // (dP^T overwrites the previous dQ: its drain was awaited above)
          issue_sdp(s, 0);
          issue_sdp(s, 1);
          for (int hf = 0; hf < 2 && ok; ++hf) {
            if (!(ok = wait_ds(s, hf))) break;
            tc_fence_after();
            issue_dvdk(s, hf);
          }
          if (!ok || !(ok = issue_dq(s))) break;
        }
      }
      if (ok) mma_commit_p(&bars->dkdv_full, leader);
    }
  } else if (warp >= 4 && warp < C::WG_DRAIN) {
    // ---------------------------------------------------------------- softmax-gradient
    // One thread per key (TMEM lane).  Warps 4-7 and 8-11 take columns [0, 32) and
    // [32, 64) of query half A and then of half B, in two sub-chunks of 16 columns each.
    // (Four warpgroups, two per half with the halves running concurrently, were measured
    // slower: 1.240 against 1.077 ms for the training backward, at 80 registers per thread.)
    const int wc = (warp - 4) >> 2;  // 32-column chunk of each half
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // key within the tile == TMEM lane
    const int key = k0 + r;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const float sl2 = p.scale_log2, scale = p.scale;
    bool ok = true;
    if constexpr (C::KV_TMEM) {
      // key row r of K_j (warps 4-7) or V_j (warps 8-11) from shared memory (128-byte
      // swizzle: 16-byte chunk u of row r sits at chunk u ^ (r % 8)) into TMEM lane r as 32
      // columns of bf16 pairs, the A-operand layout of the TS MMAs
      if (n_steps > 0) {
        ok = warp_wait(&bars->kv_full, 0, p.wait_ns, abort_flag, 223);
        if (ok) {
          const uint8_t* row = smem + (wc == 0 ? C::OFF_K : C::OFF_V) + r * 128;
          uint32_t a[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 x = *reinterpret_cast<const uint4*>(row + ((u ^ (r & 7)) << 4));
            a[4 * u] = x.x;
            a[4 * u + 1] = x.y;
            a[4 * u + 2] = x.z;
            a[4 * u + 3] = x.w;
          }
          tmem_st32(tmem + lane_off + (wc == 0 ? C::COL_KA : C::COL_VA), a);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->kv_tmem);
        }
      }
    }
    for (int s = 0; s < n_steps && ok; ++s) {
      const int st = s & 1;
      const int i = i_begin + s % n_i;
      ok = warp_wait(&bars->qdo_full[st], (s >> 1) & 1, p.wait_ns, abort_flag, 221);
#pragma unroll 1
      for (int hf = 0; hf < 2 && ok; ++hf) {
      ok = warp_wait(&bars->sdp_full[hf], s & 1, p.wait_ns, abort_flag, 220);
      if (!ok) break;
      tc_fence_after();
      const int q0 = 64 * hf + 32 * wc;  // first query (column) of this warp's chunk
      // columns q < lim of the chunk are masked for this key; a key past Nkv masks all
      int lim = 0;
      if (key >= p.Nkv) lim = 32;
      else if (CAUSAL) lim = min(32, max(0, key - off - i * C::BM - q0));
      const float* lse_s = reinterpret_cast<const float*>(smem + C::OFF_STAT + st * 1024) + q0;
      const float* d_s = lse_s + 128;
      const bool any_masked = __any_sync(0xffffffffu, lim > 0);
      // dS (query-major, 128-byte swizzle): half hf is block hf, this chunk units 4wc..4wc+3
      uint8_t* dsrow = smem + C::OFF_DS + (s % C::DS_BUF) * (128 * 128 * 2) + hf * (128 * 128) + r * 128;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[16], dv[16];
        tmem_ld16(tmem + lane_off + C::COL_S + q0 + 16 * c, sv);
        tmem_ld16(tmem + lane_off + C::COL_DP + q0 + 16 * c, dv);
        tmem_wait_ld();
        uint32_t pp[8], pd[8];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse_s + 16 * c + e);
          const float4 d4 = *reinterpret_cast<const float4*>(d_s + 16 * c + e);
          const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])),
                                        make_float2(sl2, sl2), make_float2(-l4.x, -l4.y));
          const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3])),
                                        make_float2(sl2, sl2), make_float2(-l4.z, -l4.w));
          float2 p01 = make_float2(ex2(x01.x), ex2(x01.y));
          float2 p23 = make_float2(ex2(x23.x), ex2(x23.y));
          if (any_masked) {
            const int col = 16 * c + e;
            if (col < lim) p01.x = 0.f;
            if (col + 1 < lim) p01.y = 0.f;
            if (col + 2 < lim) p23.x = 0.f;
            if (col + 3 < lim) p23.y = 0.f;
          }
          // dS * scale = P * (dP * scale - D * scale)  (d4 holds D * scale)
          const float2 g01 = __fmul2_rn(
              p01, __ffma2_rn(make_float2(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])),
                              make_float2(scale, scale), make_float2(-d4.x, -d4.y)));
          const float2 g23 = __fmul2_rn(
              p23, __ffma2_rn(make_float2(__uint_as_float(dv[e + 2]), __uint_as_float(dv[e + 3])),
                              make_float2(scale, scale), make_float2(-d4.z, -d4.w)));
          pp[e / 2] = pack_bf16x2(p01.x, p01.y);
          pp[e / 2 + 1] = pack_bf16x2(p23.x, p23.y);
          pd[e / 2] = pack_bf16x2(g01.x, g01.y);
          pd[e / 2 + 1] = pack_bf16x2(g23.x, g23.y);
        }
        // P^T and dS^T as bf16 pairs over the first 8 of the sub-chunk's pair of 8-column
        // groups: queries 16k..16k+15 of the half land at columns 64hf + (k>>1)*32 + (k&1)*8,
        // where the dV/dK MMAs read k-step k (columns of S^T / dP^T already consumed)
        tmem_st8(tmem + lane_off + C::COL_S + q0 + 8 * c, pp);
        tmem_st8(tmem + lane_off + C::COL_DP + q0 + 8 * c, pd);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int unit = wc * 4 + 2 * c + u;
          *reinterpret_cast<uint4*>(dsrow + ((unit ^ (r & 7)) * 16)) =
              make_uint4(pd[4 * u], pd[4 * u + 1], pd[4 * u + 2], pd[4 * u + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();  // dS written by the generic proxy, read by the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready[hf]);
      }
    }
    // ---- dK_j (warps 4-7) and dV_j (warps 8-11); the scale is already folded into dS.
    // Each warp stages its 32 key rows in shared memory (128-byte swizzle) and writes them
    // with TMA tensor stores, which drop the rows past Nkv and the columns past dout.
    const bool is_dk = wc == 0;
    const uint32_t col = is_dk ? C::COL_DK : C::COL_DV;
    const CUtensorMap* tmap = is_dk ? &tmDK : &tmDV;
    if (ok && n_steps > 0) ok = warp_wait(&bars->dkdv_full, 0, p.wait_ns, abort_flag, 222);
    if (ok && n_steps > 0) {
      tc_fence_after();
      uint8_t* stg = smem + C::OFF_Q + (warp - 4) * C::STG_WARP;  // every MMA is done: Q, dO free
      const int nch = p.dout / 32;
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + col + c * 32, v);
        tmem_wait_ld();
        if (p.grad_bf16) {
          // 64-column boxes of 32 rows x 128 bytes: chunk c fills half c & 1 of box c / 2
          uint8_t* row = stg + (c >> 1) * 4096 + lane * 128;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(row + (((4 * (c & 1) + u) ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16x2(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
                           pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                           pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                           pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
        } else {
          uint8_t* row = stg + c * 4096 + lane * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(row + ((u ^ (lane & 7)) << 4)) =
                make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int nbox = p.grad_bf16 ? (nch + 1) / 2 : nch;
        for (int x = 0; x < nbox; ++x)
          tma_store_3d(tmap, stg + x * 4096, x * (p.grad_bf16 ? 64 : 32), k0 + wq * 32, bk);
        bulk_commit();
        bulk_wait_all();  // the stores have read the staging before the CTA ends
      }
    } else if (n_steps == 0 && key < p.Nkv) {
      // no query row can see these keys: their gradients are zero
      void* dst = is_dk ? p.dk : p.dv;
      const size_t base = (size_t(bk) * p.Nkv + key) * p.dout;
      for (int c = 0; c < p.dout; c += 4) {
        if (p.grad_bf16)
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(dst) + base + c) = make_uint2(0, 0);
        else
          *reinterpret_cast<float4*>(static_cast<float*>(dst) + base + c) = make_float4(0, 0, 0, 0);
      }
    }
  } else if (warp >= C::WG_DRAIN) {
    // ---------------------------------------------------------------- dQ drain (query rows)
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    bool ok = true;
    for (int s = 0; s < n_steps && ok; ++s) {
      const int qb = 0;
      ok = warp_wait(&bars->dq_full[qb], s & 1, p.wait_ns, abort_flag, 230);
      if (!ok) break;
      tc_fence_after();
      const int h = hk * G + s / n_i, i = i_begin + s % n_i;
      const int q = i * C::BM + r;
      if constexpr (C::DQ_TMA) {
        uint8_t* stg = smem + C::OFF_DQS + wq * (32 * 64 * 4);  // two 32x32 fp32 boxes
        if (lane == 0) bulk_wait_read();  // this warp's previous reduces have read the staging
        __syncwarp();
#pragma unroll 1
        for (int hb = 0; hb < 2; ++hb) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + C::col_dq(qb) + 32 * hb, v);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(stg + hb * 4096 + lane * 128 + ((u ^ (lane & 7)) << 4)) =
                make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int row0 = i * C::BM + wq * 32, z = b * p.Hq + h;
          tma_reduce_add_3d(&tmDQ, stg, 0, row0, z);
          tma_reduce_add_3d(&tmDQ, stg + 4096, 32, row0, z);
          bulk_commit();
        }
      } else {
        float* dstq = p.dq_acc + ((size_t(b) * p.Hq + h) * p.Nq + q) * p.dout;
#pragma unroll 1
        for (int c = 0; c < p.dout / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + C::col_dq(qb) + c * 32, v);
          tmem_wait_ld();
          if (q < p.Nq) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              red_add_v4(dstq + c * 32 + e, __uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                         __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_free[qb]);
    }
    if (C::DQ_TMA && lane == 0) bulk_wait_all();  // the reduce-adds complete before exit
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
