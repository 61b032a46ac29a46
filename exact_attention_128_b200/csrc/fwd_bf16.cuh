// fwd_bf16.cuh — bf16 forward pass on the 5th-generation tensor cores (sm_100a).
//
// Computes O = softmax(Q K^T * scale) V and lse = m + ln(l) per query row
// ("Autoatención, kernels CUDA y FlashAttention" §1) tile by tile, never writing the
// score matrix to device memory (same page, §3 "Procesamiento por bloques"), with the
// online-softmax recurrence of "FlashAttention" (paweldubiel.com notes), "No basta con
// promediar los resultados de los bloques": running max m, sum l and numerator u; when
// a tile raises the maximum, l and u are rescaled by e^{m - m'} before the tile's own
// terms are added; the output is u / l.
//
// One CTA owns two 128-row query tiles (Q0, Q1) of one (batch, query head) and streams
// the 128-key tiles of its key/value head (GQA: head h reads h / (Hq/Hkv)).
//   warp 0      TMA producer: Q0/Q1 once, then K_j and V_j into a ring of stages.
//   warp 1      MMA issuer (one thread): S_t = Q_t K_j^T into TMEM (SS MMA), then
//               u_t += P_t V_j with P_t read from TMEM (TS MMA).
//   warps 4-7   softmax for Q0, warps 8-11 softmax for Q1: each thread owns one
//               query row = one TMEM lane; it reads S_t, updates (m, l), writes P_t
//               (bf16) over S_t in TMEM, and rescales u_t in TMEM when m rose.
// While one warpgroup runs the softmax of its tile, the tensor core works on the
// other tile, so the exponentials overlap the MMAs.
//
// TMEM columns (512 allocated): S0 [0,128), S1 [128,256), u0 [256,256+D), u1 after.
// Shared memory: Q0, Q1, then NSTAGE K tiles and NSTAGE V tiles, each stored as
// D/64 column blocks of [rows x 128 bytes] with the 128-byte swizzle TMA writes
// and the MMA descriptors expect.
#pragma once
#include "common.cuh"

namespace fa {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;  // rows per query tile (two tiles per CTA)
  static constexpr int BN = 128;  // keys per tile
  static constexpr int KB = D / 64;
  static constexpr int Q_TILE = BM * D * 2;
  static constexpr int KV_TILE = BN * D * 2;
  static constexpr int NSTAGE = (D == 128) ? 2 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * Q_TILE;
  static constexpr int OFF_V = OFF_K + NSTAGE * KV_TILE;
  static constexpr int OFF_BAR = OFF_V + NSTAGE * KV_TILE;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // + barriers + alignment slack
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0;    // + t * 128
  static constexpr uint32_t COL_O = 256;  // + t * D
};

struct FwdBf16Params {
  __nv_bfloat16* o;
  float* lse;
  int Hq, Hkv, Nq, Nkv;
  float scale_log2;  // scale * log2(e)
  uint64_t wait_ns;
};

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[4];
  uint64_t v_full[4];
  uint64_t kv_empty[4];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_final[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdBf16Params p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = warp_id(), lane = lane_id();
  const int qt = CAUSAL ? int(gridDim.x - 1 - blockIdx.x) : int(blockIdx.x);  // heavy causal tiles first
  const int bh = blockIdx.y;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int hk = h / (p.Hq / p.Hkv);
  const int q_row0 = qt * 2 * C::BM;
  const int off = p.Nkv - p.Nq;  // bottom-right causal alignment
  int kv_end = p.Nkv;
  if (CAUSAL) kv_end = min(p.Nkv, min(q_row0 + 2 * C::BM, p.Nq) + off);
  const int n = (kv_end + C::BN - 1) / C::BN;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 4);
      mbar_init(&bars->o_final[t], 1);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sK = smem_u32(smem + C::OFF_K);
  const uint32_t sV = smem_u32(smem + C::OFF_V);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::Q_TILE);
      for (int t = 0; t < 2; ++t)
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(smem + C::OFF_Q + t * C::Q_TILE + kb * C::BM * 128, &tmQ, &bars->q_full, kb * 64,
                      q_row0 + t * C::BM, bh);
      const int zkv = b * p.Hkv + hk;
      for (int j = 0; j < n; ++j) {
        const int st = j % C::NSTAGE, round = j / C::NSTAGE;
        if (round > 0 && !mbar_wait(&bars->kv_empty[st], (round - 1) & 1, p.wait_ns, abort_flag, 10)) break;
        mbar_arrive_expect_tx(&bars->k_full[st], C::KV_TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(smem + C::OFF_K + st * C::KV_TILE + kb * C::BN * 128, &tmK, &bars->k_full[st], kb * 64,
                      j * C::BN, zkv);
        mbar_arrive_expect_tx(&bars->v_full[st], C::KV_TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(smem + C::OFF_V + st * C::KV_TILE + kb * C::BN * 128, &tmV, &bars->v_full[st], kb * 64,
                      j * C::BN, zkv);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, C::BN, 0);  // K-major A (Q) and B (K)
      constexpr uint32_t idPV = idesc_bf16_f32(128, D, 1);     // B (V) is MN-major
      auto issue_S = [&](int t, int st) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;
          const uint64_t a = sdesc_sw128(sQ + t * C::Q_TILE + kb * C::BM * 128 + kin * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sK + st * C::KV_TILE + kb * C::BN * 128 + kin * 32, 16, 1024);
          mma_ss(tmem + C::COL_S + t * 128, a, bd, idS, ks > 0 ? 1u : 0u);
        }
      };
      auto issue_PV = [&](int t, int st, int j) {
#pragma unroll
        for (int ks = 0; ks < C::BN / 16; ++ks) {
          const uint64_t bd = sdesc_sw128(sV + st * C::KV_TILE + ks * 16 * 128, C::BN * 128, 1024);
          mma_ts(tmem + C::COL_O + t * D, tmem + C::COL_S + t * 128 + ks * 8, bd, idPV,
                 (j > 0 || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&bars->q_full, 0, p.wait_ns, abort_flag, 20) &&
                mbar_wait(&bars->k_full[0], 0, p.wait_ns, abort_flag, 21);
      if (ok) {
        tc_fence_after();
        issue_S(0, 0);
        mma_commit(&bars->s_full[0]);
        issue_S(1, 0);
        mma_commit(&bars->s_full[1]);
        for (int j = 0; j < n && ok; ++j) {
          const int st = j % C::NSTAGE;
          const int st2 = (j + 1) % C::NSTAGE;
          const bool more = j + 1 < n;
          ok = mbar_wait(&bars->v_full[st], (j / C::NSTAGE) & 1, p.wait_ns, abort_flag, 22) &&
               mbar_wait(&bars->p_full[0], j & 1, p.wait_ns, abort_flag, 23);
          if (!ok) break;
          tc_fence_after();
          issue_PV(0, st, j);
          if (more) {
            ok = mbar_wait(&bars->k_full[st2], ((j + 1) / C::NSTAGE) & 1, p.wait_ns, abort_flag, 24);
            if (!ok) break;
            tc_fence_after();
            issue_S(0, st2);
            mma_commit(&bars->s_full[0]);
          } else {
            mma_commit(&bars->o_final[0]);
          }
          ok = mbar_wait(&bars->p_full[1], j & 1, p.wait_ns, abort_flag, 25);
          if (!ok) break;
          tc_fence_after();
          issue_PV(1, st, j);
          mma_commit(&bars->kv_empty[st]);
          if (more) {
            issue_S(1, st2);
            mma_commit(&bars->s_full[1]);
          } else {
            mma_commit(&bars->o_final[1]);
          }
        }
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax
    const int t = (warp - 4) >> 2;              // which query tile
    const int wq = warp & 3;                    // TMEM lane quarter this warp may access
    const int r = wq * 32 + lane;               // row within the tile == TMEM lane
    const int row = q_row0 + t * C::BM + r;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::COL_S + t * 128;
    const uint32_t tO = tmem + lane_off + C::COL_O + t * D;
    const int row_limit = CAUSAL ? min(p.Nkv, row + off + 1) : p.Nkv;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;

    for (int j = 0; j < n; ++j) {
      ok = warp_wait(&bars->s_full[t], j & 1, p.wait_ns, abort_flag, 30 + t);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[C::BN];
#pragma unroll
      for (int c = 0; c < C::BN / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      float f[C::BN];
      const int lim = row_limit - j * C::BN;
#pragma unroll
      for (int c = 0; c < C::BN; ++c) f[c] = __uint_as_float(sr[c]);
      if (lim < C::BN) {
#pragma unroll
        for (int c = 0; c < C::BN; ++c) f[c] = (c < lim) ? f[c] : -INFINITY;
      }
      float mx = f[0];
#pragma unroll
      for (int c = 1; c < C::BN; ++c) mx = fmaxf(mx, f[c]);
      const float m_new = fmaxf(m, mx * sl2);
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m_new == m) ? 1.f : ex2(m - base);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < C::BN / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2(fmaf(f[c * 32 + 2 * i], sl2, -base));
          const float p1 = ex2(fmaf(f[c * 32 + 2 * i + 1], sl2, -base));
          rs += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + c * 16, pk);
      }
      l = l * alpha + rs;
      // u (TMEM) holds the P.V sums of tiles < j; rescale its rows whose max rose
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[t]);
      m = m_new;
    }
    if (ok) ok = warp_wait(&bars->o_final[t], 0, p.wait_ns, abort_flag, 40 + t);
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.o + (size_t(bh) * p.Nq + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (row < p.Nq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      if (row < p.Nq) p.lse[size_t(bh) * p.Nq + row] = (m + __log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
