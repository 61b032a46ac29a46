// bwd_d256.cuh — backward pass at head dimension 256 on the 5th-generation tensor cores.
//
// The same gradients as bwd_bf16.cuh ("Autoatención, kernels CUDA y FlashAttention" §3,
// "Recálculo durante la retropropagación": the score tiles are recomputed from the saved
// lse instead of being stored), with P = exp(S - lse), dV = P^T dO, dP = dO V^T,
// dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q.
//
// At d = 256 the accumulators of one 128-key tile, dK and dV (256 fp32 columns each), fill
// the whole of TMEM, and K, V, Q and dO tiles would need 256 KB of shared memory.  So each
// CTA owns a 128-key tile AND one 128-column half h of the head dimension:
//   - it recomputes the full-d S^T = K Q^T and dP^T = V dO^T (the two CTAs of a key tile
//     both do; 40 % more MMA work than the five contractions of the method),
//   - accumulates dV[:, h] and dK[:, h] in TMEM,
//   - computes dQ^T[h] = K[:, h]^T dS^T (M = the 128 columns of h, N = the step's queries)
//     and adds it, transposed through shared memory, into the fp32 dQ accumulator with
//     TMA reduce-adds.
// Query steps are 64 rows; Q and dO are double-buffered.  V lives in TMEM as the A operand
// of dP^T (copied once from shared memory), which frees the shared memory it would take.
//
// TMEM (512 columns): S^T [0, 64), dP^T [64, 128) (dQ^T after dK has consumed dS^T),
// dV_h [128, 256), dK_h [256, 384), V [384, 512) (bf16 pairs, 128 columns for 256 d).
// Shared memory: K 64 KB (four [128 keys][64 d] swizzled blocks), dO stages 2 x 32 KB (V
// is staged there first), Q stages 2 x 32 KB, dS^T [128 keys][64 queries] 16 KB, lse/D,
// dQ staging 16 KB.
// Roles: warp 0 TMA producer, warp 1 MMA issuer (elected lane), warps 4-11 softmax-
// gradient (one thread per key; warps 4-7 queries [0, 32), warps 8-11 [32, 64)), warps
// 12-15 dQ^T drain (one thread per d-row of the half).
#pragma once
#include "common.cuh"
#include "bwd_bf16.cuh"

namespace fa {

struct Bwd256Cfg {
  static constexpr int D = 256;
  static constexpr int BM = 64;   // query rows per step
  static constexpr int BN = 128;  // keys per CTA
  static constexpr int DH = 128;  // head-dimension columns per CTA
  static constexpr int OFF_K = 0;                // 4 x [128][64] bf16
  static constexpr int OFF_DO = 65536;           // + st * 32768: 4 x [64][64]; V (4 x [128][64]) first
  static constexpr int OFF_Q = OFF_DO + 65536;   // + st * 32768
  static constexpr int OFF_DS = OFF_Q + 65536;   // [128 keys][64 queries] bf16, 128-byte swizzle
  static constexpr int OFF_STAT = OFF_DS + 16384;  // + st * 512: lse2[64], D[64]
  static constexpr int OFF_DQS = OFF_STAT + 1024;   // dQ staging: per drain warp [32 queries][32 d] fp32
  static constexpr int OFF_BAR = OFF_DQS + 4 * 4096;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int THREADS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 64, COL_DV = 128, COL_DK = 256, COL_VA = 384;
};

struct Bwd256Bars {
  uint64_t kv_full;
  uint64_t v_tmem;  // V copied into TMEM (8 softmax-gradient warps arrive)
  uint64_t qdo_full[2];
  uint64_t qdo_empty[2];
  uint64_t s_full;   // S^T of the step is in TMEM
  uint64_t dp_full;  // dP^T of the step is in TMEM
  uint64_t ds_ready;
  uint64_t dq_full;
  uint64_t dq_free;
  uint64_t dkdv_full;
  uint32_t tmem_base;
  int abort_flag;
};

template <bool CAUSAL>
__global__ void __launch_bounds__(Bwd256Cfg::THREADS, 1)
    fa_bwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  // tmQ / tmO map Q and dO with (64, 64) boxes, tmK / tmV map K and V with (64, 128) boxes,
  // tmDQ the fp32 dQ accumulator with (32, 32) boxes and the 128-byte swizzle
  using C = Bwd256Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bwd256Bars* bars = reinterpret_cast<Bwd256Bars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = warp_id(), lane = lane_id();
  const int nj = (p.Nkv + C::BN - 1) / C::BN;
  int j, u;  // key tile, unit = (batch, kv head) x 2 + head-dimension half
  bwd_tile_order(blockIdx.x, nj, gridDim.x / nj, j, u);
  const int bk = u >> 1;
  const int hh = u & 1;  // head-dimension half
  const int b = bk / p.Hkv, hk = bk % p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int off = p.Nkv - p.Nq;
  const int k0 = j * C::BN;
  const int i_begin = CAUSAL ? max(0, k0 - off) / C::BM : 0;  // first query tile that sees key k0
  const int n_qt = (p.Nq + C::BM - 1) / C::BM;
  const int n_i = max(0, n_qt - i_begin);
  const int n_steps = G * n_i;  // step s: head hk*G + s / n_i, tile i_begin + s % n_i

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->v_tmem, 8);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->qdo_full[s], 1);
      mbar_init(&bars->qdo_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->ds_ready, 8);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, 4);
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
      mbar_arrive_expect_tx(&bars->kv_full, 2 * 65536);
      for (int kb = 0; kb < 4; ++kb) {
        tma_load_3d(smem + C::OFF_K + kb * 16384, &tmK, &bars->kv_full, kb * 64, k0, bk);
        tma_load_3d(smem + C::OFF_DO + kb * 16384, &tmV, &bars->kv_full, kb * 64, k0, bk);
      }
      // dO shares its buffers with the staged V: wait until V is in TMEM
      bool ok = mbar_wait(&bars->v_tmem, 0, p.wait_ns, abort_flag, 300);
      for (int s = 0; s < n_steps && ok; ++s) {
        const int st = s & 1;
        if (s >= 2 && !(ok = mbar_wait(&bars->qdo_empty[st], ((s >> 1) - 1) & 1, p.wait_ns, abort_flag, 301))) break;
        const int h = hk * G + s / n_i, i = i_begin + s % n_i;
        const int bh = b * p.Hq + h;
        mbar_arrive_expect_tx(&bars->qdo_full[st], 2 * 32768 + 512);
        for (int kb = 0; kb < 4; ++kb) {
          tma_load_3d(smem + C::OFF_Q + st * 32768 + kb * 8192, &tmQ, &bars->qdo_full[st], kb * 64, i * C::BM, bh);
          tma_load_3d(smem + C::OFF_DO + st * 32768 + kb * 8192, &tmO, &bars->qdo_full[st], kb * 64, i * C::BM, bh);
        }
        const size_t srow = size_t(bh) * p.Nq_pad + size_t(i) * C::BM;
        bulk_load(smem + C::OFF_STAT + st * 512, p.lse2 + srow, 256, &bars->qdo_full[st]);
        bulk_load(smem + C::OFF_STAT + st * 512 + 256, p.dstat + srow, 256, &bars->qdo_full[st]);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (n_steps > 0) {
      const uint32_t leader = elect_one();
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, 0);                  // S^T, dP^T: N = 64 queries
      constexpr uint32_t idKV = idesc_bf16_f32(128, 128, 1);                // dV_h, dK_h: B MN-major
      constexpr uint32_t idQT = idesc_bf16_f32(128, 64, 1) | (1u << 15);   // dQ^T: A, B MN-major
      const uint64_t dK = sdesc_sw128(sbase + C::OFF_K, 16, 1024);          // K-major, 128-row blocks
      const uint64_t dQk = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);         // K-major, 64-row blocks
      const uint64_t dOk = sdesc_sw128(sbase + C::OFF_DO, 16, 1024);
      const uint64_t dQm = sdesc_sw128(sbase + C::OFF_Q, 8192, 1024);       // MN-major over d: 64-row blocks
      const uint64_t dOm = sdesc_sw128(sbase + C::OFF_DO, 8192, 1024);
      const uint64_t dKm = sdesc_sw128(sbase + C::OFF_K, 16384, 1024);      // MN-major over d: 128-row blocks
      const uint64_t dSm = sdesc_sw128(sbase + C::OFF_DS, 8192, 1024);      // MN-major over queries
      // S^T = K Q^T over all 256 d: 16 k-steps of 16 (block ks / 4, 32 bytes per k-step within it)
      auto issue_s = [&](int s) {
        const uint32_t qo = (s & 1) * 32768;
#pragma unroll
        for (int ks = 0; ks < 16; ++ks)
          mma_ss_p(tmem + C::COL_S, desc_add(dK, (ks >> 2) * 16384 + (ks & 3) * 32),
                   desc_add(dQk, qo + (ks >> 2) * 8192 + (ks & 3) * 32), idS, ks > 0, leader);
        mma_commit_p(&bars->s_full, leader);
      };
      // dP^T = V dO^T with V from TMEM (8 columns = 16 bf16 per k-step)
      auto issue_dp = [&](int s) {
        const uint32_t qo = (s & 1) * 32768;
#pragma unroll
        for (int ks = 0; ks < 16; ++ks)
          mma_ts_p(tmem + C::COL_DP, tmem + C::COL_VA + ks * 8, desc_add(dOk, qo + (ks >> 2) * 8192 + (ks & 3) * 32),
                   idS, ks > 0, leader);
        mma_commit_p(&bars->dp_full, leader);
      };
      // dV_h += P^T dO[:, h] and dK_h += dS^T Q[:, h] (K dimension = 64 queries: 4 k-steps;
      // P^T / dS^T of queries 16k..16k+15 at columns (k >> 1) * 32 + (k & 1) * 8)
      auto issue_dvdk = [&](int s) {
        const uint32_t qo = (s & 1) * 32768 + hh * 2 * 8192;
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const uint32_t acc = (s > 0 || kq > 0) ? 1u : 0u;
          const uint32_t pcol = (kq >> 1) * 32 + (kq & 1) * 8;
          mma_ts_p(tmem + C::COL_DV, tmem + C::COL_S + pcol, desc_add(dOm, qo + kq * 2048), idKV, acc, leader);
          mma_ts_p(tmem + C::COL_DK, tmem + C::COL_DP + pcol, desc_add(dQm, qo + kq * 2048), idKV, acc, leader);
        }
        mma_commit_p(&bars->qdo_empty[s & 1], leader);
      };
      // dQ^T_h = K[:, h]^T dS^T: M = 128 d-columns, N = 64 queries, K = 128 keys (8 k-steps)
      auto issue_dq = [&]() {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss_p(tmem + C::COL_DP, desc_add(dKm, hh * 2 * 16384 + ks * 2048), desc_add(dSm, ks * 2048), idQT,
                   ks > 0, leader);
        mma_commit_p(&bars->dq_full, leader);
      };
      bool ok = warp_wait(&bars->kv_full, 0, p.wait_ns, abort_flag, 310) &&
                warp_wait(&bars->v_tmem, 0, p.wait_ns, abort_flag, 311) &&
                warp_wait(&bars->qdo_full[0], 0, p.wait_ns, abort_flag, 312);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int s = 0; s < n_steps && ok; ++s) {
        if (!(ok = warp_wait(&bars->ds_ready, s & 1, p.wait_ns, abort_flag, 313))) break;
        tc_fence_after();
        issue_dvdk(s);
        // dQ^T of this step next (it reads dS^T from shared memory and writes over dS^T in
        // TMEM after dK has read it: the MMAs run in issue order), so that its drain runs
        // while S^T of the next step is computed
        issue_dq();
        // S^T of the next step may overwrite P^T now
        if (s + 1 < n_steps) {
          if (!(ok = warp_wait(&bars->qdo_full[(s + 1) & 1], ((s + 1) >> 1) & 1, p.wait_ns, abort_flag, 314))) break;
          tc_fence_after();
          issue_s(s + 1);
        }
        if (s + 1 < n_steps) {
          // dP^T of the next step overwrites dQ^T: wait for its drain
          if (!(ok = warp_wait(&bars->dq_free, s & 1, p.wait_ns, abort_flag, 315))) break;
          tc_fence_after();
          issue_dp(s + 1);
        }
      }
      if (ok) mma_commit_p(&bars->dkdv_full, leader);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------------------------------------------------------- softmax-gradient
    const int wc = (warp - 4) >> 2;  // queries [32 wc, 32 wc + 32) of the step
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // key within the tile == TMEM lane
    const int key = k0 + r;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const int q0 = 32 * wc;
    const float sl2 = p.scale_log2, scale = p.scale;
    bool ok = true;
    if (n_steps > 0) {
      // V row r (staged in the dO buffers as four [128][64] swizzled blocks) into TMEM lane r:
      // warps 4-7 take d-columns [0, 128), warps 8-11 [128, 256)
      ok = warp_wait(&bars->kv_full, 0, p.wait_ns, abort_flag, 320);
      if (ok) {
#pragma unroll 1
        for (int kb = 2 * wc; kb < 2 * wc + 2; ++kb) {
          const uint8_t* row = smem + C::OFF_DO + kb * 16384 + r * 128;
          uint32_t a[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 x = *reinterpret_cast<const uint4*>(row + ((u ^ (r & 7)) << 4));
            a[4 * u] = x.x;
            a[4 * u + 1] = x.y;
            a[4 * u + 2] = x.z;
            a[4 * u + 3] = x.w;
          }
          tmem_st32(tmem + lane_off + C::COL_VA + kb * 32, a);
        }
        tmem_wait_st();
        fence_proxy_async_smem();  // these reads precede the TMA writes of dO into the buffers
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->v_tmem);
      }
    }
    for (int s = 0; s < n_steps && ok; ++s) {
      const int st = s & 1;
      const int i = i_begin + s % n_i;
      // P first, as soon as S^T has landed (the tensor core is meanwhile computing dP^T),
      // then dS once dP^T has
      ok = warp_wait(&bars->qdo_full[st], (s >> 1) & 1, p.wait_ns, abort_flag, 321) &&
           warp_wait(&bars->s_full, s & 1, p.wait_ns, abort_flag, 322);
      if (!ok) break;
      tc_fence_after();
      int lim = 0;  // columns q < lim of this warp's 32 are masked for this key
      if (key >= p.Nkv) lim = 32;
      else if (CAUSAL) lim = min(32, max(0, key - off - i * C::BM - q0));
      const float* lse_s = reinterpret_cast<const float*>(smem + C::OFF_STAT + st * 512) + q0;
      const float* d_s = lse_s + 64;
      const bool any_masked = __any_sync(0xffffffffu, lim > 0);
      uint8_t* dsrow = smem + C::OFF_DS + r * 128;
      float pr[32];  // P of this key and the warp's 32 queries
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[16];
        tmem_ld16(tmem + lane_off + C::COL_S + q0 + 16 * c, sv);
        tmem_wait_ld();
        uint32_t pp[8];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse_s + 16 * c + e);
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
          pr[16 * c + e] = p01.x;
          pr[16 * c + e + 1] = p01.y;
          pr[16 * c + e + 2] = p23.x;
          pr[16 * c + e + 3] = p23.y;
          pp[e / 2] = pack_bf16x2(p01.x, p01.y);
          pp[e / 2 + 1] = pack_bf16x2(p23.x, p23.y);
        }
        // packed P^T of queries 16k..16k+15 at columns (k >> 1) * 32 + (k & 1) * 8
        tmem_st8(tmem + lane_off + C::COL_S + q0 + 8 * c, pp);
      }
      if (!(ok = warp_wait(&bars->dp_full, s & 1, p.wait_ns, abort_flag, 324))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dv[16];
        tmem_ld16(tmem + lane_off + C::COL_DP + q0 + 16 * c, dv);
        tmem_wait_ld();
        uint32_t pd[8];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(d_s + 16 * c + e);
          // dS * scale = P * (dP * scale - D * scale)  (d4 holds D * scale)
          const float2 g01 = __fmul2_rn(
              make_float2(pr[16 * c + e], pr[16 * c + e + 1]),
              __ffma2_rn(make_float2(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])), make_float2(scale, scale),
                         make_float2(-d4.x, -d4.y)));
          const float2 g23 = __fmul2_rn(
              make_float2(pr[16 * c + e + 2], pr[16 * c + e + 3]),
              __ffma2_rn(make_float2(__uint_as_float(dv[e + 2]), __uint_as_float(dv[e + 3])), make_float2(scale, scale),
                         make_float2(-d4.z, -d4.w)));
          pd[e / 2] = pack_bf16x2(g01.x, g01.y);
          pd[e / 2 + 1] = pack_bf16x2(g23.x, g23.y);
        }
        // packed dS^T at the same columns, over dP^T
        tmem_st8(tmem + lane_off + C::COL_DP + q0 + 8 * c, pd);
        // dS^T row r: [64 queries] of 128 bytes, 16-byte unit q/8 at unit ^ (r % 8)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int unit = wc * 4 + 2 * c + u;
          *reinterpret_cast<uint4*>(dsrow + ((unit ^ (r & 7)) * 16)) =
              make_uint4(pd[4 * u], pd[4 * u + 1], pd[4 * u + 2], pd[4 * u + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();  // dS^T written by the generic proxy, read by the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready);
    }
    // ---- dK[:, h] (warps 4-7) and dV[:, h] (warps 8-11); the scale is already in dS
    const uint32_t col = wc == 0 ? C::COL_DK : C::COL_DV;
    void* dst = wc == 0 ? p.dk : p.dv;
    const size_t base = (size_t(bk) * p.Nkv + key) * C::D + hh * C::DH;
    if (ok && n_steps > 0) ok = warp_wait(&bars->dkdv_full, 0, p.wait_ns, abort_flag, 323);
    if (ok && n_steps > 0) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < C::DH / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + col + c * 32, v);
        tmem_wait_ld();
        if (key < p.Nkv) {
          if (p.grad_bf16) {
            uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + base + c * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              o4[q4] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q4]), __uint_as_float(v[8 * q4 + 1])),
                                  pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3])),
                                  pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5])),
                                  pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7])));
          } else {
            float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(dst) + base + c * 32);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              o4[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                   __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
          }
        }
      }
    } else if (n_steps == 0 && key < p.Nkv) {
      // no query row can see these keys: their gradients are zero
      for (int c = 0; c < C::DH; c += 4) {
        if (p.grad_bf16)
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(dst) + base + c) = make_uint2(0, 0);
        else
          *reinterpret_cast<float4*>(static_cast<float*>(dst) + base + c) = make_float4(0, 0, 0, 0);
      }
    }
  } else if (warp >= 12) {
    // ---------------------------------------------------------------- dQ^T drain
    // Thread r holds d-column h * 128 + r of the step's 64 queries.  The warp reads all 64
    // columns from TMEM, releases them (the next step's dP^T may overwrite them), then for
    // each half of the queries writes a transposed [32 queries][32 d] fp32 tile (each query a
    // 128-byte row, 128-byte swizzle) and adds it into the fp32 accumulator with a TMA
    // reduce-add.
    const int wq = warp & 3;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    uint8_t* stg = smem + C::OFF_DQS + wq * 4096;
    bool ok = true;
    for (int s = 0; s < n_steps && ok; ++s) {
      ok = warp_wait(&bars->dq_full, s & 1, p.wait_ns, abort_flag, 330);
      if (!ok) break;
      tc_fence_after();
      const int h = hk * G + s / n_i, i = i_begin + s % n_i;
      uint32_t v0[32], v1[32];
      tmem_ld32(tmem + lane_off + C::COL_DP, v0);
      tmem_ld32(tmem + lane_off + C::COL_DP + 32, v1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_free);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (lane == 0) bulk_wait_read();  // the previous reduce-add has read the staging
        __syncwarp();
#pragma unroll
        for (int e = 0; e < 32; ++e)
          *reinterpret_cast<uint32_t*>(stg + e * 128 + (((lane >> 2) ^ (e & 7)) << 4) + (lane & 3) * 4) =
              c == 0 ? v0[e] : v1[e];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tmDQ, stg, hh * C::DH + wq * 32, i * C::BM + 32 * c, b * p.Hq + h);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // the reduce-adds complete before exit
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
