// fwd_d256.cuh — bf16 forward for head dimension 256 on the 5th-generation tensor cores.
//
// Same result as fa_fwd_bf16_kernel: O = softmax(Q K^T * scale) V and lse = m + ln(l) per
// query row ("Autoatención, kernels CUDA y FlashAttention" §1), tile by tile with the
// online-softmax recurrence of "FlashAttention" (paweldubiel.com notes, "No basta con
// promediar los resultados de los bloques"; the reference maximum moves lazily as in the
// d <= 128 kernel), never writing the score matrix to device memory.
//
// At d = 256 one 128-row output accumulator fills 256 of the 512 TMEM columns, so a CTA
// holds ONE query tile (not the d <= 128 kernel's two).  The tensor core is kept busy by
// double-buffering the score tile instead: S for key tile j+1 is computed into one
// 64-column buffer while the softmax works on tile j in the other.
// TMEM: S/P buffers at columns [0, 64) and [64, 128), Q at [128, 256) (bf16 pairs, the A
// operand of S = Q K^T, so that S reads only K from shared memory), O at [256, 512).
// Shared memory: Q (64 KB, four 64-column blocks), two K/V stages of 64 keys (32 KB each
// for K and V), per-warp epilogue staging.
//   warp 0      TMA producer (one thread)
//   warp 1      MMA issuer (one thread)
//   warps 4-7   softmax + epilogue (one query row per thread = one TMEM lane)
// Work items: one 128-row query tile of one (batch, head); causal items longest first,
// non-causal items head-major (as the d <= 128 kernel).
#pragma once
#include "common.cuh"
#include "fwd_bf16.cuh"

namespace fa {

struct D256Cfg {
  static constexpr int D = 256;
  static constexpr int BM = 128;
  static constexpr int BN = 64;
  static constexpr int KB = D / 64;
  static constexpr int Q_TILE = BM * D * 2;   // 64 KB
  static constexpr int KV_TILE = BN * D * 2;  // 32 KB
  static constexpr int NSTAGE = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_TILE;
  static constexpr int OFF_V = OFF_K + NSTAGE * KV_TILE;
  static constexpr int OFF_STG = OFF_V + NSTAGE * KV_TILE;  // 4 KB per softmax warp
  static constexpr int OFF_BAR = OFF_STG + 4 * 4096;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int THREADS = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0;  // + (tile & 1) * BN
  static constexpr uint32_t COL_QA = 128;
  static constexpr uint32_t COL_O = 256;
};

struct D256Bars {
  uint64_t q_full, q_empty;  // Q in shared memory loaded / copied out (4 softmax warps arrive)
  uint64_t q_tmem;           // Q copied into TMEM (4 softmax warps arrive)
  uint64_t q_tmem_free;      // the item's last S, the last reader of Q in TMEM, has run
  uint64_t k_full[2], v_full[2];
  uint64_t k_empty[2];  // the S that read a K stage has completed
  uint64_t v_empty[2];  // the P.V that read a V stage has completed
  uint64_t s_full[2];  // per S buffer
  uint64_t p_full;     // P of the current tile written (4 softmax warps)
  uint64_t o_ready;    // the P.V of a tile has completed (one completion per tile)
  uint64_t o_final;    // the item's last P.V has completed
  uint32_t tmem_base;
  int abort_flag;
};

template <bool CAUSAL>
__global__ void __launch_bounds__(D256Cfg::THREADS, 1)
    fa_fwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const FwdBf16Params p) {
  using C = D256Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  D256Bars* bars = reinterpret_cast<D256Bars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = warp_id(), lane = lane_id();
  const int n_qt = (p.Nq + C::BM - 1) / C::BM;
  const int n_items = n_qt * p.BH;
  const int off = p.Nkv - p.Nq;  // bottom-right causal alignment
  auto item_qt = [&](int it) { return CAUSAL ? n_qt - 1 - it / p.BH : it % n_qt; };
  auto item_bh = [&](int it) { return CAUSAL ? it % p.BH : it / n_qt; };
  // this CTA's k-th item: boustrophedon order over the longest-first causal items,
  // round-robin over the equal non-causal ones
  auto item_at = [&](int k) {
    return CAUSAL ? snake_item(k, int(blockIdx.x), int(gridDim.x)) : int(blockIdx.x) + k * int(gridDim.x);
  };
  auto item_ntiles = [&](int qt) {
    const int kv_end = CAUSAL ? min(p.Nkv, min(qt * C::BM + C::BM, p.Nq) + off) : p.Nkv;
    return (kv_end + C::BN - 1) / C::BN;
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 4);
    mbar_init(&bars->q_tmem, 4);
    mbar_init(&bars->q_tmem_free, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
    }
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->o_ready, 1);
    mbar_init(&bars->o_final, 1);
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

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int kv = 0, local = 0;
      bool ok = true;
      for (int k = 0, it = item_at(0); it < n_items && ok; it = item_at(++k), ++local) {
        const int qt = item_qt(it), bh = item_bh(it), n = item_ntiles(qt);
        const int zkv = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / (p.Hq / p.Hkv);
        if (local > 0 && !(ok = mbar_wait(&bars->q_empty, (local - 1) & 1, p.wait_ns, abort_flag, 211))) break;
        mbar_arrive_expect_tx(&bars->q_full, C::Q_TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(smem + C::OFF_Q + kb * C::BM * 128, &tmQ, &bars->q_full, kb * 64, qt * C::BM, bh);
        for (int j = 0; j < n; ++j, ++kv) {
          // K and V stages are released separately: a K stage as soon as the S that read it
          // has run.  S of tile j + 2 is issued right after the P.V of tile j, so a K stage
          // freed only by that P.V (as the V stage is) would make every S wait for its load.
          const int st = kv & 1, round = kv >> 1;
          if (round > 0 && !(ok = mbar_wait(&bars->k_empty[st], (round - 1) & 1, p.wait_ns, abort_flag, 210)))
            break;
          mbar_arrive_expect_tx(&bars->k_full[st], C::KV_TILE);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_3d(smem + C::OFF_K + st * C::KV_TILE + kb * C::BN * 128, &tmK, &bars->k_full[st], kb * 64,
                        j * C::BN, zkv);
          if (round > 0 && !(ok = mbar_wait(&bars->v_empty[st], (round - 1) & 1, p.wait_ns, abort_flag, 213)))
            break;
          mbar_arrive_expect_tx(&bars->v_full[st], C::KV_TILE);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_3d(smem + C::OFF_V + st * C::KV_TILE + kb * C::BN * 128, &tmV, &bars->v_full[st], kb * 64,
                        j * C::BN, zkv);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, C::BN, 0);  // K-major Q and K
      constexpr uint32_t idPV = idesc_bf16_f32(128, C::D, 1);  // V is MN-major
      const uint32_t sK = smem_u32(smem + C::OFF_K);
      const uint32_t sV = smem_u32(smem + C::OFF_V);
      // S of key tile g (global tile count) into buffer g & 1
      auto issue_S = [&](int st, int g) {
#pragma unroll
        for (int ks = 0; ks < C::D / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;
          mma_ts(tmem + C::COL_S + (g & 1) * C::BN, tmem + C::COL_QA + ks * 8,
                 sdesc_sw128(sK + st * C::KV_TILE + kb * C::BN * 128 + kin * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[g & 1]);
        mma_commit(&bars->k_empty[st]);
      };
      int kv = 0, g = 0, local = 0;
      bool ok = true;
      for (int k = 0, it = item_at(0); it < n_items && ok; it = item_at(++k), ++local) {
        const int n = item_ntiles(item_qt(it));
        ok = mbar_wait(&bars->q_tmem, local & 1, p.wait_ns, abort_flag, 220) &&
             mbar_wait(&bars->k_full[kv & 1], (kv >> 1) & 1, p.wait_ns, abort_flag, 221);
        if (!ok) break;
        tc_fence_after();
        issue_S(kv & 1, g);
        if (n == 1) mma_commit(&bars->q_tmem_free);
        for (int j = 0; j < n; ++j, ++kv, ++g) {
          const int st = kv & 1;
          if (j + 1 < n) {
            // the next tile's scores, while the softmax works on this one
            if (!(ok = mbar_wait(&bars->k_full[st ^ 1], ((kv + 1) >> 1) & 1, p.wait_ns, abort_flag, 222))) break;
            tc_fence_after();
            issue_S(st ^ 1, g + 1);
            if (j + 2 == n) mma_commit(&bars->q_tmem_free);  // the item's last S
          }
          ok = mbar_wait(&bars->v_full[st], (kv >> 1) & 1, p.wait_ns, abort_flag, 223) &&
               mbar_wait(&bars->p_full, g & 1, p.wait_ns, abort_flag, 224);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < C::BN / 16; ++ks)
            mma_ts(tmem + C::COL_O, tmem + C::COL_S + (g & 1) * C::BN + ks * 8,
                   sdesc_sw128(sV + st * C::KV_TILE + ks * 16 * 128, C::BN * 128, 1024), idPV,
                   (j > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&bars->v_empty[st]);
          mma_commit(&bars->o_ready);
          if (j + 1 == n) mma_commit(&bars->o_final);
        }
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax + epilogue
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::COL_O;
    const float sl2 = p.scale_log2;
    const float2 sl2v = make_float2(sl2, sl2);
    // Q of the CTA's item number `lq` from shared memory into TMEM: row r (TMEM lane r) as
    // 128 columns of bf16 pairs in d order, the A-operand layout of the TS MMA.  Every warp
    // copies its 32 rows, idle or not.  Item lq's copy waits for item lq - 1's last S.
    auto copy_q = [&](int lq) -> bool {
      if (lq > 0 && !warp_wait(&bars->q_tmem_free, (lq - 1) & 1, p.wait_ns, abort_flag, 234)) return false;
      if (!warp_wait(&bars->q_full, lq & 1, p.wait_ns, abort_flag, 235)) return false;
      tc_fence_after();
#pragma unroll 1
      for (int kb = 0; kb < C::KB; ++kb) {
        const uint8_t* qrow = smem + C::OFF_Q + kb * C::BM * 128 + r * 128;  // 128-byte swizzle
        uint32_t a[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 x = *reinterpret_cast<const uint4*>(qrow + ((u ^ (r & 7)) << 4));
          a[4 * u] = x.x;
          a[4 * u + 1] = x.y;
          a[4 * u + 2] = x.z;
          a[4 * u + 3] = x.w;
        }
        tmem_st32(tmem + lane_off + C::COL_QA + kb * 32, a);
      }
      tmem_wait_st();
      fence_proxy_async_smem();  // these reads precede the TMA writes of the next Q
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->q_tmem);
        mbar_arrive(&bars->q_empty);
      }
      return true;
    };
    int g = 0, local = 0;
    bool ok = item_at(0) < n_items ? copy_q(0) : true;
    for (int k = 0, it = item_at(0); it < n_items && ok; it = item_at(++k), ++local) {
      const int qt = item_qt(it), bh = item_bh(it), n = item_ntiles(qt);
      const int row = qt * C::BM + r;
      const int row_limit = CAUSAL ? min(p.Nkv, row + off + 1) : p.Nkv;
      const bool idle = __all_sync(0xffffffffu, row >= p.Nq);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j, ++g) {
        if (!(ok = warp_wait(&bars->s_full[g & 1], (g >> 1) & 1, p.wait_ns, abort_flag, 230))) break;
        if (!idle) {
          tc_fence_after();
          const uint32_t tS = tmem + lane_off + C::COL_S + (g & 1) * C::BN;
          uint32_t sr[C::BN];
          tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_wait_ld();
          float f[C::BN];
          const int lim = row_limit - j * C::BN;  // columns >= lim are masked for this row
#pragma unroll
          for (int c = 0; c < C::BN; ++c) f[c] = (c < lim) ? __uint_as_float(sr[c]) : -INFINITY;
          float mx8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(f[k], f[8 + k]);
#pragma unroll
          for (int c = 16; c < C::BN; c += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], f[c + k], f[c + 8 + k]);
          const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                                 fmaxf(fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
          // lazy reference maximum, as in the d <= 128 kernel (u / l does not depend on it)
          const float m_cand = fmaxf(m, mx * sl2);
          const float m_new = (m_cand > m + FA_RESCALE_LOG2) ? m_cand : m;
          const float base = (m_new == -INFINITY) ? 0.f : m_new;
          const float alpha = (m_new == m) ? 1.f : ex2(m - base);
          const float2 nbase = make_float2(-base, -base);
          float2 rs0 = make_float2(0.f, 0.f), rs1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < C::BN / 32; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int k = c * 32 + 2 * i;
              const float2 x = __ffma2_rn(make_float2(f[k], f[k + 1]), sl2v, nbase);
              const float2 pv = make_float2(k < lim ? ex2(x.x) : 0.f, k + 1 < lim ? ex2(x.y) : 0.f);
              if (i & 1)
                rs1 = __fadd2_rn(rs1, pv);
              else
                rs0 = __fadd2_rn(rs0, pv);
              pk[i] = pack_bf16x2(pv.x, pv.y);
            }
            tmem_st16(tS + c * 16, pk);
          }
          const float2 rs = __fadd2_rn(rs0, rs1);
          l = l * alpha + (rs.x + rs.y);
          // u (TMEM) holds the P.V sums of tiles < j: rescale its rows whose reference rose,
          // once the previous tile's P.V has landed
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            if (!(ok = warp_wait(&bars->o_ready, (g - 1) & 1, p.wait_ns, abort_flag, 231))) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < C::D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])),
                                            make_float2(alpha, alpha));
                o[i] = __float_as_uint(v.x);
                o[i + 1] = __float_as_uint(v.y);
              }
              tmem_st32(tO + c * 32, o);
            }
          }
          tmem_wait_st();
          m = m_new;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full);
      }
      if (!ok) break;
      // the next item's Q goes into TMEM now (this item's last S has run), so its first S
      // overlaps this item's epilogue
      if (item_at(k + 1) < n_items && !(ok = copy_q(local + 1))) break;
      if (!(ok = warp_wait(&bars->o_final, local & 1, p.wait_ns, abort_flag, 232))) break;
      if (idle) continue;
      tc_fence_after();
      // O = u / l through per-warp staging (32 rows x 64 columns, 128-byte swizzle) and TMA
      // stores, which drop the rows past Nq
      const float inv = 1.f / l;
      uint8_t* stg = smem + C::OFF_STG + (warp - 4) * 4096;
      const int row0 = qt * C::BM + wq * 32;
#pragma unroll 1
      for (int c = 0; c < C::D / 64; ++c) {
        uint32_t o[64];
        tmem_ld32(tO + c * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
        tmem_ld32(tO + c * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
        tmem_wait_ld();
        if (lane == 0) bulk_wait_read();
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float2 a = __fmul2_rn(make_float2(__uint_as_float(o[8 * u]), __uint_as_float(o[8 * u + 1])),
                                      make_float2(inv, inv));
          const float2 b2 = __fmul2_rn(make_float2(__uint_as_float(o[8 * u + 2]), __uint_as_float(o[8 * u + 3])),
                                       make_float2(inv, inv));
          const float2 c2 = __fmul2_rn(make_float2(__uint_as_float(o[8 * u + 4]), __uint_as_float(o[8 * u + 5])),
                                       make_float2(inv, inv));
          const float2 d2 = __fmul2_rn(make_float2(__uint_as_float(o[8 * u + 6]), __uint_as_float(o[8 * u + 7])),
                                       make_float2(inv, inv));
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((u ^ (lane & 7)) << 4)) =
              make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(b2.x, b2.y), pack_bf16x2(c2.x, c2.y),
                         pack_bf16x2(d2.x, d2.y));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmO, stg, c * 64, row0, bh);
          bulk_commit();
        }
      }
      if (row < p.Nq) p.lse[size_t(bh) * p.Nq + row] = (m + __log2f(l)) * 0.69314718055994531f;
    }
    if (lane == 0) bulk_wait_all();
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
