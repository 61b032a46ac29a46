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
// 128-column buffer while the softmax works on tile j in the other.  128-key tiles keep
// the S MMA at N = 128 (an N = 64 MMA runs at about 70 % of that rate).
// TMEM: S/P buffers at columns [0, 128) and [128, 256), O at [256, 512).
// Shared memory: Q (64 KB, four 64-column blocks) and a ring of NSLOT pieces of 32 KB, each
// one half (128 of the 256 head-dimension columns) of a 128-key K or V tile.  The pieces go
// through the ring in the order the MMAs consume them: for each item K_0, then per tile j
// K_{j+1} (S_{j+1} is computed while the softmax works on tile j) and V_j.
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
  static constexpr int BM = 128;   // query rows per item
  static constexpr int BN = 128;   // keys per tile
  static constexpr int DH = 128;   // head-dimension columns per K or V piece
  static constexpr int KB = D / 64;
  static constexpr int Q_TILE = BM * D * 2;  // 64 KB
  static constexpr int PIECE = BN * DH * 2;  // 32 KB: [2 blocks of 64 columns][128 keys][128 B]
  static constexpr int NSLOT = 5;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = Q_TILE;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * PIECE;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int THREADS = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0;  // + (tile & 1) * BN
  static constexpr uint32_t COL_O = 256;
};

struct D256Bars {
  uint64_t q_full, q_empty;
  uint64_t slot_full[D256Cfg::NSLOT];   // a piece has landed
  uint64_t slot_empty[D256Cfg::NSLOT];  // the MMAs that read a piece have run
  uint64_t s_full[2];  // per S buffer
  // P of a tile written (4 softmax warps), one barrier per S buffer: with the scores double
  // buffered, a warp with no rows to process can finish tile j + 1 before another warp has
  // finished tile j, and on one shared barrier its early arrival would complete tile j's
  // phase.  Per buffer, a warp is at most one tile ahead (S of tile j + 2 waits for tile j's
  // P.V, which waits for every warp's P of tile j).
  uint64_t p_full[2];
  uint64_t o_ready;    // the P.V of a tile has completed (one completion per tile)
  uint64_t o_final;    // the item's last P.V has completed
  uint32_t tmem_base;
  int abort_flag;
};

template <bool CAUSAL>
__global__ void __launch_bounds__(D256Cfg::THREADS, 1)
    fa_fwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdBf16Params p) {
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
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&bars->slot_full[s], 1);
      mbar_init(&bars->slot_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(&bars->s_full[s], 1);
    for (int s = 0; s < 2; ++s) mbar_init(&bars->p_full[s], 4);
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
      int pc = 0, local = 0;  // pieces issued so far (ring position), items started
      bool ok = true;
      // half h (head-dimension columns [128 h, 128 h + 128)) of key tile j of K or V
      auto load_piece = [&](const CUtensorMap* tm, int j, int h, int zkv) -> bool {
        const int slot = pc % C::NSLOT, round = pc / C::NSLOT;
        if (round > 0 && !mbar_wait(&bars->slot_empty[slot], (round - 1) & 1, p.wait_ns, abort_flag, 210))
          return false;
        uint8_t* dst = smem + C::OFF_RING + slot * C::PIECE;
        mbar_arrive_expect_tx(&bars->slot_full[slot], C::PIECE);
        for (int b = 0; b < 2; ++b)
          tma_load_3d(dst + b * C::BN * 128, tm, &bars->slot_full[slot], (2 * h + b) * 64, j * C::BN, zkv);
        ++pc;
        return true;
      };
      for (int k = 0, it = item_at(0); it < n_items && ok; it = item_at(++k), ++local) {
        const int qt = item_qt(it), bh = item_bh(it), n = item_ntiles(qt);
        const int zkv = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / (p.Hq / p.Hkv);
        if (local > 0 && !(ok = mbar_wait(&bars->q_empty, (local - 1) & 1, p.wait_ns, abort_flag, 211))) break;
        mbar_arrive_expect_tx(&bars->q_full, C::Q_TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(smem + C::OFF_Q + kb * C::BM * 128, &tmQ, &bars->q_full, kb * 64, qt * C::BM, bh);
        ok = load_piece(&tmK, 0, 0, zkv) && load_piece(&tmK, 0, 1, zkv);
        for (int j = 0; j < n && ok; ++j) {
          if (j + 1 < n) ok = load_piece(&tmK, j + 1, 0, zkv) && load_piece(&tmK, j + 1, 1, zkv);
          ok = ok && load_piece(&tmV, j, 0, zkv) && load_piece(&tmV, j, 1, zkv);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, C::BN, 0);   // K-major Q and K, N = 128 keys
      constexpr uint32_t idPV = idesc_bf16_f32(128, C::DH, 1);  // V MN-major, N = 128 columns
      const uint32_t sQ = smem_u32(smem + C::OFF_Q), sRing = smem_u32(smem + C::OFF_RING);
      int pc = 0, g = 0, local = 0;  // pieces consumed, tiles, items
      bool ok = true;
      auto wait_piece = [&]() {
        return mbar_wait(&bars->slot_full[pc % C::NSLOT], (pc / C::NSLOT) & 1, p.wait_ns, abort_flag, 221);
      };
      // S of tile gg (global count) into buffer gg & 1: 8 k-steps over each K half
      auto issue_S = [&](int gg) -> bool {
        for (int h = 0; h < 2; ++h) {
          if (!wait_piece()) return false;
          tc_fence_after();
          const uint32_t sk = sRing + (pc % C::NSLOT) * C::PIECE;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int ks = h * 8 + kk;  // k-step over the 256 columns
            mma_ss(tmem + C::COL_S + (gg & 1) * C::BN,
                   sdesc_sw128(sQ + (ks >> 2) * C::BM * 128 + (ks & 3) * 32, 16, 1024),
                   sdesc_sw128(sk + (kk >> 2) * C::BN * 128 + (kk & 3) * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
          }
          mma_commit(&bars->slot_empty[pc % C::NSLOT]);
          ++pc;
        }
        mma_commit(&bars->s_full[gg & 1]);
        return true;
      };
      // O[:, 128 h .. 128 h + 128) += P V[:, half h] for tile gg: 8 k-steps of 16 keys each
      auto issue_PV = [&](int gg, int j) -> bool {
        for (int h = 0; h < 2; ++h) {
          if (!wait_piece()) return false;
          tc_fence_after();
          const uint32_t sv = sRing + (pc % C::NSLOT) * C::PIECE;
#pragma unroll
          for (int ks = 0; ks < C::BN / 16; ++ks)
            mma_ts(tmem + C::COL_O + h * C::DH, tmem + C::COL_S + (gg & 1) * C::BN + ks * 8,
                   sdesc_sw128(sv + ks * 16 * 128, C::BN * 128, 1024), idPV, (j > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&bars->slot_empty[pc % C::NSLOT]);
          ++pc;
        }
        return true;
      };
      for (int k = 0, it = item_at(0); it < n_items && ok; it = item_at(++k), ++local) {
        const int n = item_ntiles(item_qt(it));
        if (!(ok = mbar_wait(&bars->q_full, local & 1, p.wait_ns, abort_flag, 220))) break;
        tc_fence_after();
        if (!(ok = issue_S(g))) break;
        if (n == 1) mma_commit(&bars->q_empty);
        for (int j = 0; j < n; ++j, ++g) {
          if (j + 1 < n) {
            // the next tile's scores, while the softmax works on this one
            if (!(ok = issue_S(g + 1))) break;
            if (j + 2 == n) mma_commit(&bars->q_empty);  // the item's last S
          }
          if (!(ok = mbar_wait(&bars->p_full[g & 1], (g >> 1) & 1, p.wait_ns, abort_flag, 224))) break;
          tc_fence_after();
          if (!(ok = issue_PV(g, j))) break;
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
    int g = 0, local = 0;
    bool ok = true;
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
#pragma unroll
          for (int c = 0; c < C::BN / 32; ++c)
            tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
          tmem_wait_ld();
          float f[C::BN];
          const int lim = row_limit - j * C::BN;  // columns >= lim are masked for this row
#pragma unroll
          for (int c = 0; c < C::BN; ++c) f[c] = (c < lim) ? __uint_as_float(sr[c]) : -INFINITY;
          float mx8[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) mx8[q] = fmaxf(f[q], f[8 + q]);
#pragma unroll
          for (int c = 16; c < C::BN; c += 16)
#pragma unroll
            for (int q = 0; q < 8; ++q) mx8[q] = fmax3(mx8[q], f[c + q], f[c + 8 + q]);
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
              const int q = c * 32 + 2 * i;
              const float2 x = __ffma2_rn(make_float2(f[q], f[q + 1]), sl2v, nbase);
              const float2 pv = make_float2(q < lim ? ex2(x.x) : 0.f, q + 1 < lim ? ex2(x.y) : 0.f);
              if (i & 1)
                rs1 = __fadd2_rn(rs1, pv);
              else
                rs0 = __fadd2_rn(rs0, pv);
              pk[i] = pack_bf16x2(pv.x, pv.y);
            }
            // P (bf16 pairs) over the scores already read: columns [16 c, 16 c + 16)
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
        if (lane == 0) mbar_arrive(&bars->p_full[g & 1]);
      }
      if (!ok) break;
      if (!(ok = warp_wait(&bars->o_final, local & 1, p.wait_ns, abort_flag, 232))) break;
      if (idle) continue;
      tc_fence_after();
      // O = u / l, the thread's row straight to device memory (rows past Nq are not written)
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.o + (size_t(bh) * p.Nq + row) * C::D;
#pragma unroll 1
      for (int c = 0; c < C::D / 64; ++c) {
        uint32_t o[64];
        tmem_ld32(tO + c * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
        tmem_ld32(tO + c * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
        tmem_wait_ld();
        if (row < p.Nq) {
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
            *reinterpret_cast<uint4*>(orow + c * 64 + 8 * u) =
                make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(b2.x, b2.y), pack_bf16x2(c2.x, c2.y),
                           pack_bf16x2(d2.x, d2.y));
          }
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
