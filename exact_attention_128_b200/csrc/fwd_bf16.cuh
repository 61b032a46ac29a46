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
// Persistent kernel: CTAs walk work items (two 128-row query tiles Q0, Q1 of one (batch,
// query head)), item = blockIdx.x + k * gridDim.x, ordered head-major (non-causal: K/V
// reuse in L2); causal items go in head-major units of a long and a short item of equal
// total length (paged causal: requests in L2-sized groups, longest first inside a group).
// Each item streams the 128-key tiles of its key/value head (GQA: head h reads
// h / (Hq/Hkv)).  The K/V ring and the Q buffers run ahead across item
// boundaries, so loads for the next item overlap the current item's tail and epilogue.
//   warp 0      TMA producer: Q0/Q1 per item (QBUF buffers), K_j and V_j into a ring.
//   warp 1      MMA issuer (the warp runs the role, one elected lane issues): S_t = Q_t K_j^T
//               into TMEM (SS MMA), then u_t += P_t V_j with P_t read from TMEM (TS MMA).
//   warps 4-7   softmax for Q0, warps 8-11 softmax for Q1: each thread owns one
//               query row = one TMEM lane; it reads S_t, updates (m, l), writes P_t
//               (bf16) over S_t in TMEM, rescales u_t in TMEM when m rose, and at the
//               end of an item writes O = u/l and lse.
// While one warpgroup runs the softmax of its tile, the tensor core works on the
// other tile, so the exponentials overlap the MMAs.  The Q buffer is released when an
// item's last S has been computed, so the next item's Q loads during its last tile.
//
// PAGED (fa_paged_prefill): the same roles over a paged KV cache.  Each request has its
// own key count and query-row count (its last positions); the producer warp gathers the
// K/V tiles block by block through the block table ("Atención tipo FlashAttention y
// atención paginada", the-ai.news).
//
// TMEM columns (d = 128, 512 allocated): S0 [0,128), S1 [128,256), u0 [256,256+D), u1
// after; d = 64 (256 allocated, two CTAs per SM): S0, S1, u0, u1 of 64 columns each.
// Shared memory: QBUF x (Q0, Q1), then NSTAGE K tiles and NSTAGE V tiles, each stored
// as D/64 column blocks of [rows x 128 bytes] with the 128-byte swizzle TMA writes and
// the MMA descriptors expect.
#pragma once
#include "common.cuh"

namespace fa {

// Lazy rescaling threshold (base-2 units) for the running reference maximum; see the
// softmax loop.  8 keeps every P <= 256, far inside bf16 and fp32 range.
#ifndef FA_RESCALE_LOG2
#define FA_RESCALE_LOG2 8.0f
#endif

// Two configurations:
//   BN = 128 (d = 128): 384 threads (softmax warps 4-11), 512 TMEM columns, one CTA/SM.
//   BN = 64  (d = 64):  320 threads (softmax warps 2-9), 256 TMEM columns and ~97 KB of
//            shared memory, so two CTAs share an SM and four query tiles are in flight;
//            at d = 64 the softmax, not the tensor core, sets the pace, and the second
//            CTA hides its latency.
// d = 64 kernel: K/V ring depth and the output columns a softmax warp stages per TMA store
// (64: 4 KB per warp, 128-byte swizzle; 32: 2 KB per warp, 64-byte swizzle, two stores).
// Measured on B200: 32-column staging 3-5 % faster (ViT-B/16 layer 34.8 -> 33.1 us, N = 4096
// causal 441 -> 426 us); 3 or 4 stages no faster than 2.
#ifndef FA_FWD_D64_NSTAGE
#define FA_FWD_D64_NSTAGE 2
#endif
#ifndef FA_FWD_D64_STG_COLS
#define FA_FWD_D64_STG_COLS 32
#endif

template <int D, int BN_>
struct FwdCfg {
  static constexpr int BM = 128;   // rows per query tile (two tiles per item)
  static constexpr int BN = BN_;   // keys per tile
  static constexpr int KB = D / 64;
  static constexpr int Q_TILE = BM * D * 2;
  static constexpr int KV_TILE = BN * D * 2;
  static constexpr int QBUF = (D == 128 || BN == 64) ? 1 : 2;
  static constexpr int NSTAGE = (BN == 64) ? FA_FWD_D64_NSTAGE : (D == 128 ? 2 : 4);
  static constexpr int STG_COLS = (BN == 64) ? FA_FWD_D64_STG_COLS : 64;
  static constexpr int STG_WARP = 32 * STG_COLS * 2;  // staging bytes per softmax warp
  static constexpr int OFF_Q = 0;  // + qb * 2 * Q_TILE + t * Q_TILE
  static constexpr int OFF_K = QBUF * 2 * Q_TILE;
  static constexpr int OFF_V = OFF_K + NSTAGE * KV_TILE;
  static constexpr int OFF_STG = OFF_V + NSTAGE * KV_TILE;  // epilogue staging, per softmax warp
  static constexpr int OFF_BAR = OFF_STG + 8 * STG_WARP;
  // paged causal prefill: the requests' order, longest first (PERM_MAX requests at most)
  static constexpr int PERM_MAX = 256;
  static constexpr int OFF_PERM = OFF_BAR + 256;
  static constexpr int END = OFF_PERM + 4 * PERM_MAX;
  static constexpr int WG0 = (BN == 64) ? 2 : 4;     // first softmax warp
  static constexpr int THREADS = 32 * (WG0 + 8);
  static constexpr int CTAS_PER_SM = (BN == 64) ? 2 : 1;
  // room for aligning the dynamic shared memory base up to 1024 bytes: up to 1 KB, less
  // when that is what lets CTAS_PER_SM blocks share the SM's 228 KB (1 KB of it reserved
  // per block); the kernel checks at run time that the slack it needs is there
  static constexpr int SMEM_CAP = 233472 / CTAS_PER_SM - 1024;
  static constexpr int SLACK = (SMEM_CAP - END) < 1024 ? (SMEM_CAP - END) : 1024;
  static_assert(SLACK >= 0, "shared memory over budget");
  static_assert(NSTAGE <= 4, "barrier arrays hold 4 stages");
  static_assert(8 * STG_WARP >= 4 * PERM_MAX, "the request lengths are sorted in the staging area");
  static constexpr int SMEM = END + SLACK;  // + barriers, request order, alignment slack
  static constexpr uint32_t TMEM_COLS = (BN == 64) ? 256 : 512;
  static constexpr uint32_t COL_S = 0;       // + t * BN
  static constexpr uint32_t COL_O = 2 * BN;  // + t * D
};

struct FwdBf16Params {
  __nv_bfloat16* o;
  float* lse;
  int BH, Hq, Hkv, Nq, Nkv;
  float scale_log2;  // scale * log2(e)
  uint64_t wait_ns;
  // paged mode (prefill over a paged KV cache): per-request lengths and the block table
  const int* bt;
  const int* ctx;   // cached tokens of request b (the keys)
  const int* qlen;  // query rows of request b (the last qlen positions of its sequence)
  int max_blocks, num_blocks;
  int group;  // paged causal: requests per group of the item order (>= 1)
};

struct FwdBars {
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t k_full[4];
  uint64_t v_full[4];
  uint64_t kv_empty[4];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_final[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, int BN, bool CAUSAL, bool PAGED>
__global__ void __launch_bounds__(FwdCfg<D, BN>::THREADS, FwdCfg<D, BN>::CTAS_PER_SM)
    fa_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const FwdBf16Params p) {
  using C = FwdCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (smem - smem_raw > C::SLACK) {  // (uniform over the CTA) the buffers would not fit
    if (threadIdx.x == 0) set_status(FA_ERR_UNSUPPORTED, 62);
    return;
  }
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = warp_id(), lane = lane_id();
  const int n_qp = (p.Nq + 2 * C::BM - 1) / (2 * C::BM);
  // Causal dense items come in units of two query-tile pairs of one head, qt and
  // n_qp - 1 - qt, whose key ranges add up to the same length for every unit; units are
  // head-major, so the CTAs running at the same time stream the K/V prefix of one or two
  // key/value heads and share it in L2, and each CTA runs whole units, which balances the
  // very unequal causal lengths.  Index it = 2 * unit + (0: the longer pair, 1: the
  // shorter); the middle pair of an odd n_qp has no partner (index 1 is empty).
  constexpr bool PAIRS = CAUSAL && !PAGED;
  const int n_units = (n_qp + 1) / 2;
  const int n_items = PAIRS ? 2 * n_units * p.BH : n_qp * p.BH;
  // index of this CTA's k-th item (>= n_items once it has none left), round-robin; paired
  // units go to one CTA whole
  auto item_index = [&](int k) {
    if constexpr (PAIRS) return 2 * (int(blockIdx.x) + (k >> 1) * int(gridDim.x)) + (k & 1);
    else return int(blockIdx.x) + k * int(gridDim.x);
  };
  // paged causal: the requests by query rows, longest first (filled after the grid
  // dependency wait below; with more than PERM_MAX requests the request order is kept)
  const int* s_perm = reinterpret_cast<const int*>(smem + C::OFF_PERM);
  // keys (L) and query rows (ql) of a sequence; paged mode reads them per request and
  // gives out-of-range lengths no work (flagging them in the status word)
  auto seq_len = [&](int bh, int& L, int& ql) {
    if constexpr (PAGED) {
      const int r = bh / p.Hq;
      L = __ldg(p.ctx + r);
      ql = __ldg(p.qlen + r);
      if (L < 1 || L > p.max_blocks * 16 || ql < 1 || ql > L || ql > p.Nq) {
        if (threadIdx.x == 0 && bh % p.Hq == 0) set_status(FA_ERR_INVALID_ARG, 60);
        L = 0;
        ql = 0;
      }
    } else {
      L = p.Nkv;
      ql = p.Nq;
    }
  };
  // item -> (query-tile pair qt, batch*head bh, its sequence's L and ql, key tiles n; n = 0:
  // nothing to do).  Non-causal items are head-major, so the CTAs running at the same time
  // share one or two heads' K/V in L2 (at N = 8192 this cut DRAM traffic per launch from
  // 4.2 GB to the 0.64 GB of the algorithm); causal items are the paired units above.  In
  // paged mode the causal items go by groups of p.group requests (the host sizes a group
  // so that its K/V stays in L2 while every query tile of the group reads it), the groups
  // and the requests inside them longest first; inside a group, rank k of the tile pairs
  // counted from each request's own last one, then the request, then the head: so the
  // long items of a group run first and its short ones fill the gaps at its end.
  struct Item {
    int qt, bh, L, ql, n;
  };
  auto item_of = [&](int it) {
    Item x;
    x.n = 0;
    if constexpr (PAIRS) {
      const int u = it >> 1, a = u % n_units;
      x.bh = u / n_units;
      seq_len(x.bh, x.L, x.ql);
      x.qt = (it & 1) ? a : n_qp - 1 - a;
      if ((it & 1) && x.qt == n_qp - 1 - a) return x;  // the unpaired middle pair
    } else if constexpr (CAUSAL) {  // paged (dense causal items are the paired units)
      const int n_req = p.BH / p.Hq, per_req = n_qp * p.Hq;  // item slots of one request
      const int g = it / (p.group * per_req), g_n = min(p.group, n_req - g * p.group);
      const int in_g = it - g * p.group * per_req;
      const int rank = in_g / (g_n * p.Hq);
      const int j = in_g - rank * g_n * p.Hq, pos = g * p.group + j / p.Hq;
      x.bh = (n_req <= C::PERM_MAX ? s_perm[pos] : pos) * p.Hq + j % p.Hq;
      seq_len(x.bh, x.L, x.ql);
      x.qt = (x.ql + 2 * C::BM - 1) / (2 * C::BM) - 1 - rank;
    } else {
      x.bh = it / n_qp;
      seq_len(x.bh, x.L, x.ql);
      x.qt = it % n_qp;
    }
    if (x.qt >= 0 && x.qt * 2 * C::BM < x.ql) {
      int kv_end = x.L;
      if (CAUSAL) kv_end = min(x.L, min(x.qt * 2 * C::BM + 2 * C::BM, x.ql) + (x.L - x.ql));
      x.n = (kv_end + C::BN - 1) / C::BN;
    }
    return x;
  };

  if (threadIdx.x == 0) {
    for (int q = 0; q < C::QBUF; ++q) {
      mbar_init(&bars->q_full[q], 1);
      mbar_init(&bars->q_empty[q], 1);
    }
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
  // Launched as a programmatic dependent: everything above touches only this CTA's shared
  // memory and TMEM, so its launch and set-up overlap the tail of the grid before it.  Wait
  // here, before any global access, until that grid has completed and its writes are
  // visible.  (No early trigger for the grid after this one: with it the causal d = 64
  // forward ran 20 % slower, its CTAs finishing at different times; each CTA's exit triggers
  // it instead.)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if constexpr (CAUSAL && PAGED) {
    // rank each request by its query rows (descending, ties by index: a strict order, so
    // the ranks are a permutation) against a copy of the lengths in the epilogue staging
    // area, which no epilogue has used yet
    const int n_req = p.BH / p.Hq;
    if (n_req <= C::PERM_MAX) {
      int* s_len = reinterpret_cast<int*>(smem + C::OFF_STG);
      int* perm = reinterpret_cast<int*>(smem + C::OFF_PERM);
      for (int r = threadIdx.x; r < n_req; r += blockDim.x) s_len[r] = __ldg(p.qlen + r);
      __syncthreads();
      for (int r = threadIdx.x; r < n_req; r += blockDim.x) {
        const int key = s_len[r];
        int pos = 0;
        for (int t = 0; t < n_req; ++t) pos += (s_len[t] > key) || (s_len[t] == key && t < r);
        perm[pos] = r;
      }
    }
    __syncthreads();
  }
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sK = smem_u32(smem + C::OFF_K);
  const uint32_t sV = smem_u32(smem + C::OFF_V);

  if (warp == 0 && !PAGED) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int kv = 0;  // K/V tiles issued so far (ring position)
      int local = 0;
      bool ok = true;
      for (int k = 0, it = item_index(0); it < n_items && ok; it = item_index(++k)) {
        const Item x = item_of(it);
        if (x.n == 0) continue;
        const int zkv = (x.bh / p.Hq) * p.Hkv + (x.bh % p.Hq) / (p.Hq / p.Hkv);
        const int qb = local % C::QBUF, quse = local / C::QBUF;
        ++local;
        if (quse > 0 && !(ok = mbar_wait(&bars->q_empty[qb], (quse - 1) & 1, p.wait_ns, abort_flag, 11))) break;
        mbar_arrive_expect_tx(&bars->q_full[qb], 2 * C::Q_TILE);
        for (int t = 0; t < 2; ++t)
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_3d(smem + C::OFF_Q + (qb * 2 + t) * C::Q_TILE + kb * C::BM * 128, &tmQ, &bars->q_full[qb],
                        kb * 64, x.qt * 2 * C::BM + t * C::BM, x.bh);
        for (int j = 0; j < x.n; ++j, ++kv) {
          const int st = kv % C::NSTAGE, round = kv / C::NSTAGE;
          if (round > 0 && !(ok = mbar_wait(&bars->kv_empty[st], (round - 1) & 1, p.wait_ns, abort_flag, 10)))
            break;
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
    }
  } else if (warp == 0) {
    // ------------------------------------------------- TMA producer, paged K/V (whole warp)
    // A tile's BN keys are NB = BN/16 cache blocks.  Lane i < NB owns block i of the tile:
    // it reads the block-table entry one tile ahead and issues that block's 16-row boxes
    // (one per 64-column block of K and of V) at the physical rows the entry gives.
    // Blocks past the sequence are not loaded: their V rows are zeroed (their P is 0, and
    // 0 * NaN would not be), their K rows keep stale data (those scores are masked).
    constexpr int NB = C::BN / 16;
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    int kv = 0, local = 0;
    bool ok = true;
    for (int k = 0, it = item_index(0); it < n_items && ok; it = item_index(++k)) {
      const Item x = item_of(it);
      if (x.n == 0) continue;
      const int b = x.bh / p.Hq;
      const int hk = (x.bh % p.Hq) / (p.Hq / p.Hkv);
      const int* bt = p.bt + size_t(b) * p.max_blocks;
      const int nblk = (x.L + 15) / 16;
      int ph = (lane < NB && lane < nblk) ? __ldg(bt + lane) : 0;  // entry for tile 0
      const int qb = local % C::QBUF, quse = local / C::QBUF;
      ++local;
      if (quse > 0 && !(ok = warp_wait(&bars->q_empty[qb], (quse - 1) & 1, p.wait_ns, abort_flag, 11))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars->q_full[qb], 2 * C::Q_TILE);
        for (int t = 0; t < 2; ++t)
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_3d(smem + C::OFF_Q + (qb * 2 + t) * C::Q_TILE + kb * C::BM * 128, &tmQ, &bars->q_full[qb],
                        kb * 64, x.qt * 2 * C::BM + t * C::BM, x.bh);
      }
      for (int j = 0; j < x.n; ++j, ++kv) {
        const int st = kv % C::NSTAGE, round = kv / C::NSTAGE;
        const int lb = j * NB + lane;
        const int ph_next = (lane < NB && lb + NB < nblk) ? __ldg(bt + lb + NB) : 0;
        if (round > 0 && !(ok = warp_wait(&bars->kv_empty[st], (round - 1) & 1, p.wait_ns, abort_flag, 10))) break;
        uint8_t* sk = smem + C::OFF_K + st * C::KV_TILE;
        uint8_t* sv = smem + C::OFF_V + st * C::KV_TILE;
        const int nload = min(NB, nblk - j * NB);  // >= 1: every tile starts inside the sequence
        if (nload < NB) {
          const int z0 = nload * 16 * 8, z1 = C::BN * 8;  // 16-byte units of one 64-column block
          for (int kb = 0; kb < C::KB; ++kb)
            for (int i = z0 + lane; i < z1; i += 32)
              *reinterpret_cast<uint4*>(sv + kb * C::BN * 128 + i * 16) = make_uint4(0, 0, 0, 0);
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          const uint32_t bytes = uint32_t(nload) * 16 * 128 * C::KB;
          mbar_arrive_expect_tx(&bars->k_full[st], bytes);
          mbar_arrive_expect_tx(&bars->v_full[st], bytes);
        }
        __syncwarp();
        if (lane < nload) {
          int pb = ph;
          if (pb < 0 || pb >= p.num_blocks) {  // a bad table entry: flagged, block 0 read instead
            set_status(FA_ERR_INVALID_ARG, 61);
            pb = 0;
          }
          const int crow = (pb * p.Hkv + hk) * 16;
          for (int kb = 0; kb < C::KB; ++kb) {
            tma_load_2d(smem_u32(sk + kb * C::BN * 128 + lane * 16 * 128), &tmK, &bars->k_full[st], kb * 64, crow);
            tma_load_2d(smem_u32(sv + kb * C::BN * 128 + lane * 16 * 128), &tmV, &bars->v_full[st], kb * 64, crow);
          }
        }
        ph = ph_next;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs this role so descriptors stay warp-uniform; the elected lane
    // issues the MMAs and commits.
    {
      const uint32_t leader = elect_one();
      constexpr uint32_t idS = idesc_bf16_f32(128, C::BN, 0);  // K-major A (Q) and B (K)
      constexpr uint32_t idPV = idesc_bf16_f32(128, D, 1);     // B (V) is MN-major
      const uint64_t dQ = sdesc_sw128(sQ, 16, 1024), dK = sdesc_sw128(sK, 16, 1024);
      const uint64_t dV = sdesc_sw128(sV, C::BN * 128, 1024);
      auto issue_S = [&](int qb, int t, int st) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;
          mma_ss_p(tmem + C::COL_S + t * C::BN, desc_add(dQ, (qb * 2 + t) * C::Q_TILE + kb * C::BM * 128 + kin * 32),
                   desc_add(dK, st * C::KV_TILE + kb * C::BN * 128 + kin * 32), idS, ks > 0 ? 1u : 0u, leader);
        }
      };
      auto issue_PV = [&](int t, int st, int j) {
#pragma unroll
        for (int ks = 0; ks < C::BN / 16; ++ks)
          mma_ts_p(tmem + C::COL_O + t * D, tmem + C::COL_S + t * C::BN + ks * 8,
                   desc_add(dV, st * C::KV_TILE + ks * 16 * 128), idPV, (j > 0 || ks > 0) ? 1u : 0u, leader);
      };
      int kv = 0;  // K/V tiles consumed so far (ring position)
      int g = 0;   // query-tile steps so far (s_full / p_full phase)
      int local = 0;
      bool ok = true;
      for (int k = 0, it = item_index(0); it < n_items && ok; it = item_index(++k)) {
        const Item x = item_of(it);
        const int n = x.n, L = x.L;
        if (n == 0) continue;
        const int qb = local % C::QBUF, quse = local / C::QBUF;
        ++local;
        ok = warp_wait(&bars->q_full[qb], quse & 1, p.wait_ns, abort_flag, 20) &&
             warp_wait(&bars->k_full[kv % C::NSTAGE], (kv / C::NSTAGE) & 1, p.wait_ns, abort_flag, 21);
        if (!ok) break;
        tc_fence_after();
        issue_S(qb, 0, kv % C::NSTAGE);
        mma_commit_p(&bars->s_full[0], leader);
        issue_S(qb, 1, kv % C::NSTAGE);
        mma_commit_p(&bars->s_full[1], leader);
        // the Q buffer is free once the item's last S has been computed (not its last P.V):
        // the producer then loads the next item's Q while this item's last tile finishes
        if (n == 1) mma_commit_p(&bars->q_empty[qb], leader);
        for (int j = 0; j < n; ++j, ++kv, ++g) {
          const int st = kv % C::NSTAGE;
          const int st2 = (kv + 1) % C::NSTAGE;
          const bool more = j + 1 < n;
          ok = warp_wait(&bars->v_full[st], (kv / C::NSTAGE) & 1, p.wait_ns, abort_flag, 22);
          if (!ok) break;
          if constexpr (PAGED) {
            // the sequence's last cache block is partly filled: zero the V rows of its
            // unused slots (loaded with the block; their P is 0, and 0 * NaN would not be)
            const int last = (L - 1) / 16;
            if ((L & 15) != 0 && last / (C::BN / 16) == j) {
              uint8_t* sv = smem + C::OFF_V + st * C::KV_TILE;
              const int r0 = L - j * C::BN, r1 = (last + 1) * 16 - j * C::BN;
              for (int kb = 0; kb < C::KB; ++kb)
                for (int i = r0 * 8 + lane; i < r1 * 8; i += 32)
                  *reinterpret_cast<uint4*>(sv + kb * C::BN * 128 + i * 16) = make_uint4(0, 0, 0, 0);
              fence_proxy_async_smem();
              __syncwarp();
            }
          }
          ok = warp_wait(&bars->p_full[0], g & 1, p.wait_ns, abort_flag, 23);
          if (!ok) break;
          tc_fence_after();
          issue_PV(0, st, j);
          if (more) {
            ok = warp_wait(&bars->k_full[st2], ((kv + 1) / C::NSTAGE) & 1, p.wait_ns, abort_flag, 24);
            if (!ok) break;
            tc_fence_after();
            issue_S(qb, 0, st2);
            mma_commit_p(&bars->s_full[0], leader);
          } else {
            mma_commit_p(&bars->o_final[0], leader);
          }
          ok = warp_wait(&bars->p_full[1], g & 1, p.wait_ns, abort_flag, 25);
          if (!ok) break;
          tc_fence_after();
          issue_PV(1, st, j);
          mma_commit_p(&bars->kv_empty[st], leader);
          if (more) {
            issue_S(qb, 1, st2);
            mma_commit_p(&bars->s_full[1], leader);
            if (j + 2 == n) mma_commit_p(&bars->q_empty[qb], leader);  // that was the item's last S
          } else {
            mma_commit_p(&bars->o_final[1], leader);
          }
        }
      }
    }
  } else if (warp >= C::WG0) {
    // ---------------------------------------------------------------- softmax + epilogue
    const int t = (warp - C::WG0) >> 2;         // which query tile
    const int wq = warp & 3;                    // TMEM lane quarter this warp may access
    const int r = wq * 32 + lane;               // row within the tile == TMEM lane
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::COL_S + t * C::BN;
    const uint32_t tO = tmem + lane_off + C::COL_O + t * D;
    const float sl2 = p.scale_log2;
    int g = 0, local = 0;
    bool ok = true;
    for (int k = 0, it = item_index(0); it < n_items && ok; it = item_index(++k)) {
      const Item x = item_of(it);
      const int qt = x.qt, bh = x.bh, L = x.L, ql = x.ql, n = x.n;
      if (n == 0) continue;
      const int item_local = local++;
      const int row = qt * 2 * C::BM + t * C::BM + r;
      const int row_limit = CAUSAL ? min(L, row + (L - ql) + 1) : L;
      float m = -INFINITY, l = 0.f;
      // a warp whose rows are all padding (past the query rows) skips the arithmetic: its
      // P rows only feed output rows that are never part of the result
      const bool idle = __all_sync(0xffffffffu, row >= ql);
      for (int j = 0; j < n; ++j, ++g) {
        ok = warp_wait(&bars->s_full[t], g & 1, p.wait_ns, abort_flag, 30 + t);
        if (!ok) break;
        if (!idle) {
          tc_fence_after();
          uint32_t sr[C::BN];
#pragma unroll
          for (int c = 0; c < C::BN / 32; ++c)
            tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
          tmem_wait_ld();
          float f[C::BN];
          const int lim = row_limit - j * C::BN;  // columns >= lim are masked for this row
          const bool masked = __any_sync(0xffffffffu, lim < C::BN);
#pragma unroll
          for (int c = 0; c < C::BN; ++c) f[c] = __uint_as_float(sr[c]);
          if (masked) {
#pragma unroll
            for (int c = 0; c < C::BN; ++c) f[c] = (c < lim) ? f[c] : -INFINITY;
          }
          float mx8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(f[k], f[8 + k]);
#pragma unroll
          for (int c = 16; c < C::BN; c += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], f[c + k], f[c + 8 + k]);
          const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                                 fmaxf(fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
          // The reference m that l and u share moves only when the row maximum exceeds it
          // by more than FA_RESCALE_LOG2 (base 2): u / l does not depend on which reference
          // they share, and until then every P = 2^(s - m) stays below 2^FA_RESCALE_LOG2.
          // With FA_RESCALE_LOG2 = 0 this is the recurrence with m the exact running max.
          const float m_cand = fmaxf(m, mx * sl2);
          const float m_new = (m_cand > m + FA_RESCALE_LOG2) ? m_cand : m;
          const float base = (m_new == -INFINITY) ? 0.f : m_new;
          const float alpha = (m_new == m) ? 1.f : ex2(m - base);
          const float2 sl2v = make_float2(sl2, sl2), nbase = make_float2(-base, -base);
          float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
          if (masked) {
            // boundary tile: every exponential on the SFU (exactly 0 for masked scores);
            // 32-column chunks that are masked for the whole warp are skipped
#pragma unroll
            for (int c = 0; c < C::BN / 32; ++c) {
              uint32_t pk[16];
              if (__all_sync(0xffffffffu, lim <= c * 32)) {
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = 0u;
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float2 x =
                      __ffma2_rn(make_float2(f[c * 32 + 2 * i], f[c * 32 + 2 * i + 1]), sl2v, nbase);
                  const float2 pv = make_float2(ex2(x.x), ex2(x.y));
                  rs2[i & 3] = __fadd2_rn(rs2[i & 3], pv);
                  pk[i] = pack_bf16x2(pv.x, pv.y);
                }
              }
              tmem_st16(tS + c * 16, pk);
            }
          } else {
            // interior tile: no masked column
#pragma unroll
            for (int c = 0; c < C::BN / 32; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 x = __ffma2_rn(make_float2(f[c * 32 + 2 * i], f[c * 32 + 2 * i + 1]), sl2v, nbase);
                const float2 pv = make_float2(ex2(x.x), ex2(x.y));
                rs2[i & 3] = __fadd2_rn(rs2[i & 3], pv);
                pk[i] = pack_bf16x2(pv.x, pv.y);
              }
              tmem_st16(tS + c * 16, pk);
            }
          }
          const float2 rsa = __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
          l = l * alpha + (rsa.x + rsa.y);
          // u (TMEM) holds the P.V sums of tiles < j; rescale its rows whose max rose
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
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
        if (lane == 0) mbar_arrive(&bars->p_full[t]);
      }
      if (ok) ok = warp_wait(&bars->o_final[t], item_local & 1, p.wait_ns, abort_flag, 40 + t);
      if (!ok) break;
      if (idle) continue;
      tc_fence_after();
      // O = u / l, staged per warp (32 rows x STG_COLS columns, swizzled as the O map
      // expects: 128-byte rows with the 128-byte pattern, or 64-byte rows with the 64-byte
      // one) and written by TMA stores, which also drop the rows past the query rows' end
      const float inv = 1.f / l;
      uint8_t* stg = smem + C::OFF_STG + (warp - C::WG0) * C::STG_WARP;
      const int row0 = qt * 2 * C::BM + t * C::BM + wq * 32;
#pragma unroll
      for (int c = 0; c < D / C::STG_COLS; ++c) {
        uint32_t o[C::STG_COLS];
#pragma unroll
        for (int h2 = 0; h2 < C::STG_COLS / 32; ++h2)
          tmem_ld32(tO + c * C::STG_COLS + h2 * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[h2 * 32]));
        tmem_wait_ld();
        if (lane == 0) bulk_wait_read();  // the previous store from this staging buffer
        __syncwarp();
#pragma unroll
        for (int u = 0; u < C::STG_COLS / 8; ++u) {
          const float2 a = __fmul2_rn(make_float2(__uint_as_float(o[8 * u]), __uint_as_float(o[8 * u + 1])),
                                      make_float2(inv, inv));
          const float2 b2 = __fmul2_rn(make_float2(__uint_as_float(o[8 * u + 2]), __uint_as_float(o[8 * u + 3])),
                                       make_float2(inv, inv));
          const float2 c2 = __fmul2_rn(make_float2(__uint_as_float(o[8 * u + 4]), __uint_as_float(o[8 * u + 5])),
                                       make_float2(inv, inv));
          const float2 d2 = __fmul2_rn(make_float2(__uint_as_float(o[8 * u + 6]), __uint_as_float(o[8 * u + 7])),
                                       make_float2(inv, inv));
          const int chunk = (C::STG_COLS == 64) ? (u ^ (lane & 7)) : (u ^ ((lane >> 1) & 3));
          *reinterpret_cast<uint4*>(stg + lane * (C::STG_COLS * 2) + (chunk << 4)) =
              make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(b2.x, b2.y), pack_bf16x2(c2.x, c2.y),
                         pack_bf16x2(d2.x, d2.y));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmO, stg, c * C::STG_COLS, row0, bh);
          bulk_commit();
        }
      }
      if (row < ql) p.lse[size_t(bh) * p.Nq + row] = (m + __log2f(l)) * 0.69314718055994531f;
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
