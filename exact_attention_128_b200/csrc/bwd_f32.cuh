// bwd_f32.cuh — fp32 backward pass on the CUDA cores (head dim 64).
//
// Gradients of the exact attention O = softmax(Q K^T * scale) V, recomputing the score
// tiles from the saved lse instead of storing P ("Autoatención, kernels CUDA y
// FlashAttention" §3, "Recálculo durante la retropropagación").  Per (query i, key j):
//   P_ij = exp(scale q_i.k_j - lse_i)       (0 where masked)
//   dV_j += P_ij dO_i                       dP_ij = dO_i . v_j
//   D_i  = sum_c dO_ic O_ic                 dS_ij = P_ij (dP_ij - D_i)
//   dQ_i += scale dS_ij k_j                 dK_j += scale dS_ij q_i
// (the gradient of sum(O * dO) by matrix calculus; dK and dV summed over the query heads
// that share a key/value head).
//
// fp32 inputs need fp32 products, so this path uses FFMA, like the fp32 forward.  Two
// kernels, no atomics, every result written once:
//   fa_bwd_f32_pre_kernel   D_i, one warp per query row
//   fa_bwd_f32_kernel       two kinds of CTA in one grid, which run side by side (each kind
//                           alone leaves the SMs with few warps to hide its latencies):
//     dK/dV CTA  one per (BR-key block, batch, kv head): walks the group's query heads and
//                the query blocks that see the keys
//     dQ CTA     one per (BR-row query block, batch, query head): walks the key blocks the
//                rows see
// Each step recomputes a BR x BR score tile in shared memory (8 threads per row, BR/8
// scores each) and accumulates 8 output columns per thread; the library launches BR = 32.
#pragma once
#include "common.cuh"

namespace fa {

namespace b32 {
constexpr int D = 64;
constexpr int RP = D + 1;  // padded row of a [BR x 64] tile
}  // namespace b32

struct BwdF32Params {
  const float* q;
  const float* k;
  const float* v;
  const float* o;
  const float* lse;  // natural log, [B,Hq,Nq]
  const float* dO;
  float* dq;
  float* dk;
  float* dv;
  float* Dvec;  // [B,Hq,Nq] workspace
  int Hq, Hkv, Nq, Nkv;
  float scale;
  int causal;
};

__global__ void __launch_bounds__(256) fa_bwd_f32_pre_kernel(const float* o, const float* dO, float* Dvec,
                                                             long rows) {
  const long row = long(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* a = o + row * b32::D;
  const float* g = dO + row * b32::D;
  float s = a[lane] * g[lane] + a[lane + 32] * g[lane + 32];
#pragma unroll
  for (int w = 16; w > 0; w >>= 1) s += __shfl_xor_sync(0xffffffffu, s, w);
  if (lane == 0) Dvec[row] = s;
}

namespace b32 {

// rows [r0, r0 + BR) of a [n, 64] matrix into a padded tile; rows past n read as zero.
// Each of the 8 * BR threads loads its D / 8 elements before storing any, so the loads'
// latencies overlap instead of adding up.
template <int BR>
__device__ __forceinline__ void load_tile(float (*dst)[RP], const float* src, int r0, int n) {
  constexpr int PER = D / 8;
  float x[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int e = threadIdx.x + u * 8 * BR;
    const int r = e / D, c = e % D;
    x[u] = (r0 + r < n) ? src[size_t(r0 + r) * D + c] : 0.f;
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int e = threadIdx.x + u * 8 * BR;
    dst[e / D][e % D] = x[u];
  }
}

// the N dot products a[i] . b[j0 + u], u < N, of 64-long rows
template <int N>
__device__ __forceinline__ void dotn(const float (*a)[RP], const float (*b)[RP], int i, int j0, float (&out)[N]) {
#pragma unroll
  for (int u = 0; u < N; ++u) out[u] = 0.f;
#pragma unroll 16
  for (int c = 0; c < D; ++c) {
    const float x = a[i][c];
#pragma unroll
    for (int u = 0; u < N; ++u) out[u] = fmaf(x, b[j0 + u][c], out[u]);
  }
}

// P and dS of one BR x BR tile: rows qi0 + i (query), columns kj0 + j (key); thread owns
// row i = tid / 8 and columns j0 .. j0 + BR/8 - 1, j0 = (tid % 8) * BR/8.
template <int BR>
__device__ __forceinline__ void p_ds_tile(const float (*sQ)[RP], const float (*sK)[RP], const float (*sdO)[RP],
                                          const float (*sV)[RP], const float* sL, const float* sD,
                                          float (*sP)[BR + 1], float (*sS)[BR + 1], int qi0, int kj0,
                                          const BwdF32Params& p) {
  constexpr int N = BR / 8;
  const int i = threadIdx.x >> 3, j0 = (threadIdx.x & 7) * N;
  float s[N], dp[N];
  dotn<N>(sQ, sK, i, j0, s);
  dotn<N>(sdO, sV, i, j0, dp);
  const int qi = qi0 + i, off = p.Nkv - p.Nq;
#pragma unroll
  for (int u = 0; u < N; ++u) {
    const int kj = kj0 + j0 + u;
    const bool ok = qi < p.Nq && kj < p.Nkv && (!p.causal || kj <= qi + off);
    const float pij = ok ? expf(s[u] * p.scale - sL[i]) : 0.f;
    sP[i][j0 + u] = pij;
    sS[i][j0 + u] = pij * (dp[u] - sD[i]);
  }
}

}  // namespace b32

template <int BR>
struct BwdF32Smem {
  float sK[BR][b32::RP], sV[BR][b32::RP], sQ[BR][b32::RP], sdO[BR][b32::RP];
  float sP[BR][BR + 1], sS[BR][BR + 1], sL[BR], sD[BR];
};

// dK and dV of key block kb of (batch, kv head) bk
template <int BR>
__device__ __forceinline__ void bwd_f32_dkdv(const BwdF32Params& p, BwdF32Smem<BR>& sm, int kb, int bk) {
  using namespace b32;
  constexpr int BQ = BR, BK = BR;
  auto& sK = sm.sK;
  auto& sV = sm.sV;
  auto& sQ = sm.sQ;
  auto& sdO = sm.sdO;
  auto& sP = sm.sP;
  auto& sS = sm.sS;
  auto& sL = sm.sL;
  auto& sD = sm.sD;
  const int b = bk / p.Hkv, hk = bk % p.Hkv, G = p.Hq / p.Hkv;
  const int kj0 = kb * BK;
  load_tile<BR>(sK, p.k + size_t(bk) * p.Nkv * D, kj0, p.Nkv);
  load_tile<BR>(sV, p.v + size_t(bk) * p.Nkv * D, kj0, p.Nkv);
  // thread owns key j = tid / 8, columns c0 .. c0 + 7
  const int j = threadIdx.x >> 3, c0 = (threadIdx.x & 7) * 8;
  float adk[8], adv[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) adk[u] = adv[u] = 0.f;
  // the first query block with a row that sees key kj0 (causal: row qi sees kj <= qi + off)
  const int off = p.Nkv - p.Nq;
  const int qb0 = p.causal ? max(0, (kj0 - off) / BQ) : 0;
  for (int g = 0; g < G; ++g) {
    const size_t bh = size_t(b) * p.Hq + hk * G + g;
    for (int qb = qb0; qb * BQ < p.Nq; ++qb) {
      const int qi0 = qb * BQ;
      __syncthreads();  // the previous step's tiles are consumed
      load_tile<BR>(sQ, p.q + bh * p.Nq * D, qi0, p.Nq);
      load_tile<BR>(sdO, p.dO + bh * p.Nq * D, qi0, p.Nq);
      if (threadIdx.x < BQ) {
        const int qi = qi0 + threadIdx.x;
        sL[threadIdx.x] = qi < p.Nq ? p.lse[bh * p.Nq + qi] : 0.f;
        sD[threadIdx.x] = qi < p.Nq ? p.Dvec[bh * p.Nq + qi] : 0.f;
      }
      __syncthreads();
      p_ds_tile<BR>(sQ, sK, sdO, sV, sL, sD, sP, sS, qi0, kj0, p);
      __syncthreads();
#pragma unroll 4
      for (int i = 0; i < BQ; ++i) {
        const float pij = sP[i][j], dsij = sS[i][j];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          adv[u] = fmaf(pij, sdO[i][c0 + u], adv[u]);
          adk[u] = fmaf(dsij, sQ[i][c0 + u], adk[u]);
        }
      }
    }
  }
  const int kj = kj0 + j;
  if (kj < p.Nkv) {
    float* dk = p.dk + (size_t(bk) * p.Nkv + kj) * D + c0;
    float* dv = p.dv + (size_t(bk) * p.Nkv + kj) * D + c0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      dk[u] = adk[u] * p.scale;
      dv[u] = adv[u];
    }
  }
}

// dQ of query block qb of (batch, query head) bh
template <int BR>
__device__ __forceinline__ void bwd_f32_dq(const BwdF32Params& p, BwdF32Smem<BR>& sm, int qb, int bh) {
  using namespace b32;
  constexpr int BQ = BR, BK = BR;
  auto& sK = sm.sK;
  auto& sV = sm.sV;
  auto& sQ = sm.sQ;
  auto& sdO = sm.sdO;
  auto& sP = sm.sP;
  auto& sS = sm.sS;
  auto& sL = sm.sL;
  auto& sD = sm.sD;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const size_t bk = size_t(b) * p.Hkv + h / (p.Hq / p.Hkv);
  const int qi0 = qb * BQ;
  load_tile<BR>(sQ, p.q + size_t(bh) * p.Nq * D, qi0, p.Nq);
  load_tile<BR>(sdO, p.dO + size_t(bh) * p.Nq * D, qi0, p.Nq);
  if (threadIdx.x < BQ) {
    const int qi = qi0 + threadIdx.x;
    sL[threadIdx.x] = qi < p.Nq ? p.lse[size_t(bh) * p.Nq + qi] : 0.f;
    sD[threadIdx.x] = qi < p.Nq ? p.Dvec[size_t(bh) * p.Nq + qi] : 0.f;
  }
  // thread owns query row i = tid / 8, columns c0 .. c0 + 7
  const int i = threadIdx.x >> 3, c0 = (threadIdx.x & 7) * 8;
  float adq[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) adq[u] = 0.f;
  // keys the block's rows see: all, or (causal) up to its last row + off
  const int kv_end = p.causal ? min(p.Nkv, qi0 + BQ + (p.Nkv - p.Nq)) : p.Nkv;
  for (int kj0 = 0; kj0 < kv_end; kj0 += BK) {
    __syncthreads();  // the previous step's tiles are consumed (and this block's Q, dO loaded)
    load_tile<BR>(sK, p.k + bk * p.Nkv * D, kj0, p.Nkv);
    load_tile<BR>(sV, p.v + bk * p.Nkv * D, kj0, p.Nkv);
    __syncthreads();
    p_ds_tile<BR>(sQ, sK, sdO, sV, sL, sD, sP, sS, qi0, kj0, p);
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < BK; ++jj) {
      const float dsij = sS[i][jj];
#pragma unroll
      for (int u = 0; u < 8; ++u) adq[u] = fmaf(dsij, sK[jj][c0 + u], adq[u]);
    }
  }
  const int qi = qi0 + i;
  if (qi < p.Nq) {
    float* dq = p.dq + (size_t(bh) * p.Nq + qi) * D + c0;
#pragma unroll
    for (int u = 0; u < 8; ++u) dq[u] = adq[u] * p.scale;
  }
}

// CTAs [0, n_dkdv) compute dK/dV (key block, batch * Hkv + kv head), the rest dQ (query
// block, batch * Hq + query head); both index orders are key/query block fastest.
template <int BR>
__global__ void __launch_bounds__(8 * BR) fa_bwd_f32_kernel(const BwdF32Params p, int n_kb, int n_dkdv, int n_qb) {
  __shared__ BwdF32Smem<BR> sm;
  const int c = blockIdx.x;
  if (c < n_dkdv)
    bwd_f32_dkdv<BR>(p, sm, c % n_kb, c / n_kb);
  else
    bwd_f32_dq<BR>(p, sm, (c - n_dkdv) % n_qb, (c - n_dkdv) / n_qb);
}

}  // namespace fa
