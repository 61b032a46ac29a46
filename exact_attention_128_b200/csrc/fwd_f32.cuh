// fwd_f32.cuh — fp32 forward pass on the CUDA cores (head dim 64).
//
// Exact attention, softmax(Q K^T * scale) V ("Autoatención, kernels CUDA y
// FlashAttention" §1), evaluated tile by tile with the online-softmax recurrence of
// "FlashAttention" (paweldubiel.com notes), "No basta con promediar los resultados de
// los bloques": running maximum m, sum l and numerator u; when a tile raises the
// maximum, l and u are multiplied by e^{m - m'} before the tile's terms are added.
//
// fp32 inputs need fp32 products (TF32 tensor-core inputs would lose ~3 decimal
// digits), so this kernel uses FFMA.  It serves the small fp32 ViT layer; the bf16
// tensor-core kernel is the throughput path.
#pragma once
#include "common.cuh"

namespace fa {

namespace f32 {
constexpr int D = 64;
constexpr int BQ = 64;        // query rows per CTA (16 when 64-row CTAs would not fill the GPU)
constexpr int BK = 32;        // keys per tile
constexpr int THREADS = 256;  // 4 threads per query row (4 * BQ)
constexpr int KPAD = D + 1;   // padded K row (bank-conflict free score loop)
constexpr int PPAD = BK + 1;  // padded P row
}  // namespace f32

struct FwdF32Params {
  const float* q;
  const float* k;
  const float* v;
  float* o;
  float* lse;
  int Hq, Hkv, Nq, Nkv;
  float scale;
  int causal;
};

template <int BQ>
__global__ void __launch_bounds__(4 * BQ) fa_fwd_f32_kernel(const FwdF32Params p) {
  using f32::D;
  using f32::BK;
  using f32::KPAD;
  using f32::PPAD;
  constexpr int THREADS = 4 * BQ;
  __shared__ float Ks[BK * KPAD];
  __shared__ __align__(16) float Vs[BK * D];
  __shared__ float Ps[BQ * PPAD];

  const int tid = threadIdx.x;
  const int r = tid >> 2;   // query row within the tile
  const int qd = tid & 3;   // quarter: keys qd, qd+4, ... of a tile; output columns [16*qd, 16*qd+16)
  const int bh = blockIdx.y;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int hk = h / (p.Hq / p.Hkv);
  const int q0 = blockIdx.x * BQ;
  const int row = q0 + r;
  const bool row_ok = row < p.Nq;
  const int off = p.Nkv - p.Nq;  // bottom-right causal alignment

  const float* Qh = p.q + (size_t(bh) * p.Nq) * D;
  const float* Kh = p.k + (size_t(b) * p.Hkv + hk) * size_t(p.Nkv) * D;
  const float* Vh = p.v + (size_t(b) * p.Hkv + hk) * size_t(p.Nkv) * D;

  float qr[D];
#pragma unroll
  for (int c = 0; c < D; c += 4) {
    float4 t = row_ok ? *reinterpret_cast<const float4*>(Qh + size_t(row) * D + c) : make_float4(0, 0, 0, 0);
    qr[c] = t.x; qr[c + 1] = t.y; qr[c + 2] = t.z; qr[c + 3] = t.w;
  }

  float m = -INFINITY, l = 0.f;
  float acc[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) acc[c] = 0.f;

  // keys visible to this CTA's last row
  int kv_end = p.Nkv;
  if (p.causal) kv_end = min(p.Nkv, min(q0 + BQ, p.Nq) - 1 + off + 1);
  const int ntiles = (kv_end + BK - 1) / BK;
  // per-row limit on visible keys
  const int row_limit = p.causal ? min(p.Nkv, row + off + 1) : p.Nkv;

  for (int t = 0; t < ntiles; ++t) {
    const int k0 = t * BK;
    // stage K (padded rows) and V tiles; rows past Nkv are zero.  A thread's loads are all
    // issued before its first store, so their latencies overlap.
    {
      constexpr int IT = BK * (D / 4) / THREADS;
      static_assert(IT * THREADS == BK * (D / 4), "the tile splits evenly over the threads");
      float4 kk[IT], vv[IT];
#pragma unroll
      for (int u = 0; u < IT; ++u) {
        const int i = tid + u * THREADS;
        const int kr = i / (D / 4), c4 = (i % (D / 4)) * 4;
        kk[u] = make_float4(0, 0, 0, 0);
        vv[u] = make_float4(0, 0, 0, 0);
        if (k0 + kr < p.Nkv) {
          kk[u] = *reinterpret_cast<const float4*>(Kh + size_t(k0 + kr) * D + c4);
          vv[u] = *reinterpret_cast<const float4*>(Vh + size_t(k0 + kr) * D + c4);
        }
      }
#pragma unroll
      for (int u = 0; u < IT; ++u) {
        const int i = tid + u * THREADS;
        const int kr = i / (D / 4), c4 = (i % (D / 4)) * 4;
        float* kd = Ks + kr * KPAD + c4;
        kd[0] = kk[u].x; kd[1] = kk[u].y; kd[2] = kk[u].z; kd[3] = kk[u].w;
        *reinterpret_cast<float4*>(Vs + kr * D + c4) = vv[u];
      }
    }
    __syncthreads();

    constexpr int KQ = BK / 4;  // keys per thread
    float s[KQ];
#pragma unroll
    for (int c = 0; c < KQ; ++c) s[c] = 0.f;
#pragma unroll
    for (int dd = 0; dd < D; ++dd) {
      const float qv = qr[dd];
#pragma unroll
      for (int c = 0; c < KQ; ++c) s[c] = fmaf(qv, Ks[(c * 4 + qd) * KPAD + dd], s[c]);
    }
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < KQ; ++c) {
      const int key = k0 + c * 4 + qd;
      s[c] = (key < row_limit) ? s[c] * p.scale : -INFINITY;
      mx = fmaxf(mx, s[c]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    // a row whose visible keys all lie in later tiles keeps m = -inf; use 0 as the base
    const float base = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = expf(m - base);  // e^{m - m'}; 0 when m = -inf
    float rs = 0.f;
#pragma unroll
    for (int c = 0; c < KQ; ++c) {
      const float e = expf(s[c] - base);
      rs += e;
      Ps[r * PPAD + c * 4 + qd] = e;
    }
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    l = l * alpha + rs;
    m = m_new;
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] *= alpha;
    __syncthreads();

    const int kn = min(BK, kv_end - k0);
    for (int kk = 0; kk < kn; ++kk) {
      const float pv = Ps[r * PPAD + kk];
      const float4* vrow = reinterpret_cast<const float4*>(Vs + kk * D + qd * 16);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const float4 vv = vrow[c4];
        acc[c4 * 4 + 0] = fmaf(pv, vv.x, acc[c4 * 4 + 0]);
        acc[c4 * 4 + 1] = fmaf(pv, vv.y, acc[c4 * 4 + 1]);
        acc[c4 * 4 + 2] = fmaf(pv, vv.z, acc[c4 * 4 + 2]);
        acc[c4 * 4 + 3] = fmaf(pv, vv.w, acc[c4 * 4 + 3]);
      }
    }
    __syncthreads();
  }

  if (row_ok) {
    const float inv = 1.f / l;
    float* orow = p.o + (size_t(bh) * p.Nq + row) * D + qd * 16;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      *reinterpret_cast<float4*>(orow + c4 * 4) =
          make_float4(acc[c4 * 4] * inv, acc[c4 * 4 + 1] * inv, acc[c4 * 4 + 2] * inv, acc[c4 * 4 + 3] * inv);
    if (qd == 0) p.lse[size_t(bh) * p.Nq + row] = m + logf(l);
  }
}

// Short key sequences (Nkv <= SMALL_NKV, the ViT regime): one pass per CTA instead of a
// walk over key tiles.  The CTA's 16 query rows see every key of their head at once: K
// (padded rows) and V are loaded into shared memory together, so the CTA pays one
// global-load round trip instead of one per 32-key tile, and the softmax needs no running
// rescale (m and l are the row's exact maximum and sum).  512 threads: 16 per query row;
// thread j of a row computes the scores of keys j, j + 16, ... and output columns
// [4 j, 4 j + 4).  One CTA per SM (its shared memory), so 32-row CTAs keep a ViT layer
// (12 heads x 196 rows) to a single wave.
namespace f32 {
constexpr int SMALL_NKV = 256;
constexpr int SROWS = 32;  // query rows per CTA
constexpr int STHREADS = 16 * SROWS;
constexpr int QPAD = D + 4;  // padded Q row: the two rows a warp reads sit 4 banks apart
}  // namespace f32

// floats of the padded K rows of nk keys, rounded up so that V, read with 16-byte vectors,
// starts on a 16-byte boundary
__host__ __device__ inline int f32_small_kfloats(int nk) { return (nk * f32::KPAD + 3) & ~3; }

inline size_t fwd_f32_small_smem(int nk) {  // bytes of dynamic shared memory for nk keys
  return sizeof(float) * (size_t(f32::SROWS) * f32::QPAD + size_t(f32_small_kfloats(nk)) + size_t(nk) * f32::D +
                          size_t(f32::SROWS) * (nk + 1));
}

__global__ void __launch_bounds__(f32::STHREADS) fa_fwd_f32_small_kernel(const FwdF32Params p) {
  using f32::D;
  using f32::KPAD;
  using f32::SROWS;
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x;
  const int r = tid >> 4;  // query row within the CTA
  const int j = tid & 15;  // lane within the row's 16 threads
  const int bh = blockIdx.y;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int hk = h / (p.Hq / p.Hkv);
  const int q0 = blockIdx.x * SROWS;
  const int row = q0 + r;
  const int off = p.Nkv - p.Nq;  // bottom-right causal alignment
  // keys any row of this CTA sees
  const int nk = p.causal ? min(p.Nkv, min(q0 + SROWS, p.Nq) + off) : p.Nkv;
  float* Qs = sm;                      // [SROWS][QPAD]
  float* Ks = Qs + SROWS * f32::QPAD;  // [nk][KPAD]
  float* Vs = Ks + f32_small_kfloats(nk);  // [nk][D], 16-byte aligned rows
  float* Ps = Vs + size_t(nk) * D;   // [SROWS][nk + 1]
  const float* Qh = p.q + size_t(bh) * p.Nq * D;
  const float* Kh = p.k + (size_t(b) * p.Hkv + hk) * size_t(p.Nkv) * D;
  const float* Vh = p.v + (size_t(b) * p.Hkv + hk) * size_t(p.Nkv) * D;
  for (int i = tid; i < SROWS * (D / 4); i += f32::STHREADS) {
    const int rr = i / (D / 4), c4 = (i % (D / 4)) * 4;
    const float4 x = (q0 + rr < p.Nq) ? *reinterpret_cast<const float4*>(Qh + size_t(q0 + rr) * D + c4)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(Qs + rr * f32::QPAD + c4) = x;
  }
  // every K and V load of the thread is issued before the first store, so their L2 / DRAM
  // latencies overlap (nk * D / 4 <= 4096 vectors each: at most 8 per thread)
  {
    constexpr int IT = f32::SMALL_NKV * (D / 4) / f32::STHREADS;
    float4 kk[IT], vv[IT];
#pragma unroll
    for (int u = 0; u < IT; ++u) {
      const int i = tid + f32::STHREADS * u;
      if (i < nk * (D / 4)) {
        const int kr = i / (D / 4), c4 = (i % (D / 4)) * 4;
        kk[u] = *reinterpret_cast<const float4*>(Kh + size_t(kr) * D + c4);
        vv[u] = *reinterpret_cast<const float4*>(Vh + size_t(kr) * D + c4);
      }
    }
#pragma unroll
    for (int u = 0; u < IT; ++u) {
      const int i = tid + f32::STHREADS * u;
      if (i < nk * (D / 4)) {
        const int kr = i / (D / 4), c4 = (i % (D / 4)) * 4;
        float* kd = Ks + kr * KPAD + c4;
        kd[0] = kk[u].x; kd[1] = kk[u].y; kd[2] = kk[u].z; kd[3] = kk[u].w;
        *reinterpret_cast<float4*>(Vs + kr * D + c4) = vv[u];
      }
    }
  }
  __syncthreads();

  const int row_limit = p.causal ? min(p.Nkv, row + off + 1) : p.Nkv;  // keys < row_limit are visible
  constexpr int KT = f32::SMALL_NKV / 16;  // keys per thread at most
  float qr[D];  // the thread's query row, from shared memory once
#pragma unroll
  for (int c = 0; c < D; c += 4) {
    const float4 x = *reinterpret_cast<const float4*>(Qs + r * f32::QPAD + c);
    qr[c] = x.x; qr[c + 1] = x.y; qr[c + 2] = x.z; qr[c + 3] = x.w;
  }
  float s[KT];
  float mx = -INFINITY;
#pragma unroll
  for (int t = 0; t < KT; ++t) {
    const int key = j + 16 * t;
    s[t] = -INFINITY;
    if (key < nk) {
      float acc = 0.f;
      const float* kr = Ks + key * KPAD;
#pragma unroll
      for (int d = 0; d < D; ++d) acc = fmaf(qr[d], kr[d], acc);
      s[t] = (key < row_limit) ? acc * p.scale : -INFINITY;
    }
    mx = fmaxf(mx, s[t]);
  }
#pragma unroll
  for (int w = 1; w < 16; w <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, w));
  // every row sees at least one key (key 0 at causal offset >= 0), so mx is finite for rows
  // < Nq; padding rows past Nq have zero scores
  float ls = 0.f;
#pragma unroll
  for (int t = 0; t < KT; ++t) {
    const int key = j + 16 * t;
    if (key < nk) {
      const float e = (s[t] == -INFINITY) ? 0.f : expf(s[t] - mx);
      ls += e;
      Ps[r * (nk + 1) + key] = e;
    }
  }
#pragma unroll
  for (int w = 1; w < 16; w <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, w);
  __syncwarp();  // a row's P is written and read by the same 16 threads (half a warp)

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* prow = Ps + r * (nk + 1);
  const float* vcol = Vs + 4 * j;
  for (int key = 0; key < nk; ++key) {
    const float pv = prow[key];
    const float4 v4 = *reinterpret_cast<const float4*>(vcol + key * D);
    acc.x = fmaf(pv, v4.x, acc.x);
    acc.y = fmaf(pv, v4.y, acc.y);
    acc.z = fmaf(pv, v4.z, acc.z);
    acc.w = fmaf(pv, v4.w, acc.w);
  }
  if (row < p.Nq) {
    const float inv = 1.f / ls;
    *reinterpret_cast<float4*>(p.o + (size_t(bh) * p.Nq + row) * D + 4 * j) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (j == 0) p.lse[size_t(bh) * p.Nq + row] = mx + logf(ls);
  }
}

}  // namespace fa
