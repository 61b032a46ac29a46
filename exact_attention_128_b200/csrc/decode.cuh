// decode.cuh — one decode step of exact attention over a paged KV cache.
//
// "Kernels de atención rápida y fusión de operadores" (the-ai.news), "Atención tipo
// FlashAttention y atención paginada": the KV cache is stored in fixed-size blocks and
// a block table links each request's logical positions to physical blocks, so the
// kernel translates every position through the table.  The attention itself is the
// definition of "Autoatención, kernels CUDA y FlashAttention" §1 with one query token
// per request, evaluated with the online-softmax recurrence of "FlashAttention"
// (paweldubiel.com notes).  The G = Hq/Hkv query heads that share a key/value head
// ("Mecanismo y detalles", GQA) are processed together, so each K/V byte is read once.
//
// Work split (split-KV): CTA (split s, kv head g, request r) covers logical blocks
// [s*CHUNK, (s+1)*CHUNK) of request r.  Each of its 4 warps takes every 4th block and
// keeps its own (m, l, u) state; the warps' states and then the splits' partial
// results are merged by weighting each part with its unnormalised mass e^{lse_s}
// ("No basta con promediar los resultados de los bloques": block results are never
// simply averaged).  A request that fits in one split writes its output directly.
//
// Data path: the step is bound by reading K and V from device memory.  Every thread
// copies its own 16-byte pieces of each 4 KB (block, kv head) slab into shared memory
// with cp.async (a ring of STAGES blocks per warp) and later reads back exactly those
// pieces, so no intra-warp synchronisation is needed and the reads are
// conflict-free.  The pieces are chosen so that they already form mma.sync fragments:
// the head dimension is permuted consistently between q and K (a dot product does not
// depend on the order of its terms) and between V and the output columns.
#pragma once
#include "common.cuh"

namespace fa {
namespace dec {
constexpr int D = 128;
constexpr int BS = 16;          // tokens per cache block
constexpr int WARPS = 4;
constexpr int STAGES = 3;       // blocks in flight per warp
constexpr int CHUNK = 32;       // logical blocks per CTA (split size = 512 tokens)
constexpr int SLAB = BS * D * 2;  // 4096 bytes: one (block, kv head) slab of K or V
constexpr int SMEM = WARPS * STAGES * 2 * SLAB;
constexpr int MAX_G = 16;
}  // namespace dec

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kc;
  const __nv_bfloat16* vc;
  const int* bt;
  const int* ctx;
  __nv_bfloat16* o;
  float* lse;  // may be null
  float* part_o;
  float* part_lse;
  int R, Hq, Hkv, max_blocks, num_blocks, max_splits;
  float scale_log2;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(dec::WARPS * 32) fa_paged_decode_kernel(const DecodeParams p) {
  using namespace dec;
  extern __shared__ __align__(16) uint8_t dsmem[];
  const int s = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  const int ctx = p.ctx[r];
  if (ctx < 1 || ctx > p.max_blocks * BS) {
    if (s == 0 && g == 0 && threadIdx.x == 0) set_status(FA_ERR_INVALID_ARG, 100);
    return;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int nsplit = (nblk + CHUNK - 1) / CHUNK;
  const int b0 = s * CHUNK;
  if (b0 >= nblk) return;
  const int b1 = min(nblk, b0 + CHUNK);

  const int warp = warp_id(), lane = lane_id();
  const int gq = lane >> 2;  // mma group id: query head row (and +8), key token, output column group
  const int t4 = lane & 3;
  const int nb = (b1 - b0 - warp + WARPS - 1) / WARPS;  // blocks for this warp (may be <= 0)

  // q fragments (A operand, 16 rows = heads of the group, zero past G), with the head
  // dimension permuted: virtual k (2*t4 + {0,1}, 2*t4 + 8 + {0,1}) of k-step ks is
  // physical d = 32*t4 + 4*ks + {0,1} and {2,3}.
  uint32_t qa[8][4];
  {
    const int h0 = g * G + gq, h1 = g * G + gq + 8;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(p.q + (size_t(r) * p.Hq + h0) * D + 32 * t4);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(p.q + (size_t(r) * p.Hq + h1) * D + 32 * t4);
    const bool v0 = gq < G, v1 = gq + 8 < G;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = v0 ? q0[2 * ks] : 0u;
      qa[ks][1] = v1 ? q1[2 * ks] : 0u;
      qa[ks][2] = v0 ? q0[2 * ks + 1] : 0u;
      qa[ks][3] = v1 ? q1[2 * ks + 1] : 0u;
    }
  }

  const uint32_t sbase = smem_u32(dsmem) + warp * STAGES * 2 * SLAB;
  const size_t slab_elems = size_t(BS) * D;
  const int* bt_row = p.bt + size_t(r) * p.max_blocks;

  // Issue the copies of this warp's i-th block into stage i % STAGES (always commits a
  // group, possibly empty, so group counting stays uniform).
  auto issue = [&](int i) {
    if (i < nb) {
      const int lb = b0 + warp + i * WARPS;
      int phys = bt_row[lb];
      if (phys < 0 || phys >= p.num_blocks) {
        set_status(FA_ERR_INVALID_ARG, 101);
        phys = 0;  // never dereference an out-of-range id; the result is flagged invalid
      }
      const __nv_bfloat16* ks = p.kc + (size_t(phys) * p.Hkv + g) * slab_elems;
      const __nv_bfloat16* vs = p.vc + (size_t(phys) * p.Hkv + g) * slab_elems;
      const uint32_t dk = sbase + (i % STAGES) * 2 * SLAB;
      const uint32_t dv = dk + SLAB;
      // K: tokens gq and gq + 8, d in [32*t4, 32*t4 + 32): 4 pieces each
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int tok = gq + 8 * (c >> 2);
        cp_async16(dk + (c * 32 + lane) * 16, ks + tok * D + 32 * t4 + 8 * (c & 3));
      }
      // V: tokens 2*t4 + {0, 1, 8, 9}, d in [16*gq, 16*gq + 16): 2 pieces each
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int tok = 2 * t4 + (c >> 1 & 1) + 8 * (c >> 2);
        cp_async16(dv + (c * 32 + lane) * 16, vs + tok * D + 16 * gq + 8 * (c & 1));
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int i = 0; i < STAGES; ++i) issue(i);

  float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 units) of rows gq, gq + 8
  float l0 = 0.f, l1 = 0.f;              // this thread's share of the running sums
  float acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  const float sl2 = p.scale_log2;

  for (int i = 0; i < nb; ++i) {
    cp_async_wait<STAGES - 1>();
    const uint32_t dk = sbase + (i % STAGES) * 2 * SLAB;
    const uint32_t dv = dk + SLAB;
    const int lb = b0 + warp + i * WARPS;
    const int valid = min(BS, ctx - lb * BS);  // tokens of this block that are cached

    // ---- scores S[head][token] = q . k over the permuted head dimension
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      uint32_t kr[16];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 v4;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v4.x), "=r"(v4.y), "=r"(v4.z), "=r"(v4.w)
                     : "r"(dk + ((nt * 4 + c) * 32 + lane) * 16));
        kr[4 * c] = v4.x; kr[4 * c + 1] = v4.y; kr[4 * c + 2] = v4.z; kr[4 * c + 3] = v4.w;
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_bf16_16816(sc[nt], qa[ks], kr[2 * ks], kr[2 * ks + 1]);
    }
    // ---- mask tokens past ctx (selection, so garbage in unused slots cannot leak)
    if (valid < BS) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (nt * 8 + 2 * t4 + (e & 1) >= valid) sc[nt][e] = -INFINITY;
    }
    float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
    float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0 * sl2), n1 = fmaxf(m1, mx1 * sl2);  // the first block has a valid token
    const float a0 = ex2(m0 - n0), a1 = ex2(m1 - n1);                  // 0 on the first block
    m0 = n0;
    m1 = n1;
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pr[nt][0] = ex2(fmaf(sc[nt][0], sl2, -n0));
      pr[nt][1] = ex2(fmaf(sc[nt][1], sl2, -n0));
      pr[nt][2] = ex2(fmaf(sc[nt][2], sl2, -n1));
      pr[nt][3] = ex2(fmaf(sc[nt][3], sl2, -n1));
    }
    l0 = l0 * a0 + pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1];
    l1 = l1 * a1 + pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
    if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        acc[nt][0] *= a0; acc[nt][1] *= a0;
        acc[nt][2] *= a1; acc[nt][3] *= a1;
      }
    }
    uint32_t pa[4];
    pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
    pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
    pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
    pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);

    // ---- u += P V: V pieces -> B fragments (two tokens per 32-bit register)
    uint32_t vr[4][4];  // [token slot: 2t4, 2t4+1, 2t4+8, 2t4+9][4 x bf16x2 of 8 d's] per half
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
      for (int ts = 0; ts < 4; ++ts) {
        const int c = 2 * ts + half;  // piece: token slot ts, d half
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(vr[ts][0]), "=r"(vr[ts][1]), "=r"(vr[ts][2]), "=r"(vr[ts][3])
                     : "r"(dv + (c * 32 + lane) * 16));
      }
      if (valid < BS) {  // zero V rows of uncached tokens (P is 0 there; 0 * NaN would not be)
#pragma unroll
        for (int ts = 0; ts < 4; ++ts) {
          const int tok = 2 * t4 + (ts & 1) + 8 * (ts >> 1);
          if (tok >= valid) vr[ts][0] = vr[ts][1] = vr[ts][2] = vr[ts][3] = 0u;
        }
      }
      // output column n-tile nt holds physical d = 16*n + nt; this half covers nt in [8*half, 8*half+8)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int nt = 8 * half + 2 * w + e;
          const uint32_t sel = e ? 0x7632u : 0x5410u;
          const uint32_t bb0 = __byte_perm(vr[0][w], vr[1][w], sel);
          const uint32_t bb1 = __byte_perm(vr[2][w], vr[3][w], sel);
          mma_bf16_16816(acc[nt], pa, bb0, bb1);
        }
      }
    }
    issue(i + STAGES);
  }
  cp_async_wait<0>();

  // ---- merge the 4 warps' (m, l, u) states
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();  // all warps done with their stages: reuse shared memory
  float* so = reinterpret_cast<float*>(dsmem);              // [WARPS][MAX_G][D]
  float* sm = so + WARPS * MAX_G * D;                        // [WARPS][MAX_G]
  float* sl = sm + WARPS * MAX_G;                            // [WARPS][MAX_G]
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int d0 = 16 * (2 * t4) + nt, d1 = 16 * (2 * t4 + 1) + nt;
    so[(warp * MAX_G + gq) * D + d0] = acc[nt][0];
    so[(warp * MAX_G + gq) * D + d1] = acc[nt][1];
    so[(warp * MAX_G + gq + 8) * D + d0] = acc[nt][2];
    so[(warp * MAX_G + gq + 8) * D + d1] = acc[nt][3];
  }
  if (t4 == 0) {
    sm[warp * MAX_G + gq] = m0;
    sm[warp * MAX_G + gq + 8] = m1;
    sl[warp * MAX_G + gq] = l0;
    sl[warp * MAX_G + gq + 8] = l1;
  }
  __syncthreads();
  const bool single = nsplit == 1;
  for (int idx = threadIdx.x; idx < G * D; idx += WARPS * 32) {
    const int hr = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, sm[w * MAX_G + hr]);
    float L = 0.f, U = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float mw = sm[w * MAX_G + hr];
      const float wt = (mw == -INFINITY) ? 0.f : ex2(mw - M);
      L += sl[w * MAX_G + hr] * wt;
      U += so[(w * MAX_G + hr) * D + d] * wt;
    }
    const int h = g * G + hr;
    const float lse_nat = (M + __log2f(L)) * 0.69314718055994531f;
    if (single) {
      p.o[(size_t(r) * p.Hq + h) * D + d] = __float2bfloat16_rn(U / L);
      if (d == 0 && p.lse) p.lse[size_t(r) * p.Hq + h] = lse_nat;
    } else {
      const size_t pi = (size_t(r) * p.Hq + h) * p.max_splits + s;
      p.part_o[pi * D + d] = U / L;
      if (d == 0) p.part_lse[pi] = lse_nat;
    }
  }
}

// Merge the split partials of requests that needed more than one split: each split's
// normalised output is weighted by e^{lse_s - lse}, lse = ln sum_s e^{lse_s}.
__global__ void __launch_bounds__(128) fa_paged_decode_combine_kernel(const DecodeParams p) {
  using namespace dec;
  const int rh = blockIdx.x;
  const int r = rh / p.Hq;
  const int ctx = p.ctx[r];
  if (ctx < 1 || ctx > p.max_blocks * BS) return;
  const int nsplit = ((ctx + BS - 1) / BS + CHUNK - 1) / CHUNK;
  if (nsplit <= 1) return;
  const float* pl = p.part_lse + size_t(rh) * p.max_splits;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, pl[s]);
  float W = 0.f, U = 0.f;
  const int d = threadIdx.x;
  for (int s = 0; s < nsplit; ++s) {
    const float w = __expf(pl[s] - M);
    W += w;
    U += w * p.part_o[(size_t(rh) * p.max_splits + s) * D + d];
  }
  p.o[size_t(rh) * D + d] = __float2bfloat16_rn(U / W);
  if (d == 0 && p.lse) p.lse[rh] = M + __logf(W);
}

}  // namespace fa
