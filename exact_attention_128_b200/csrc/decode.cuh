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
// [s*chunk, (s+1)*chunk) of request r; the host picks chunk (a multiple of 4 blocks, at
// most MAX_CHUNK = 128 blocks = 2048 tokens) per call.  Each of its 4 warps takes every
// 4th block and keeps its own (m, l, u) state; the warps'
// states and then the splits' partial results are merged by weighting each part with
// its unnormalised mass e^{lse_s}
// ("No basta con promediar los resultados de los bloques": block results are never
// simply averaged).  A request that fits in one split writes its output directly.
//
// Data path: the step is bound by reading K and V from device memory.  Each warp owns
// a ring of STAGES shared-memory stages; its lane 0 prefetches the warp's block-table
// entries once, then issues TMA loads of each 4 KB (block, kv head) slab (two 64-column
// boxes with the 128-byte swizzle, so ldmatrix reads are conflict-free) addressed by the
// physical block id.  Scores and P.V use mma.sync m16n8k16 with the group's query heads
// as the 16 rows (rows >= G are zero): ldmatrix for K, ldmatrix.trans for V.
#pragma once
#include "common.cuh"

namespace fa {
namespace dec {
constexpr int D = 128;
constexpr int BS = 16;          // tokens per cache block
#ifndef FA_DEC_STAGES
#define FA_DEC_STAGES 2
#endif
constexpr int WARPS = 4;
constexpr int STAGES = FA_DEC_STAGES;  // blocks in flight per warp
constexpr int MAX_CHUNK = 128;         // largest split, in logical blocks (2048 tokens)
constexpr int MIN_CHUNK = 32;          // smallest split the host may choose (workspace sizing)
static_assert(MAX_CHUNK / WARPS <= 32, "a warp's block-table entries are held one per lane");
constexpr int SLAB = BS * D * 2;  // 4096 bytes: one (block, kv head) slab of K or V
constexpr int STAGE_BYTES = 2 * SLAB;
constexpr int OFF_BAR = WARPS * STAGES * STAGE_BYTES;
constexpr int SMEM = OFF_BAR + WARPS * STAGES * 8 + 1024;
constexpr int MAX_G = 16;
constexpr int OP = D + 8;  // padded row of the warp-merge buffer (floats)
static_assert(WARPS * MAX_G * OP * 4 + 2 * WARPS * MAX_G * 4 <= OFF_BAR, "merge buffer must fit the stages");
}  // namespace dec

struct DecodeParams {
  const __nv_bfloat16* q;
  const int* bt;
  const int* ctx;
  __nv_bfloat16* o;
  float* lse;  // may be null
  float* part_o;
  float* part_lse;
  int R, Hq, Hkv, max_blocks, num_blocks, max_splits;
  int chunk;  // logical blocks per split: a multiple of WARPS, at most MAX_CHUNK
  float scale_log2;
  uint64_t wait_ns;
};

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Byte offset of 16-byte chunk `chunk` (0..15) of slab row `row` (0..15) in a stage
// half-pair: chunks 0-7 live in the first 2 KB box, 8-15 in the second, each row 128 B
// with the 128-byte swizzle (chunk index XOR row % 8).
__device__ __forceinline__ uint32_t slab_off(int row, int chunk) {
  return uint32_t((chunk >> 3) * 2048 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(dec::WARPS * 32)
    fa_paged_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const DecodeParams p) {
  using namespace dec;
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* dsmem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  const int s = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  // launched as a programmatic dependent: wait for the grid before it on the stream (the
  // previous step's merge, or the append that wrote this step's key/value rows) to
  // complete before reading anything it may have written; the launch itself overlaps it
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int ctx = p.ctx[r];
  if (ctx < 1 || ctx > p.max_blocks * BS) {
    if (s == 0 && g == 0 && threadIdx.x == 0) set_status(FA_ERR_INVALID_ARG, 100);
    return;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int nsplit = (nblk + p.chunk - 1) / p.chunk;
  const int b0 = s * p.chunk;
  if (b0 >= nblk) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    return;
  }
  const int b1 = min(nblk, b0 + p.chunk);

  const int warp = warp_id(), lane = lane_id();
  const int gq = lane >> 2;  // mma group id: query-head row, key token, output column
  const int t4 = lane & 3;
  const int nb = max(0, (b1 - b0 - warp + WARPS - 1) / WARPS);  // this warp's blocks
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsmem + OFF_BAR) + warp * STAGES;
  const uint32_t sbase = smem_u32(dsmem) + warp * STAGES * STAGE_BYTES;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0)
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
  fence_barrier_init();
  __syncthreads();

  // physical block of this warp's i-th block, held by lane i (chunk / WARPS <= 32)
  int my_phys = 0;
  if (lane < nb) {
    my_phys = p.bt[size_t(r) * p.max_blocks + b0 + warp + lane * WARPS];
    if (my_phys < 0 || my_phys >= p.num_blocks) {
      set_status(FA_ERR_INVALID_ARG, 101);
      my_phys = 0;  // never address an out-of-range block; the result is flagged invalid
    }
  }
  // the whole warp calls issue(i) (the shuffle needs every lane); lane 0 issues the loads
  auto issue = [&](int i) {
    const int phys = __shfl_sync(0xffffffffu, my_phys, i);
    if (lane == 0) {
      const int row = (phys * p.Hkv + g) * BS;
      uint64_t* bar = &bars[i % STAGES];
      const uint32_t st = sbase + (i % STAGES) * STAGE_BYTES;
      mbar_arrive_expect_tx(bar, STAGE_BYTES);
      tma_load_2d(st, &tmK, bar, 0, row);
      tma_load_2d(st + 2048, &tmK, bar, 64, row);
      tma_load_2d(st + SLAB, &tmV, bar, 0, row);
      tma_load_2d(st + SLAB + 2048, &tmV, bar, 64, row);
    }
  };
  for (int i = 0; i < min(nb, STAGES); ++i) issue(i);

  // q fragments (A operand): rows = heads of the group (zero past G), natural d order
  uint32_t qa[8][4];
  {
    const int h0 = g * G + gq, h1 = g * G + gq + 8;
    const bool v0 = gq < G, v1 = gq + 8 < G;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(p.q + (size_t(r) * p.Hq + (v0 ? h0 : 0)) * D);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(p.q + (size_t(r) * p.Hq + (v1 ? h1 : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = v0 ? q0[8 * ks + t4] : 0u;
      qa[ks][1] = v1 ? q1[8 * ks + t4] : 0u;
      qa[ks][2] = v0 ? q0[8 * ks + 4 + t4] : 0u;
      qa[ks][3] = v1 ? q1[8 * ks + 4 + t4] : 0u;
    }
  }

  float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 units) of rows gq, gq + 8
  float l0 = 0.f, l1 = 0.f;              // this thread's share of the running sums
  float acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  const float sl2 = p.scale_log2;
  // ldmatrix row addresses: lane -> (matrix mi = lane / 8, row rr = lane % 8)
  const int mi = lane >> 3, rr = lane & 7;
  const int k_tok = rr + 8 * (mi >> 1), k_chunk_lo = mi & 1;  // K: (token, d-chunk parity)
  const int v_tok = rr + 8 * (mi & 1), v_chunk_hi = mi >> 1;  // V: (token, n-tile parity)

  bool ok = true;
  int consumed = 0;  // stages this warp has waited for (loads issued: min(nb, consumed + STAGES))
  for (int i = 0; i < nb && ok; ++i) {
    ok = warp_wait(&bars[i % STAGES], (i / STAGES) & 1, p.wait_ns, &abort_flag, 102);
    if (!ok) break;
    consumed = i + 1;
    const uint32_t sk = sbase + (i % STAGES) * STAGE_BYTES;
    const uint32_t sv = sk + SLAB;
    const int lb = b0 + warp + i * WARPS;
    const int valid = min(BS, ctx - lb * BS);  // tokens of this block that are cached

    // ---- scores S[head][token] = q . k
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t b00, b01, b10, b11;
      ldsm_x4(sk + slab_off(k_tok, 2 * ks + k_chunk_lo), b00, b01, b10, b11);
      mma_bf16_16816(sc[0], qa[ks], b00, b01);
      mma_bf16_16816(sc[1], qa[ks], b10, b11);
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
    const float n0 = fmaxf(m0, mx0 * sl2), n1 = fmaxf(m1, mx1 * sl2);  // every block has a cached token
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

    // ---- u += P V; this thread's B fragments hold tokens 2t4, 2t4+1 (b0), +8 (b1)
    uint32_t keep0 = 0xffffffffu, keep1 = 0xffffffffu;
    if (valid < BS) {  // zero V of uncached tokens (P is 0 there; 0 * NaN would not be)
      keep0 = (2 * t4 < valid ? 0x0000ffffu : 0u) | (2 * t4 + 1 < valid ? 0xffff0000u : 0u);
      keep1 = (2 * t4 + 8 < valid ? 0x0000ffffu : 0u) | (2 * t4 + 9 < valid ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int nt = 0; nt < 16; nt += 2) {
      uint32_t v00, v01, v10, v11;
      ldsm_x4_t(sv + slab_off(v_tok, nt + v_chunk_hi), v00, v01, v10, v11);
      mma_bf16_16816(acc[nt], pa, v00 & keep0, v01 & keep1);
      mma_bf16_16816(acc[nt + 1], pa, v10 & keep0, v11 & keep1);
    }
    // all lanes have read this stage: refill it
    __syncwarp();
    if (i + STAGES < nb) {
      fence_proxy_async_smem();
      issue(i + STAGES);
    }
  }

  if (!ok) {
    // A bounded wait ran out (here or in another warp): let this warp's loads that are
    // still in flight land before the CTA gives up its shared memory, each wait again
    // bounded (and no longer cut short by the abort flag).
    if (lane == 0)
      for (int i = consumed; i < min(nb, consumed + STAGES); ++i)
        mbar_wait_bounded(&bars[i % STAGES], (i / STAGES) & 1, p.wait_ns);
    __syncwarp();
  }

  // ---- merge the warps' (m, l, u) states
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();  // all warps done with their stages: reuse shared memory
  if (abort_flag) {
    // the device status word already says FA_ERR_DEVICE_TIMEOUT; mark this split's result
    // as NaN so neither the output nor the merge of the other splits looks valid
    for (int idx = threadIdx.x; idx < G * D; idx += WARPS * 32) {
      const int h = g * G + idx / D, d = idx % D;
      if (nsplit == 1) {
        p.o[(size_t(r) * p.Hq + h) * D + d] = __float2bfloat16_rn(NAN);
        if (d == 0 && p.lse) p.lse[size_t(r) * p.Hq + h] = NAN;
      } else if (d == 0) {
        p.part_lse[(size_t(r) * p.Hq + h) * p.max_splits + s] = NAN;
      }
    }
    return;
  }
  float* so = reinterpret_cast<float*>(dsmem);  // [WARPS][MAX_G][OP]
  float* sm = so + WARPS * MAX_G * OP;          // [WARPS][MAX_G]
  float* sl = sm + WARPS * MAX_G;               // [WARPS][MAX_G]
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int d0 = 8 * nt + 2 * t4;
    *reinterpret_cast<float2*>(&so[(warp * MAX_G + gq) * OP + d0]) = make_float2(acc[nt][0], acc[nt][1]);
    *reinterpret_cast<float2*>(&so[(warp * MAX_G + gq + 8) * OP + d0]) = make_float2(acc[nt][2], acc[nt][3]);
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
      U += so[(w * MAX_G + hr) * OP + d] * wt;
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
  // the merge kernel (launched as a programmatic dependent) may start scheduling now; it
  // waits for this grid's completion and memory before reading the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Append one token per request: thread group (r, h) copies the 256-byte key and value
// rows of the new token into slot pos % 16 of physical block block_table[r][pos / 16].
__global__ void __launch_bounds__(128) fa_paged_kv_append_kernel(const uint4* k_new, const uint4* v_new, uint4* kc,
                                                                 uint4* vc, const int* bt, const int* pos, int R,
                                                                 int Hkv, int max_blocks, int num_blocks) {
  using namespace dec;
  constexpr int PER_ROW = D * 2 / 16;  // 16-byte pieces per 256-byte row
  const long gid = long(blockIdx.x) * blockDim.x + threadIdx.x;
  const long rh = gid / PER_ROW;
  const int piece = int(gid % PER_ROW);
  if (rh >= long(R) * Hkv) return;
  const int r = int(rh / Hkv), h = int(rh % Hkv);
  const int t = pos[r];
  if (t < 0 || t >= max_blocks * BS) {
    if (piece == 0) set_status(FA_ERR_INVALID_ARG, 110);
    return;
  }
  const int phys = bt[size_t(r) * max_blocks + t / BS];
  if (phys < 0 || phys >= num_blocks) {
    if (piece == 0) set_status(FA_ERR_INVALID_ARG, 111);
    return;
  }
  const size_t dst = ((size_t(phys) * Hkv + h) * BS + t % BS) * PER_ROW + piece;
  kc[dst] = k_new[rh * PER_ROW + piece];
  vc[dst] = v_new[rh * PER_ROW + piece];
}

// Merge the split partials of requests that needed more than one split: each split's
// normalised output is weighted by e^{lse_s - lse}, lse = ln sum_s e^{lse_s}.
__global__ void __launch_bounds__(128) fa_paged_decode_combine_kernel(const DecodeParams p) {
  using namespace dec;
  // launched with programmatic stream serialization: wait for the split kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int rh = blockIdx.x;
  const int r = rh / p.Hq;
  const int ctx = p.ctx[r];
  if (ctx < 1 || ctx > p.max_blocks * BS) return;
  const int nsplit = ((ctx + BS - 1) / BS + p.chunk - 1) / p.chunk;
  if (nsplit <= 1) return;
  const float* pl = p.part_lse + size_t(rh) * p.max_splits;
  const float* po = p.part_o + size_t(rh) * p.max_splits * D;
  const int d = threadIdx.x;
  // The first NPRE splits' lse and output column are all loaded before any arithmetic that
  // needs them, so their loads overlap (one L2 round trip instead of one per dependent
  // step); splits past NPRE, if any, are read as they are merged.
  constexpr int NPRE = 8;
  float lv[NPRE], ov[NPRE];
#pragma unroll
  for (int s = 0; s < NPRE; ++s)
    if (s < nsplit) {
      lv[s] = pl[s];
      ov[s] = po[size_t(s) * D + d];
    }
  float M = -INFINITY;
  bool aborted = false;  // a split whose bounded wait ran out left NaN
#pragma unroll
  for (int s = 0; s < NPRE; ++s)
    if (s < nsplit) {
      M = fmaxf(M, lv[s]);
      aborted |= isnan(lv[s]);
    }
  for (int s = NPRE; s < nsplit; ++s) {
    M = fmaxf(M, pl[s]);
    aborted |= isnan(pl[s]);
  }
  if (aborted) {
    p.o[size_t(rh) * D + d] = __float2bfloat16_rn(NAN);
    if (d == 0 && p.lse) p.lse[rh] = NAN;
    return;
  }
  float W = 0.f, U = 0.f;
#pragma unroll
  for (int s = 0; s < NPRE; ++s)
    if (s < nsplit) {
      const float w = __expf(lv[s] - M);
      W += w;
      U += w * ov[s];
    }
  for (int s = NPRE; s < nsplit; ++s) {
    const float w = __expf(pl[s] - M);
    W += w;
    U += w * po[size_t(s) * D + d];
  }
  p.o[size_t(rh) * D + d] = __float2bfloat16_rn(U / W);
  if (d == 0 && p.lse) p.lse[rh] = M + __logf(W);
}

}  // namespace fa
