// fa_api.cu — the C ABI (include/fa.h): argument validation, TMA descriptor
// encoding and kernel launches.  Everything that computes runs in the kernels;
// this file only checks arguments and launches them on the caller's stream.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "decode.cuh"
#include "fwd_bf16.cuh"
#include "fwd_d256.cuh"
#include "fwd_f32.cuh"
#include "bwd_bf16.cuh"
#include "bwd_d256.cuh"
#include "bwd_f32.cuh"

#ifndef FA_FWD_D64_BN
#define FA_FWD_D64_BN 64
#endif
#ifndef FA_F32_SMALL_BQ
#define FA_F32_SMALL_BQ 16  // rows per CTA of the tiled fp32 forward (more than 256 keys) on
                            // small grids; on the fp32 ViT layer, before the one-pass kernel took
                            // it over, 8/16/32 rows measured 38.8/36.8/41.8 us
#endif


namespace {

using namespace fa;

uint64_t g_wait_ns = 200000000ull;  // 200 ms per wait

// Logical blocks per decode split; 0 = the library's choice (kDecodeChunk).
#ifndef FA_DEC_CHUNK
#define FA_DEC_CHUNK 128
#endif
constexpr int kDecodeChunk = FA_DEC_CHUNK;
static_assert(kDecodeChunk >= fa::dec::MIN_CHUNK && kDecodeChunk <= fa::dec::MAX_CHUNK &&
                  kDecodeChunk % fa::dec::WARPS == 0, "decode split size out of range");
int g_dec_chunk = 0;
int decode_chunk() { return g_dec_chunk > 0 ? g_dec_chunk : kDecodeChunk; }
int decode_splits(int max_blocks) { return (max_blocks + decode_chunk() - 1) / decode_chunk(); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 map over [z][y][x] = [planes][rows][d] with a (box_cols, box_rows, 1) box and
// the swizzle of its row width (64 columns: 128-byte, 32 columns: 64-byte); rows past
// `rows` read as zeros.
bool make_map_bf16(CUtensorMap* m, const void* base, int d, int rows, int planes, int box_rows,
                   int box_cols = 64) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(rows), cuuint64_t(planes)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(d) * 2 * cuuint64_t(rows)};
  cuuint32_t box[3] = {cuuint32_t(box_cols), cuuint32_t(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 map over a paged cache viewed as [rows][d] with a (64, 16) box and the
// 128-byte swizzle: one box is one 64-column block of one (block, kv head) slab.
bool make_map_cache(CUtensorMap* m, const void* base, long rows, int d = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(d) * 2};
  cuuint32_t box[2] = {64, 16};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

fa_status launched() { return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

// Launch `kernel` as a programmatic dependent on stream st: it may be launched while the
// grid before it is still finishing.  Every kernel launched this way executes
// griddepcontrol.wait before its first global access, which returns once that grid has
// completed and its writes are visible.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t c = {};
  c.gridDim = grid;
  c.blockDim = block;
  c.dynamicSmemBytes = smem;
  c.stream = st;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[0].val.programmaticStreamSerializationAllowed = 1;
  c.attrs = a;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, kernel, std::forward<Args>(args)...);
}

// Number of SMs of the current device (persistent grids use one CTA per SM).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

template <int D, int BN, bool CAUSAL, bool PAGED = false>
fa_status launch_fwd_bf16(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const CUtensorMap& mo, const FwdBf16Params& prm, int Nq, cudaStream_t st) {
  using C = FwdCfg<D, BN>;
  auto kern = fa_fwd_bf16_kernel<D, BN, CAUSAL, PAGED>;
  if (set_smem(kern, C::SMEM) != cudaSuccess) return FA_ERR_CUDA;
  const long n_qp = (Nq + 2 * C::BM - 1) / (2 * C::BM);
  // causal dense items run in units of two query-tile pairs (one CTA per unit at most)
  const long items = (CAUSAL && !PAGED ? (n_qp + 1) / 2 : n_qp) * prm.BH;
  const long slots = long(sm_count()) * C::CTAS_PER_SM;
  if (slots <= 0) return FA_ERR_CUDA;
  // programmatic dependent: its launch and prologue overlap the tail of the grid before it
  if (launch_pdl(kern, dim3(unsigned(items < slots ? items : slots)), dim3(C::THREADS), C::SMEM, st, mq, mk, mv, mo,
                 prm) != cudaSuccess)
    return FA_ERR_CUDA;
  return launched();
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

template <int D, bool CAUSAL>
fa_status launch_bwd_kernel(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const CUtensorMap& mo, const CUtensorMap& mdq, const CUtensorMap& mdk,
                            const CUtensorMap& mdv, const BwdParams& prm, int B, int Hkv, int Nkv, cudaStream_t st) {
  using C = BwdCfg<D>;
  auto kern = fa_bwd_bf16_kernel<D, CAUSAL>;
  if (set_smem(kern, C::SMEM) != cudaSuccess) return FA_ERR_CUDA;
  // 1-D grid over (key tile, (batch, kv head)) in the order bwd_tile_order gives
  dim3 grid(((Nkv + C::BN - 1) / C::BN) * B * Hkv);
  kern<<<grid, C::THREADS, C::SMEM, st>>>(mq, mk, mv, mo, mdq, mdk, mdv, prm);
  return launched();
}

// 3-D fp32 map over the dQ accumulator [planes][rows][d] with a (32, 32, 1) box and the
// 128-byte swizzle (for TMA reduce-adds).
bool make_map_f32(CUtensorMap* m, const void* base, int d, int rows, int planes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(rows), cuuint64_t(planes)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 4, cuuint64_t(d) * 4 * cuuint64_t(rows)};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Backward: preprocess (D, padded lse, zeroed dQ accumulator), the tensor-core kernel,
// and, for bf16 gradients, the dQ cast.  Workspace: [dQ fp32][lse2 pad][D pad].
fa_status bwd_launch(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                     void* dq, void* dk, void* dv, fa_dtype grad_dtype, int B, int Hq, int Hkv, int Nq, int Nkv,
                     int d, float scale, int causal, void* workspace, cudaStream_t st) {
  const int Nq_pad = round_up(Nq, 128);
  const size_t rows = size_t(B) * Hq * Nq;
  const size_t rows_pad = size_t(B) * Hq * Nq_pad;
  char* ws = static_cast<char*>(workspace);
  float* dq_ws = reinterpret_cast<float*>(ws);
  float* lse2 = reinterpret_cast<float*>(ws + align256(rows * d * 4));
  float* dstat = reinterpret_cast<float*>(ws + align256(rows * d * 4) + align256(rows_pad * 4));
  float* dq_acc = grad_dtype == FA_DTYPE_F32 ? static_cast<float*>(dq) : dq_ws;

  const long pre_threads = long(rows_pad) * 8;
  const int pre_blocks = int((pre_threads + 255) / 256);
  if (d == 64)
    fa_bwd_preprocess_kernel<64><<<pre_blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2, dstat, dq_acc,
        long(rows_pad), Nq, Nq_pad, long(rows) * d, scale);
  else if (d == 96)
    fa_bwd_preprocess_kernel<96><<<pre_blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2, dstat, dq_acc,
        long(rows_pad), Nq, Nq_pad, long(rows) * d, scale);
  else if (d == 128)
    fa_bwd_preprocess_kernel<128><<<pre_blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2, dstat, dq_acc,
        long(rows_pad), Nq, Nq_pad, long(rows) * d, scale);
  else
    fa_bwd_preprocess_kernel<256><<<pre_blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2, dstat, dq_acc,
        long(rows_pad), Nq, Nq_pad, long(rows) * d, scale);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;

  if (d == 256) {
    // one CTA per (128-key tile, batch * kv head, half of the head dimension); 64-row query
    // steps (bwd_d256.cuh)
    using C = Bwd256Cfg;
    CUtensorMap mq, mk, mv, mo, mdq;
    if (!make_map_bf16(&mq, q, d, Nq, B * Hq, C::BM) || !make_map_bf16(&mk, k, d, Nkv, B * Hkv, C::BN) ||
        !make_map_bf16(&mv, v, d, Nkv, B * Hkv, C::BN) || !make_map_bf16(&mo, dO, d, Nq, B * Hq, C::BM) ||
        !make_map_f32(&mdq, dq_acc, d, Nq, B * Hq))
      return FA_ERR_CUDA;
    BwdParams prm{dq_acc, lse2, dstat, dk, dv, grad_dtype == FA_DTYPE_BF16 ? 1 : 0, d, Hq, Hkv, Nq, Nkv, Nq_pad,
                  scale, scale * 1.4426950408889634f, g_wait_ns};
    auto kern = causal ? fa_bwd_d256_kernel<true> : fa_bwd_d256_kernel<false>;
    if (set_smem(kern, C::SMEM) != cudaSuccess) return FA_ERR_CUDA;
    // 1-D grid over (key tile, (batch, kv head, half)) in the order bwd_tile_order gives
    kern<<<dim3(((Nkv + C::BN - 1) / C::BN) * B * Hkv * 2), C::THREADS, C::SMEM, st>>>(mq, mk, mv, mo, mdq, prm);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    if (grad_dtype == FA_DTYPE_BF16) {
      const long n = long(rows) * d;
      fa_bwd_finalize_kernel<<<int((n / 4 + 255) / 256), 256, 0, st>>>(dq_ws, static_cast<__nv_bfloat16*>(dq), n);
      return launched();
    }
    return FA_OK;
  }

  CUtensorMap mq, mk, mv, mo, mdq, mdk, mdv;
  if (!make_map_bf16(&mq, q, d, Nq, B * Hq, 128) || !make_map_bf16(&mk, k, d, Nkv, B * Hkv, 128) ||
      !make_map_bf16(&mv, v, d, Nkv, B * Hkv, 128) || !make_map_bf16(&mo, dO, d, Nq, B * Hq, 128) ||
      !make_map_f32(&mdq, dq_acc, d, Nq, B * Hq))
    return FA_ERR_CUDA;
  // dk, dv for the epilogue's TMA stores
  if (grad_dtype == FA_DTYPE_BF16 ? !make_map_bf16(&mdk, dk, d, Nkv, B * Hkv, 32) || !make_map_bf16(&mdv, dv, d, Nkv, B * Hkv, 32)
                                  : !make_map_f32(&mdk, dk, d, Nkv, B * Hkv) || !make_map_f32(&mdv, dv, d, Nkv, B * Hkv))
    return FA_ERR_CUDA;
  // d = 96 runs the d = 128 kernel on 96-wide maps (zero-filled columns 96..127); its
  // gradient rows are written 96 wide
  BwdParams prm{dq_acc, lse2, dstat, dk, dv, grad_dtype == FA_DTYPE_BF16 ? 1 : 0, d, Hq, Hkv, Nq, Nkv, Nq_pad,
                scale, scale * 1.4426950408889634f, g_wait_ns};
  fa_status s;
  if (d == 64)
    s = causal ? launch_bwd_kernel<64, true>(mq, mk, mv, mo, mdq, mdk, mdv, prm, B, Hkv, Nkv, st)
               : launch_bwd_kernel<64, false>(mq, mk, mv, mo, mdq, mdk, mdv, prm, B, Hkv, Nkv, st);
  else
    s = causal ? launch_bwd_kernel<128, true>(mq, mk, mv, mo, mdq, mdk, mdv, prm, B, Hkv, Nkv, st)
               : launch_bwd_kernel<128, false>(mq, mk, mv, mo, mdq, mdk, mdv, prm, B, Hkv, Nkv, st);
  if (s != FA_OK) return s;
  if (grad_dtype == FA_DTYPE_BF16) {
    const long n = long(rows) * d;
    fa_bwd_finalize_kernel<<<int((n / 4 + 255) / 256), 256, 0, st>>>(dq_ws, static_cast<__nv_bfloat16*>(dq), n);
    return launched();
  }
  return FA_OK;
}

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait(&bar, 0, limit_ns, &abort_flag, 900);  // nothing arrives: must run out
  }
}

}  // namespace

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_DEVICE_TIMEOUT: return "bounded in-kernel wait timed out";
  }
  return "unknown status";
}

int fa_version(void) { return 10000; }

void fa_set_wait_limit_ns(uint64_t ns) { g_wait_ns = ns < 1000 ? 1000 : ns; }

fa_status fa_device_status(int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (reset) {
    int z = 0;
    if (cudaMemcpyToSymbol(fa::g_status, &z, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemcpyToSymbol(fa::g_status_where, &z, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  }
  return static_cast<fa_status>(v);
}

fa_status fa_selftest_wait_timeout(void* stream) {
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(g_wait_ns);
  return launched();
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                 int Nkv, int d, float scale, int causal, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nkv <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (causal && Nq > Nkv) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARG;
  if (long(B) * Hq > 65535) return FA_ERR_UNSUPPORTED;
  if (long((Nq + 255) / 256) * B * Hq > 0x7fffffffL) return FA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  if (dtype == FA_DTYPE_F32) {
    if (d != 64) return FA_ERR_UNSUPPORTED;
    FwdF32Params prm{static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
                     static_cast<float*>(o), lse, Hq, Hkv, Nq, Nkv, scale, causal};
    if (Nkv <= f32::SMALL_NKV) {
      // every key of a head fits in shared memory: one pass per 32-row CTA
      const size_t sb = fwd_f32_small_smem(Nkv);
      if (set_smem(fa_fwd_f32_small_kernel, int(sb)) != cudaSuccess) return FA_ERR_CUDA;
      fa_fwd_f32_small_kernel<<<dim3((Nq + f32::SROWS - 1) / f32::SROWS, B * Hq), f32::STHREADS, sb, st>>>(prm);
      return launched();
    }
    // 64-row CTAs, or 16-row CTAs when the former would leave SMs idle (a single ViT layer
    // has 4 x 12 of them for 148 SMs)
    if (long((Nq + 63) / 64) * B * Hq < 2L * sm_count()) {
      fa_fwd_f32_kernel<FA_F32_SMALL_BQ><<<dim3((Nq + FA_F32_SMALL_BQ - 1) / FA_F32_SMALL_BQ, B * Hq),
                                          4 * FA_F32_SMALL_BQ, 0, st>>>(prm);
    } else {
      fa_fwd_f32_kernel<f32::BQ><<<dim3((Nq + f32::BQ - 1) / f32::BQ, B * Hq), f32::THREADS, 0, st>>>(prm);
    }
    return launched();
  }
  if (dtype != FA_DTYPE_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 96 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;

  if (d == 256) {  // one query tile per CTA, double-buffered scores (fwd_d256.cuh)
    CUtensorMap mq, mk, mv;
    if (!make_map_bf16(&mq, q, d, Nq, B * Hq, D256Cfg::BM) || !make_map_bf16(&mk, k, d, Nkv, B * Hkv, D256Cfg::BN) ||
        !make_map_bf16(&mv, v, d, Nkv, B * Hkv, D256Cfg::BN))
      return FA_ERR_CUDA;
    FwdBf16Params prm{static_cast<__nv_bfloat16*>(o), lse, B * Hq, Hq, Hkv, Nq, Nkv,
                      scale * 1.4426950408889634f, g_wait_ns, nullptr, nullptr, nullptr, 0, 0};
    auto kern = causal ? fa_fwd_d256_kernel<true> : fa_fwd_d256_kernel<false>;
    if (set_smem(kern, D256Cfg::SMEM) != cudaSuccess) return FA_ERR_CUDA;
    const long items = long((Nq + D256Cfg::BM - 1) / D256Cfg::BM) * B * Hq;
    const long slots = sm_count();
    if (slots <= 0) return FA_ERR_CUDA;
    kern<<<int(items < slots ? items : slots), D256Cfg::THREADS, D256Cfg::SMEM, st>>>(mq, mk, mv, prm);
    return launched();
  }
  constexpr int BN64 = FA_FWD_D64_BN;  // key-tile width of the d = 64 kernel
  const int bn = d == 64 ? BN64 : 128;
  const int stg_cols = d == 64 ? FwdCfg<64, BN64>::STG_COLS : FwdCfg<128, 128>::STG_COLS;
  // d = 96 runs the d = 128 kernel: the maps' rows are 96 wide, so TMA loads fill columns
  // 96..127 with zeros (adding nothing to Q K^T, giving zero columns of O) and the O stores
  // drop them
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_bf16(&mq, q, d, Nq, B * Hq, 128) || !make_map_bf16(&mk, k, d, Nkv, B * Hkv, bn) ||
      !make_map_bf16(&mv, v, d, Nkv, B * Hkv, bn) || !make_map_bf16(&mo, o, d, Nq, B * Hq, 32, stg_cols))
    return FA_ERR_CUDA;
  FwdBf16Params prm{static_cast<__nv_bfloat16*>(o), lse, B * Hq, Hq, Hkv, Nq, Nkv,
                    scale * 1.4426950408889634f, g_wait_ns, nullptr, nullptr, nullptr, 0, 0};
  if (d == 64)
    return causal ? launch_fwd_bf16<64, BN64, true>(mq, mk, mv, mo, prm, Nq, st)
                  : launch_fwd_bf16<64, BN64, false>(mq, mk, mv, mo, prm, Nq, st);
  return causal ? launch_fwd_bf16<128, 128, true>(mq, mk, mv, mo, prm, Nq, st)
                : launch_fwd_bf16<128, 128, false>(mq, mk, mv, mo, prm, Nq, st);
}

fa_status fa_paged_prefill(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                           const int* ctx_lens, const int* q_lens, void* o, float* lse, int R, int Hq, int Hkv,
                           int Nq_max, int d, int block_size, int max_blocks_per_seq, int num_blocks, float scale,
                           int causal, fa_dtype dtype, void* stream) {
  if (!q || !k_cache || !v_cache || !block_table || !ctx_lens || !q_lens || !o || !lse) return FA_ERR_INVALID_ARG;
  if (R <= 0 || Hq <= 0 || Hkv <= 0 || Nq_max <= 0 || d <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 ||
      num_blocks <= 0)
    return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(block_table, 4) || !aligned(ctx_lens, 4) || !aligned(q_lens, 4))
    return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 || (d != 64 && d != 96 && d != 128) || block_size != 16) return FA_ERR_UNSUPPORTED;
  if (long(R) * Hq > 65535) return FA_ERR_UNSUPPORTED;
  const long cache_rows = long(num_blocks) * Hkv * 16;
  if (cache_rows > 0x7fffffffL || long(max_blocks_per_seq) * 16 > 0x7fffffffL) return FA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap mq, mk, mv, mo;
  constexpr int BN64 = FA_FWD_D64_BN;
  const int stg_cols = d == 64 ? FwdCfg<64, BN64>::STG_COLS : FwdCfg<128, 128>::STG_COLS;
  if (!make_map_bf16(&mq, q, d, Nq_max, R * Hq, 128) || !make_map_bf16(&mo, o, d, Nq_max, R * Hq, 32, stg_cols) ||
      !make_map_cache(&mk, k_cache, cache_rows, d) || !make_map_cache(&mv, v_cache, cache_rows, d))
    return FA_ERR_CUDA;
  // causal item order: requests in groups whose K/V (bounded by the block table's width)
  // takes at most 32 MB, a quarter of L2, so that it stays there while the group runs
  const long kv_bytes = long(Hkv) * max_blocks_per_seq * 16 * d * 2 * 2;
  const int group = int(std::max(1L, std::min(long(R), (32L << 20) / kv_bytes)));
  FwdBf16Params prm{static_cast<__nv_bfloat16*>(o), lse, R * Hq, Hq, Hkv, Nq_max, 0,
                    scale * 1.4426950408889634f, g_wait_ns, block_table, ctx_lens, q_lens, max_blocks_per_seq,
                    num_blocks, group};
  if (d == 64)
    return causal ? launch_fwd_bf16<64, BN64, true, true>(mq, mk, mv, mo, prm, Nq_max, st)
                  : launch_fwd_bf16<64, BN64, false, true>(mq, mk, mv, mo, prm, Nq_max, st);
  return causal ? launch_fwd_bf16<128, 128, true, true>(mq, mk, mv, mo, prm, Nq_max, st)
                : launch_fwd_bf16<128, 128, false, true>(mq, mk, mv, mo, prm, Nq_max, st);
}

size_t fa_bwd_workspace_size(int B, int Hq, int Nq, int d) {
  if (B <= 0 || Hq <= 0 || Nq <= 0 || d <= 0) return 0;
  const size_t rows = size_t(B) * Hq * Nq;
  const size_t rows_pad = size_t(B) * Hq * size_t((Nq + 127) / 128 * 128);
  return align256(rows * d * sizeof(float)) + 2 * align256(rows_pad * sizeof(float));
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                 void* dq, void* dk, void* dv, fa_dtype grad_dtype, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                 float scale, int causal, fa_dtype dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nkv <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (causal && Nq > Nkv) return FA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, dO, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned(ptr, 16)) return FA_ERR_INVALID_ARG;
  if (!aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  if (dtype == FA_DTYPE_F32) {
    // fp32 inputs: CUDA-core kernels (bwd_f32.cuh), fp32 gradients, d = 64
    if (d != b32::D || grad_dtype != FA_DTYPE_F32) return FA_ERR_UNSUPPORTED;
    if (long(B) * Hq > 65535 || long(B) * Hkv > 65535) return FA_ERR_UNSUPPORTED;
    const long rows = long(B) * Hq * Nq;
    if (!workspace || workspace_bytes < fa_bwd_workspace_size(B, Hq, Nq, d) || !aligned(workspace, 256))
      return FA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    BwdF32Params prm{static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
                     static_cast<const float*>(o), lse, static_cast<const float*>(dO), static_cast<float*>(dq),
                     static_cast<float*>(dk), static_cast<float*>(dv), static_cast<float*>(workspace), Hq, Hkv, Nq,
                     Nkv, scale, causal};
    fa_bwd_f32_pre_kernel<<<unsigned((rows + 7) / 8), 256, 0, st>>>(prm.o, prm.dO, prm.Dvec, rows);
    // 32-row blocks (16-row blocks, though they fill more SMs on a single ViT layer, were
    // measured slower: 197 vs 185 us for that layer's forward + backward)
    {
      // the dK/dV and the dQ CTAs in one grid, so that they share the SMs
      const long n_kb = (Nkv + 31) / 32, n_qb = (Nq + 31) / 32;
      const long n_dkdv = n_kb * B * Hkv, n_all = n_dkdv + n_qb * B * Hq;
      if (n_all > 0x7fffffffL) return FA_ERR_UNSUPPORTED;
      fa_bwd_f32_kernel<32><<<unsigned(n_all), 256, 0, st>>>(prm, int(n_kb), int(n_dkdv), int(n_qb));
    }
    return launched();
  }
  if (dtype != FA_DTYPE_BF16) return FA_ERR_UNSUPPORTED;
  if (grad_dtype != FA_DTYPE_F32 && grad_dtype != FA_DTYPE_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 96 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (long(B) * Hq > 65535) return FA_ERR_UNSUPPORTED;
  const size_t need = fa_bwd_workspace_size(B, Hq, Nq, d);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FA_ERR_WORKSPACE;
  return bwd_launch(q, k, v, o, lse, dO, dq, dk, dv, grad_dtype, B, Hq, Hkv, Nq, Nkv, d, scale, causal, workspace,
                    static_cast<cudaStream_t>(stream));
}

fa_status fa_paged_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int* block_table, const int* positions, int R, int Hkv, int d, int block_size,
                             int max_blocks_per_seq, int num_blocks, fa_dtype dtype, void* stream) {
  if (!k_new || !v_new || !k_cache || !v_cache || !block_table || !positions) return FA_ERR_INVALID_ARG;
  if (R <= 0 || Hkv <= 0 || d <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0)
    return FA_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_table, 4) || !aligned(positions, 4))
    return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 || d != dec::D || block_size != dec::BS) return FA_ERR_UNSUPPORTED;
  const long threads = long(R) * Hkv * (dec::D * 2 / 16);
  fa_paged_kv_append_kernel<<<int((threads + 127) / 128), 128, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), block_table, positions, R, Hkv, max_blocks_per_seq, num_blocks);
  return launched();
}

size_t fa_paged_decode_workspace_size(int R, int Hq, int d, int max_blocks_per_seq, int block_size) {
  if (R <= 0 || Hq <= 0 || d <= 0 || max_blocks_per_seq <= 0 || block_size <= 0) return 0;
  const size_t splits = size_t(decode_splits(max_blocks_per_seq));
  return align256(size_t(R) * Hq * splits * d * sizeof(float)) + align256(size_t(R) * Hq * splits * sizeof(float));
}

int fa_set_decode_split(int blocks) {
  if (blocks != 0 && (blocks < dec::MIN_CHUNK || blocks > dec::MAX_CHUNK || blocks % dec::WARPS != 0)) return -1;
  const int old = g_dec_chunk;
  g_dec_chunk = blocks;
  return old;
}

fa_status fa_paged_decode(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                          const int* ctx_lens, void* o, float* lse, int R, int Hq, int Hkv, int d, int block_size,
                          int max_blocks_per_seq, int num_blocks, float scale, fa_dtype dtype, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!q || !k_cache || !v_cache || !block_table || !ctx_lens || !o) return FA_ERR_INVALID_ARG;
  if (R <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0)
    return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
      !aligned(block_table, 4) || !aligned(ctx_lens, 4) || (lse && !aligned(lse, 4)))
    return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 || d != dec::D || block_size != dec::BS) return FA_ERR_UNSUPPORTED;
  if (Hq / Hkv > dec::MAX_G || R > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
  const size_t need = fa_paged_decode_workspace_size(R, Hq, d, max_blocks_per_seq, block_size);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FA_ERR_WORKSPACE;
  const int chunk = decode_chunk();
  const int max_splits = decode_splits(max_blocks_per_seq);
  float* part_o = static_cast<float*>(workspace);
  float* part_lse =
      reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(size_t(R) * Hq * max_splits * d * 4));
  DecodeParams prm{static_cast<const __nv_bfloat16*>(q), block_table, ctx_lens, static_cast<__nv_bfloat16*>(o),
                   lse, part_o, part_lse, R, Hq, Hkv, max_blocks_per_seq, num_blocks, max_splits, chunk,
                   scale * 1.4426950408889634f, g_wait_ns};
  CUtensorMap mk, mv;
  const long cache_rows = long(num_blocks) * Hkv * dec::BS;
  if (!make_map_cache(&mk, k_cache, cache_rows) || !make_map_cache(&mv, v_cache, cache_rows)) return FA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (set_smem(fa_paged_decode_kernel, dec::SMEM) != cudaSuccess) return FA_ERR_CUDA;
  // programmatic dependent: the split kernel's launch overlaps the tail of the grid before it
  if (launch_pdl(fa_paged_decode_kernel, dim3(max_splits, Hkv, R), dim3(dec::WARPS * 32), dec::SMEM, st, mk, mv,
                 prm) != cudaSuccess)
    return FA_ERR_CUDA;
  // the merge is a programmatic dependent launch: its launch overlaps the split kernel's
  // tail and it waits (griddepcontrol.wait) for the split kernel's results
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(R * Hq);
  cfg.blockDim = dim3(dec::D);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa_paged_decode_combine_kernel, prm) != cudaSuccess) return FA_ERR_CUDA;
  return launched();
}

}  // extern "C"

// ------------------------------------------------------------------------------
// Paged decode without a caller workspace.
//
// Some callers cannot call cudaMalloc: plugins hosted inside a framework that owns
// every device allocation and offers its kernels no workspace, and latency-critical
// serving loops that must not allocate after start-up (cudaMalloc may synchronise the
// device and takes an unbounded time).  fa_paged_decode_noalloc gives them the same
// decode step with its split-KV scratch in a fixed array that lives in this library's
// device image: every GPU that loads the library holds FA_NOALLOC_SCRATCH_BYTES of it
// until the process exits.
// ------------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
  unsigned long long ctx_id;  // CUDA context the address belongs to (unique per context)
  void* ptr;
};
ScratchAddr g_noalloc_addr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (0 if it cannot be had).  A
// context that is destroyed and re-created (cudaDeviceReset) gets a new id, and its copy
// of the library's device image a new address.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call in each CUDA context of
// the device (once per device, unless its context is reset), and cached.
fa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ScratchAddr& a = g_noalloc_addr[dev];
  const unsigned long long id = current_ctx_id();
  if (!a.ptr || id == 0 || id != a.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FA_ERR_CUDA;
    a.ptr = p;
    a.ctx_id = id != 0 ? id : current_ctx_id();  // the lookup may have made the context current
  }
  *out = a.ptr;
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_paged_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                             const int* block_table, const int* ctx_lens, void* o, float* lse,
                                             int R, int Hq, int Hkv, int d, int block_size, int max_blocks_per_seq,
                                             int num_blocks, float scale, fa_dtype dtype, void* stream) {
  const size_t need = fa_paged_decode_workspace_size(R, Hq, d, max_blocks_per_seq, block_size);
  if (need > size_t(FA_NOALLOC_SCRATCH_BYTES)) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  // Invalid sizes give need == 0; fa_paged_decode then reports the argument error.
  if (need > 0) {
    const fa_status s = noalloc_scratch(&scratch);
    if (s != FA_OK) return s;
  }
  return fa_paged_decode(q, k_cache, v_cache, block_table, ctx_lens, o, lse, R, Hq, Hkv, d, block_size,
                         max_blocks_per_seq, num_blocks, scale, dtype, scratch, need, stream);
}
