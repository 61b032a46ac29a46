/*
 * fa.h — C ABI of the B200 (sm_100a) exact-attention library.
 *
 * The operation is exact scaled-dot-product attention, O = softmax(Q K^T * scale) V,
 * computed tile by tile with the online-softmax recurrence (running maximum m, sum
 * l = sum_j e^{s_j - m}, numerator u = sum_j e^{s_j - m} v_j; l and u rescaled by
 * e^{m - m'} whenever a tile raises the maximum; output u / l), so the Nq x Nkv score
 * matrix never reaches device memory.
 *   - Definition: "Autoatención, kernels CUDA y FlashAttention", §1 (Scores = QK^T /
 *     sqrt(d_k); row softmax; Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V; heads in
 *     parallel).
 *   - Blocked evaluation and recomputation in the backward pass: same page, §3
 *     ("Procesamiento por bloques", "El truco de Softmax en línea", "Recálculo durante
 *     la retropropagación").
 *   - The (m, l, u) recurrence and why block results cannot be averaged: "FlashAttention"
 *     (paweldubiel.com notes), "No basta con promediar los resultados de los bloques".
 *   - GQA: same page, "Mecanismo y detalles", last paragraph.
 *   - Paged KV cache and block table: "Kernels de atención rápida y fusión de operadores"
 *     (the-ai.news), "Atención tipo FlashAttention y atención paginada".
 *
 * Conventions common to every entry point
 *   - All tensor pointers are DEVICE pointers to contiguous row-major arrays, at least
 *     16-byte aligned.  The caller owns every buffer, workspaces included; the library
 *     never allocates device memory.  Its only state between calls is the process-wide
 *     settings of fa_set_wait_limit_ns and fa_set_decode_split and, for
 *     fa_paged_decode_noalloc, the cached address of its scratch array.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream).  FA_OK means the launch was accepted.  Faults that
 *     happen while the kernel runs surface at the caller's next synchronisation.
 *   - Arguments are validated on the host before anything is launched.  Nothing is
 *     launched when a call returns an error.  There is no CPU fallback and no
 *     alternative backend: unsupported input is an error (FA_ERR_UNSUPPORTED).
 *   - Layouts: q, o [B, Hq, Nq, d]; k, v [B, Hkv, Nkv, d]; lse [B, Hq, Nq] fp32.
 *     Query head h reads key/value head h / (Hq / Hkv) (GQA, contiguous groups).
 *   - lse = m + ln(l) of the scaled scores (natural log), one per query row.
 *   - Causal masking is bottom-right aligned: query i may attend keys
 *     j <= i + (Nkv - Nq).  causal with Nq > Nkv is rejected.
 *   - Every waiting loop inside the kernels is bounded; a wait that runs out sets a
 *     device status word (read with fa_device_status) and the kernel returns early.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, misalignment, bad shape */
  FA_ERR_UNSUPPORTED = 2,   /* valid but not built: head dim, dtype, block size */
  FA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed at launch time */
  FA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than the size query says */
  FA_ERR_DEVICE_TIMEOUT = 5 /* a bounded in-kernel wait ran out (see fa_device_status) */
} fa_status;

typedef enum { FA_DTYPE_F32 = 0, FA_DTYPE_BF16 = 1 } fa_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(fa_status s);

/* Library version as an integer (major*10000 + minor*100 + patch). */
int fa_version(void);

/*
 * fa_fwd — forward pass.  Writes O (dtype `dtype`) and lse (fp32).
 *   q [B,Hq,Nq,d], k and v [B,Hkv,Nkv,d], o [B,Hq,Nq,d]: dtype `dtype`.
 *   lse [B,Hq,Nq] fp32, may not be NULL.
 *   dtype BF16: d in {64, 96, 128, 256}, tcgen05 tensor-core kernels, fp32 accumulation,
 *   P rounded to bf16 before P·V (d == 96 runs the d == 128 kernel on zero-filled
 *   columns; d == 256 has its own one-query-tile kernel).  dtype F32: fp32 SIMT kernel,
 *   d == 64.
 *   scale > 0 (usually 1/sqrt(d)); causal 0 or 1.
 * Errors: FA_ERR_INVALID_ARG (null/misaligned pointer, size <= 0, Hq % Hkv != 0,
 * scale not finite or <= 0, causal && Nq > Nkv); FA_ERR_UNSUPPORTED (other d or dtype).
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int Nq, int Nkv, int d, float scale, int causal,
                 fa_dtype dtype, void* stream);

/*
 * fa_bwd_workspace_size — bytes of device workspace fa_bwd needs: an fp32 dQ
 * accumulator [B,Hq,Nq,d], then lse in base 2 and D_i = sum_c dO_ic O_ic, each
 * [B,Hq,ceil(Nq/128)*128] fp32; every region 256-byte aligned.  Returns 0 for invalid
 * sizes.
 */
size_t fa_bwd_workspace_size(int B, int Hq, int Nq, int d);

/*
 * fa_bwd — backward pass of fa_fwd, recomputing the score tiles from lse instead of
 * storing them ("Recálculo durante la retropropagación").
 *   q, k, v, o, dO: dtype `dtype` (BF16 only), layouts as in fa_fwd; lse from fa_fwd.
 *   dq [B,Hq,Nq,d], dk and dv [B,Hkv,Nkv,d] of dtype `grad_dtype` (F32 or BF16); dk
 *   and dv are summed over the Hq/Hkv query heads that share a key/value head.
 *   workspace: at least fa_bwd_workspace_size(B,Hq,Nq,d) bytes, 256-byte aligned;
 *   its contents on entry do not matter.
 *   dtype BF16: d in {64, 96, 128, 256}, tensor-core kernels (d == 96 on the d == 128
 *   kernel; d == 256 on a kernel whose CTAs each own one half of the head dimension and
 *   recompute the full-d score tiles).  dtype F32: d == 64 and grad_dtype F32, CUDA-core
 *   kernels (fp32 products throughout).
 * Errors: as fa_fwd, plus FA_ERR_WORKSPACE.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv, fa_dtype grad_dtype,
                 int B, int Hq, int Hkv, int Nq, int Nkv, int d, float scale, int causal,
                 fa_dtype dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_paged_decode_workspace_size — bytes of device workspace fa_paged_decode needs
 * for the split-KV partial results: fp32 O [R,Hq,splits,d] and lse [R,Hq,splits], each
 * 256-byte aligned, with splits = ceil(max_blocks_per_seq / split size) for the split
 * size in force (see fa_set_decode_split).  Returns 0 for invalid sizes.
 */
size_t fa_paged_decode_workspace_size(int R, int Hq, int d, int max_blocks_per_seq, int block_size);

/*
 * fa_paged_decode — one decode step over a paged KV cache ("Atención tipo
 * FlashAttention y atención paginada": a block table links logical positions to
 * fixed-size physical blocks, and the kernel translates every position through it).
 *   q [R,Hq,d] bf16: one new query token per request.
 *   k_cache, v_cache [num_blocks, Hkv, block_size, d] bf16.
 *   block_table [R, max_blocks_per_seq] int32: logical block -> physical block.
 *     Entries at or past ceil(ctx_lens[r] / block_size) are never read.
 *   ctx_lens [R] int32 (device): cached tokens of request r, 1 <= ctx <=
 *     max_blocks_per_seq * block_size.  The query attends to all of them.
 *   o [R,Hq,d] bf16.  lse [R,Hq] fp32 or NULL.
 *   d == 128, block_size == 16.
 *   A physical block id outside [0, num_blocks) or a ctx_len out of range is not
 *   dereferenced: the kernel skips it and sets the device status word
 *   (FA_ERR_INVALID_ARG), so the result for that request is undefined.
 *   Work split: each request's blocks are cut into splits of a fixed number of blocks
 *   (fa_set_decode_split), one CTA per (split, key/value head, request); splits of one
 *   request are merged by their lse weights.  The result does not depend on the split
 *   size beyond fp32 rounding order.
 *   If a bounded in-kernel wait runs out (fa_device_status then reports
 *   FA_ERR_DEVICE_TIMEOUT), o and lse of the affected requests are undefined (the
 *   kernels write NaN there rather than leftover partial results).
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE.
 */
fa_status fa_paged_decode(const void* q, const void* k_cache, const void* v_cache,
                          const int* block_table, const int* ctx_lens, void* o, float* lse,
                          int R, int Hq, int Hkv, int d, int block_size, int max_blocks_per_seq,
                          int num_blocks, float scale, fa_dtype dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_set_decode_split — number of cache blocks per split of fa_paged_decode (a multiple
 * of 4 in [32, 128]; 0 restores the library's default, 128 blocks = 2048 tokens at
 * block_size 16) for calls made after it, process-wide.  Smaller splits spread long
 * contexts over more CTAs at the cost of more partial results to merge.  The workspace
 * size depends on it: query fa_paged_decode_workspace_size after setting it.  Returns
 * the previous setting, or -1 (and changes nothing) for a value out of range.
 */
int fa_set_decode_split(int blocks);

/*
 * fa_paged_prefill — forward pass of a batch of variable-length sequences whose keys and
 * values sit in a paged KV cache ("Atención tipo FlashAttention y atención paginada": a
 * block table links logical positions to fixed-size physical blocks; the same page's
 * tiled online-softmax forward is run over the blocks the table names).
 *   Request r has ctx_lens[r] cached tokens (its keys and values, already written to the
 *   cache, e.g. by fa_paged_kv_append) and q_lens[r] query rows, which are the LAST
 *   q_lens[r] positions of its sequence (1 <= q_lens[r] <= ctx_lens[r]; equal for a
 *   fresh prompt, smaller for a chunk of a prompt whose earlier part is cached).
 *   q [R,Hq,Nq_max,d] bf16: query row i of request r at q[r,:,i,:], i < q_lens[r];
 *     q_lens[r] <= Nq_max.  Rows i >= q_lens[r] are not read into any result.
 *   k_cache, v_cache [num_blocks, Hkv, block_size, d] bf16; block_table [R,
 *     max_blocks_per_seq] int32 (entries at or past ceil(ctx_lens[r] / block_size) are
 *     never read); ctx_lens, q_lens [R] int32 (device).
 *   causal: 1 = query row i sees keys j <= i + ctx_lens[r] - q_lens[r] (its own position
 *     and every earlier one); 0 = it sees all ctx_lens[r] keys.
 *   o [R,Hq,Nq_max,d] bf16 and lse [R,Hq,Nq_max] fp32 (natural log): rows i >= q_lens[r]
 *     are left undefined (o) or untouched (lse).
 *   d in {64, 96, 128} (as fa_fwd), block_size == 16, GQA as in fa_fwd.
 *   A length or block id out of range is not dereferenced: the kernel skips that request
 *   (or reads block 0 for the bad entry) and sets the device status word
 *   (FA_ERR_INVALID_ARG), so that request's result is undefined.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA.
 */
fa_status fa_paged_prefill(const void* q, const void* k_cache, const void* v_cache,
                           const int* block_table, const int* ctx_lens, const int* q_lens,
                           void* o, float* lse, int R, int Hq, int Hkv, int Nq_max, int d,
                           int block_size, int max_blocks_per_seq, int num_blocks, float scale,
                           int causal, fa_dtype dtype, void* stream);

/*
 * fa_paged_kv_append — writes one new token per request into a paged KV cache ("Atención
 * tipo FlashAttention y atención paginada": the cache grows one token at a time and the
 * block table links logical positions to fixed-size physical blocks).
 *   k_new, v_new [R, Hkv, d] bf16: the new token's key and value for every KV head.
 *   positions [R] int32 (device): logical position of the new token in request r
 *     (its context length before the append); it goes to physical block
 *     block_table[r][pos / block_size], slot pos % block_size.
 *   k_cache, v_cache [num_blocks, Hkv, block_size, d] bf16, updated in place;
 *   block_table [R, max_blocks_per_seq] int32.
 *   d == 128, block_size == 16.  A position outside [0, max_blocks_per_seq*block_size)
 *   or a physical block outside [0, num_blocks) is not written; the kernel sets the
 *   device status word (FA_ERR_INVALID_ARG) instead.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED.
 */
fa_status fa_paged_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int* block_table, const int* positions, int R, int Hkv, int d,
                             int block_size, int max_blocks_per_seq, int num_blocks, fa_dtype dtype,
                             void* stream);

/*
 * fa_paged_decode_noalloc — fa_paged_decode for callers that cannot allocate device
 * memory.  (No counterpart on the pages: this is a deployment variant of the decode
 * step, not part of the method.)
 *
 * Who needs it: code hosted inside a framework that owns all device allocations and
 * gives its kernels no workspace, and latency-critical loops that must not call
 * cudaMalloc after start-up (it can synchronise the device and take unbounded time).
 *
 * Arguments and results are those of fa_paged_decode minus the workspace: the split-KV
 * partials go to a fixed scratch array compiled into the library, FA_NOALLOC_SCRATCH_BYTES
 * (8 MiB) on every GPU that loads the library, held until the process exits.  Calls
 * whose fa_paged_decode_workspace_size(R, Hq, d, max_blocks_per_seq, block_size) exceeds
 * that limit are rejected with FA_ERR_WORKSPACE before anything is launched.  The
 * function never calls cudaMalloc, cudaFree or any allocating library routine.
 *
 * The first call on a device (with that device current) looks up the scratch array's
 * device address and caches it; make that first call before any stream capture.  The
 * cache is per CUDA context: after the device's context is destroyed and re-created
 * (cudaDeviceReset), the next call looks the address up again, so that call too should
 * come before any capture.  Every
 * call shares the one array, which keeps the last call's contents; nothing in it has to
 * start at zero (each partial the merge reads is written earlier in the same call).
 * Calls that overlap on the GPU (different streams, or different host threads without
 * ordering between them) race on the array and give undefined results.
 */
#define FA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
fa_status fa_paged_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                  const int* block_table, const int* ctx_lens, void* o, float* lse,
                                  int R, int Hq, int Hkv, int d, int block_size, int max_blocks_per_seq,
                                  int num_blocks, float scale, fa_dtype dtype, void* stream);

/*
 * fa_device_status — synchronises the current device and returns the device status
 * word the kernels set when a bounded wait runs out (FA_ERR_DEVICE_TIMEOUT) or a
 * block-table entry is out of range (FA_ERR_INVALID_ARG); FA_OK if none.  With
 * reset != 0 the word is cleared afterwards.
 */
fa_status fa_device_status(int reset);

/*
 * fa_set_wait_limit_ns — upper bound, in nanoseconds, on every in-kernel wait
 * launched after this call (default 2e8 ns = 200 ms).  Values < 1000 are clamped to 1000.
 */
void fa_set_wait_limit_ns(uint64_t ns);

/*
 * fa_selftest_wait_timeout — launches a one-CTA kernel that waits, with the current
 * limit, on a shared-memory barrier that nothing completes, so the wait must run
 * out.  Returns FA_OK if the launch succeeded; the kernel then sets the device status
 * word to FA_ERR_DEVICE_TIMEOUT, which fa_device_status reports.  For tests of the
 * timeout path; never faults or hangs the device.
 */
fa_status fa_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FA_H_ */
