/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library libfa.so.
 *
 * The library computes exact scaled dot-product attention
 *     O = softmax(transform(scale * Q K^T) + mask) V
 * tile by tile with an online softmax, so the Sq x Sk score matrix never
 * reaches device memory; the backward recomputes the probabilities from the
 * saved row log-sum-exp instead of storing them.  Sources: "FlashAttention
 * 实战指南" (mhpq.cn), sections "why long sequences run out of memory" (the
 * three steps of standard attention, tiling, online softmax, recomputation,
 * exact result), "advanced parameters" (causal, window_size, softcap,
 * deterministic, MQA/GQA) and "incremental decoding" (flash_attn_with_kvcache:
 * append then attend, cache_seqlens, block_table, num_splits).
 *
 * Conventions shared by every entry point
 * --------------------------------------
 * Layout.   Q, K, V, O and their gradients are dense row-major tensors in the
 *           pages' (batch, seqlen, nheads, headdim) order: element
 *           [b][s][h][d] sits at ((b*S + s)*H + h)*D + d.  Every pointer must
 *           be 16-byte aligned.  LSE is float32 (B, Hq, Sq), natural log.
 * Types.    FA_FP16 or FA_BF16 for all 16-bit tensors of one call; every
 *           accumulation is float32.
 * Heads.    Hq must be an integer multiple of Hkv (MQA/GQA); q-head h reads
 *           kv-head h / (Hq/Hkv).  D must be 64 or 128.
 * Scale.    scale <= 0 selects 1/sqrt(D).
 * Softcap.  softcap > 0 replaces each scaled score u by softcap*tanh(u/softcap)
 *           before masking; softcap <= 0 disables it.
 * Masks.    Query i sits at key position i + Sk - Sq (bottom-right
 *           alignment).  Key j is visible iff
 *               j >= i + Sk - Sq - window_left   (when window_left  >= 0)
 *               j <= i + Sk - Sq + window_right  (when window_right >= 0)
 *           bounds inclusive, a negative extent is unbounded; causal != 0 is
 *           the same as window_right = 0 and is intersected with the window.
 *           A query with no visible key gets O = 0 and LSE = -inf.
 * Memory.   The caller owns every buffer, including workspaces; the library
 *           never allocates or frees device memory and never synchronises the
 *           stream (fa_last_device_status is the one exception, by design).
 *           Every call is asynchronous on `stream` (NULL = legacy default).
 * Errors.   Argument errors are returned before anything is launched.  A
 *           launch failure returns FA_ERR_CUDA.  Waits inside kernels are
 *           bounded; one that runs out records FA_ERR_TIMEOUT in a device
 *           status word that fa_last_device_status() reads.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so that the header needs no CUDA
 * include. */
typedef struct CUstream_st* fa_stream_t;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or Hq % Hkv != 0 */
  FA_ERR_UNSUPPORTED = 2, /* valid request the library does not implement (e.g. D=96) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  FA_ERR_TIMEOUT = 4,     /* a bounded device wait ran out (device status word) */
  FA_ERR_BOUNDS = 5       /* library built with FA_DEBUG_BOUNDS only: a kernel index fell
                             outside its buffer; the access was skipped (device status word) */
} fa_status;

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(fa_status s);

/*
 * Forward attention ("FlashAttention 实战指南", minimal example with
 * flash_attn_func and the advanced parameters).
 *   q   (B, Sq, Hq, D)  16-bit, read
 *   k,v (B, Sk, Hkv, D) 16-bit, read
 *   out (B, Sq, Hq, D)  16-bit, written
 *   lse (B, Hq, Sq)     float32, written (natural-log row log-sum-exp)
 * Sq, Sk >= 1 (Sq or Sk = 0 or B = 0 is a no-op returning FA_OK).
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                 int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                 float scale, int causal, int window_left, int window_right, float softcap,
                 fa_stream_t stream);

/*
 * Bytes of workspace fa_bwd needs: the float32 dQ accumulator (B, Sq, Hq, D),
 * the row terms Delta = rowsum(dO * O) (B, Hq, Sq) and, when deterministic,
 * one int32 ordering counter per (b, q-head, 64-row query block) plus a work
 * counter.  Linear in the sequence length.  Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int Sq, int Sk, int Hq, int Hkv, int D, int deterministic);

/*
 * Backward attention by recomputation ("FlashAttention 实战指南", the three
 * techniques: the backward pass recomputes the attention matrix; and the
 * `deterministic` parameter).
 *   dout, q, out (B, Sq, Hq, D) 16-bit, read;  k, v (B, Sk, Hkv, D) read
 *   lse          (B, Hq, Sq) float32 from fa_fwd with the same arguments
 *   dq (B, Sq, Hq, D), dk, dv (B, Sk, Hkv, D) 16-bit, written (overwritten,
 *   not accumulated into).  dK/dV of a kv-head sum over its q-heads.
 *   workspace: >= fa_bwd_workspace_size(...) bytes, 256-byte aligned,
 *   contents on entry ignored.
 *   deterministic != 0: dQ contributions are added in ascending key-block
 *   order behind bounded counters, so repeated calls give bit-identical
 *   results; otherwise they are added with float32 atomics.
 */
fa_status fa_bwd(const void* dout, const void* q, const void* k, const void* v,
                 const void* out, const float* lse, void* dq, void* dk, void* dv,
                 int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                 float scale, int causal, int window_left, int window_right, float softcap,
                 int deterministic, void* workspace, size_t ws_bytes, fa_stream_t stream);

/*
 * Forward attention on a packed batch of variable-length sequences (the
 * pages' "varlen" variant).  The B sequences are concatenated along the token
 * axis:
 *   q   (total_q, Hq, D)  16-bit, read;  k, v (total_k, Hkv, D) 16-bit, read
 *   out (total_q, Hq, D)  16-bit, written
 *   lse (Hq, total_q)     float32, written
 *   cu_seqlens_q, cu_seqlens_k: (B+1) int32 device offsets, cu[0] = 0,
 *     non-decreasing, cu[B] = total; sequence b owns query tokens
 *     cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and key tokens likewise.
 *   max_seqlen_q / max_seqlen_k: upper bounds of the sequence lengths (they
 *     size the grid).
 * Each sequence is attended on its own, masks and bottom-right alignment
 * taken from its own lengths (causal: query i of a sequence with Sq_b
 * queries and Sk_b keys sees keys j <= i + Sk_b - Sq_b).  A sequence with no
 * keys gets O = 0 and LSE = -inf.  Offsets that do not satisfy the contract
 * are clamped on the device (no access leaves the tensors) and record
 * FA_ERR_INVALID_ARG in the device status word.  Runs on the tcgen05 kernel
 * only: FA_ERR_UNSUPPORTED where it is not available or the mma.sync kernel
 * was selected.  Pointers are device pointers the caller owns.
 */
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                        int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int D, fa_dtype dt,
                        float scale, int causal, int window_left, int window_right, float softcap,
                        fa_stream_t stream);

/*
 * Workspace of fa_bwd_varlen: the float32 dQ accumulator (total_q, Hq, D),
 * Delta (Hq, total_q) and, when deterministic, one ordering counter per
 * (sequence, q-head, 64-row query block of max_seqlen_q) plus a work counter.
 */
size_t fa_bwd_varlen_workspace_size(int B, int max_seqlen_q, int total_q, int Hq, int D, int deterministic);

/*
 * Backward of fa_fwd_varlen (same packed layouts; lse from fa_fwd_varlen with
 * the same arguments).  dq (total_q, Hq, D), dk, dv (total_k, Hkv, D) written.
 * workspace >= fa_bwd_varlen_workspace_size(...) bytes, 256-byte aligned.
 * max_seqlen_k >= 1.  deterministic as in fa_bwd.  tcgen05 kernel only.
 */
fa_status fa_bwd_varlen(const void* dout, const void* q, const void* k, const void* v,
                        const void* out, const float* lse, void* dq, void* dk, void* dv,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                        int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int D, fa_dtype dt,
                        float scale, int causal, int window_left, int window_right, float softcap,
                        int deterministic, void* workspace, size_t ws_bytes, fa_stream_t stream);

/*
 * fa_fwd on tensors with arbitrary layouts (the pages' qkvpacked variant is
 * the case q, k, v = views of one (B, S, 3, H, D) tensor).  Same arguments as
 * fa_fwd plus `strides`: 12 host int64 values, the element strides
 * (batch, token, head) of q, k, v and out in that order; the head dimension
 * of every tensor is contiguous.  Each stride must be a non-negative multiple
 * of 8 elements (16-byte rows for the TMA unit) and every base pointer
 * 16-byte aligned, else FA_ERR_INVALID_ARG; a layout the tensor-map encoder
 * rejects gives FA_ERR_UNSUPPORTED.  lse stays (B, Hq, Sq) packed.  tcgen05
 * kernel only.
 */
fa_status fa_fwd_strided(const void* q, const void* k, const void* v, void* out, float* lse,
                         int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                         float scale, int causal, int window_left, int window_right, float softcap,
                         const long long* strides, fa_stream_t stream);

/*
 * fa_bwd on tensors with arbitrary layouts: `strides` holds 24 host int64
 * values, (batch, token, head) element strides of dout, q, k, v, out, dq, dk,
 * dv in that order (qkvpacked: dq, dk, dv are views of one (B, S, 3, H, D)
 * gradient).  Rules as fa_fwd_strided; the workspace is fa_bwd_workspace_size
 * of the same sizes and stays packed.
 */
fa_status fa_bwd_strided(const void* dout, const void* q, const void* k, const void* v,
                         const void* out, const float* lse, void* dq, void* dk, void* dv,
                         int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                         float scale, int causal, int window_left, int window_right, float softcap,
                         int deterministic, void* workspace, size_t ws_bytes,
                         const long long* strides, fa_stream_t stream);

/*
 * fa_fwd with ALiBi ("FlashAttention 实战指南", advanced parameters:
 * alibi_slopes, a position bias that lowers the scores of distant keys).
 * Query row i of (b, h) and key j get the bias -m * |i + Sk - Sq - j| added
 * to the (soft-capped) scaled score before the mask, m = alibi_slopes[b *
 * alibi_batch_stride + h]: a device float32 array, 4-byte aligned, borrowed
 * for the call.  alibi_batch_stride is 0 (one slope per q-head for the whole
 * batch, Hq values) or >= Hq (one row of Hq slopes per batch element);
 * anything else, or a null alibi_slopes, gives FA_ERR_INVALID_ARG.  LSE
 * includes the bias.  `strides` is NULL (packed tensors) or as in
 * fa_fwd_strided.  tcgen05 kernel only.
 */
fa_status fa_fwd_alibi(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                       float scale, int causal, int window_left, int window_right, float softcap,
                       const long long* strides, const float* alibi_slopes, int alibi_batch_stride,
                       fa_stream_t stream);

/*
 * fa_bwd of fa_fwd_alibi: the same slopes, and lse from fa_fwd_alibi.  The
 * bias is a constant of the inputs, so the gradients flow as in fa_bwd with
 * P recomputed including it.  `strides` is NULL or as in fa_bwd_strided;
 * the workspace is fa_bwd_workspace_size.  tcgen05 kernel only.
 */
fa_status fa_bwd_alibi(const void* dout, const void* q, const void* k, const void* v,
                       const void* out, const float* lse, void* dq, void* dk, void* dv,
                       int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                       float scale, int causal, int window_left, int window_right, float softcap,
                       int deterministic, void* workspace, size_t ws_bytes, const long long* strides,
                       const float* alibi_slopes, int alibi_batch_stride, fa_stream_t stream);

/*
 * FP8 forward ("FlashAttention 实战指南", versions: FlashAttention-3 adds an
 * FP8 forward; an fp8 path keeps precision and lowers bandwidth).  q
 * (B, Sq, Hq, D), k and v (B, Sk, Hkv, D) hold OCP FP8 E4M3 codes, one byte
 * each, packed, 16-byte aligned.  descale_q, descale_k, descale_v are device
 * float32 (B, Hkv) arrays (a q-head uses the factor of its kv-head) or NULL
 * for 1: the inputs are code value x factor, and the call computes the
 * exact attention of those inputs as fa_fwd does (scale, causal, window,
 * softcap alike).  out (B, Sq, Hq, D) is bf16; lse (B, Hq, Sq) fp32.
 * Internally P is quantised to E4M3 for the P.V product and O is divided by
 * the sum of the quantised P, so each output row is a convex combination of
 * V rows whose weights are off by at most the E4M3 rounding of P.  Head dim
 * 64 or 128 and Sk >= 1 (FA_ERR_UNSUPPORTED otherwise); misaligned pointers
 * give FA_ERR_INVALID_ARG.  tcgen05 kernel only.
 */
fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse,
                     int B, int Sq, int Sk, int Hq, int Hkv, int D,
                     const float* descale_q, const float* descale_k, const float* descale_v,
                     float scale, int causal, int window_left, int window_right, float softcap,
                     fa_stream_t stream);

/* Largest split count fa_fwd_kvcache accepts; num_splits <= 0 picks one. */
#define FA_MAX_SPLITS 64

/*
 * Bytes of workspace fa_fwd_kvcache needs for `num_splits` KV splits: the
 * float32 partial outputs (splits, B, Hq, Sq, D) and partial LSEs
 * (splits, B, Hq, Sq), each rounded up to 256 bytes.  num_splits <= 0
 * returns the size for FA_MAX_SPLITS.  Returns 0 when one split needs no
 * workspace.
 */
size_t fa_kvcache_workspace_size(int B, int Sq, int Hq, int D, int num_splits);

/*
 * Incremental decoding with a KV cache ("FlashAttention 实战指南", section on
 * flash_attn_with_kvcache): append the new keys/values into the cache, then
 * attend in place.
 *   q (B, Sq, Hq, D) 16-bit, read.
 *   Paged (block_table != NULL): k_cache, v_cache (num_pages, page_size, Hkv,
 *     D); block_table (B, max_pages_per_seq) int32 physical page ids in
 *     [0, num_pages_or_max_seqlen); logical token t of sequence b lives in
 *     page block_table[b][t / page_size], slot t % page_size.
 *   Contiguous (block_table == NULL): k_cache, v_cache (B,
 *     num_pages_or_max_seqlen, Hkv, D); page_size still sets the split unit.
 *   k_new, v_new (B, Snew, Hkv, D) or NULL when Snew == 0; written into the
 *     cache at logical positions cache_seqlens[b] .. cache_seqlens[b]+Snew-1.
 *   cache_seqlens (B) int32 device: valid length of each sequence BEFORE the
 *     append; not modified.  Sequence b attends over cache_seqlens[b] + Snew
 *     keys, which must fit the cache (checked on the device: an overflowing
 *     sequence is skipped and FA_ERR_INVALID_ARG is recorded in the status
 *     word).
 *   out (B, Sq, Hq, D) 16-bit written; lse (B, Hq, Sq) float32 or NULL.
 *   num_splits: KV range of each sequence split into this many page-aligned
 *     parts (<= 0: chosen from B, Hkv and the capacity); partials are merged
 *     by a log-sum-exp combine.  workspace >= fa_kvcache_workspace_size(B, Sq,
 *     Hq, D, num_splits) bytes, 256-byte aligned (may be NULL when that is 0);
 *     its contents need not be initialised.
 *   Kernels: with page_size a multiple of 8 tokens (or a contiguous cache)
 *     and no rotary tables the split kernel appends k_new / v_new itself, and
 *     the combine kernel (num_splits > 1) is launched as its programmatic
 *     dependent (scheduled during its tail).  Other page sizes run separate
 *     append, split and combine kernels.
 */
fa_status fa_fwd_kvcache(const void* q, void* k_cache, void* v_cache, const void* k_new,
                         const void* v_new, const int* cache_seqlens, const int* block_table,
                         int page_size, int max_pages_per_seq, int num_pages_or_max_seqlen,
                         void* out, float* lse, int B, int Sq, int Snew, int Hq, int Hkv, int D,
                         fa_dtype dt, float scale, int causal, int window_left, int window_right,
                         float softcap, int num_splits, void* workspace, size_t ws_bytes,
                         fa_stream_t stream);

/*
 * Workspace of fa_fwd_kvcache_rotary: the rotated copy of q (B, Sq, Hq, D
 * 16-bit, rounded up to 256 bytes) followed by fa_kvcache_workspace_size of
 * the same arguments.
 */
size_t fa_kvcache_rotary_workspace_size(int B, int Sq, int Hq, int D, int num_splits);

/*
 * fa_fwd_kvcache with the rotary position embedding the pages' kvcache call
 * takes (rotary_cos / rotary_sin).  Arguments as fa_fwd_kvcache, plus:
 *   rotary_cos, rotary_sin: float32 device tables (seqlen_ro, rotary_dim/2);
 *     entry [pos][j] is the cosine / sine of pair j's angle at position pos.
 *   rotary_dim: even, 0 < rotary_dim <= D; dims past it are not rotated.
 *   rotary_interleaved: 0 rotates pairs (j, j + rotary_dim/2), 1 pairs
 *     (2j, 2j+1).
 * New key row t of sequence b and query row t sit at position
 * cache_seqlens[b] + t: the keys are rotated on their way into the cache
 * (the cache holds rotated keys), the queries into a copy at the start of
 * the workspace.  Positions outside [0, seqlen_ro) record FA_ERR_INVALID_ARG
 * in the device status word (such a key is not appended; such a query uses
 * the nearest table row).  workspace >= fa_kvcache_rotary_workspace_size(...)
 * bytes, 256-byte aligned.
 */
fa_status fa_fwd_kvcache_rotary(const void* q, void* k_cache, void* v_cache, const void* k_new,
                                const void* v_new, const int* cache_seqlens, const int* block_table,
                                int page_size, int max_pages_per_seq, int num_pages_or_max_seqlen,
                                void* out, float* lse, int B, int Sq, int Snew, int Hq, int Hkv, int D,
                                fa_dtype dt, float scale, int causal, int window_left, int window_right,
                                float softcap, const float* rotary_cos, const float* rotary_sin,
                                int rotary_dim, int seqlen_ro, int rotary_interleaved, int num_splits,
                                void* workspace, size_t ws_bytes, fa_stream_t stream);

/* Size of the fixed device scratch array behind fa_fwd_kvcache_noalloc. */
#define FA_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)

/*
 * fa_fwd_kvcache without a workspace argument, for callers that cannot
 * allocate device memory: e.g. a plugin inside a host runtime that owns all
 * device allocations, or a serving loop whose device footprint is fixed after
 * start-up.  The pages have no counterpart to this entry point; it exists for
 * those callers only.
 *   Arguments: as fa_fwd_kvcache, minus workspace and ws_bytes.  The caller
 *   still owns and passes every input and output buffer.
 *   Scratch: the split-KV partials go to one file-scope device array of
 *   FA_STATIC_SCRATCH_BYTES (8 MiB) per GPU, part of the library's device
 *   image and held until the process exits.  A call fits when
 *   fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits) <= 8 MiB:
 *   num_splits * B * Hq * Sq <= 16,256 partial rows at D=128 (32,263 at
 *   D=64); larger requests return FA_ERR_INVALID_ARG before anything is
 *   launched.
 *   With num_splits <= 0 the call takes fa_fwd_kvcache's automatic split
 *   count, lowered to the largest count whose partials fit the array.
 *   The call allocates nothing: no cudaMalloc, cudaFree or allocating library
 *   routine.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture.  Under CUDA's lazy module loading
 *   (the default) that lookup is also when the driver loads this part of the
 *   library's device image, and with it the 8 MiB array: the device's free
 *   memory drops once, at the set-up call, and never at a later call.  cudaDeviceReset unloads the
 *   library's device image and with it the array: the cached address (and
 *   that of the device status word) is then stale, so no call of this library
 *   may follow a cudaDeviceReset in the same process.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's partials (nothing in it needs to start at zero: every partial row
 *   is written before it is read).  Calls whose executions overlap on the GPU
 *   (other streams, other host threads) race on the array and must be
 *   serialised by the caller.
 */
fa_status fa_fwd_kvcache_noalloc(const void* q, void* k_cache, void* v_cache, const void* k_new,
                                 const void* v_new, const int* cache_seqlens, const int* block_table,
                                 int page_size, int max_pages_per_seq, int num_pages_or_max_seqlen,
                                 void* out, float* lse, int B, int Sq, int Snew, int Hq, int Hkv, int D,
                                 fa_dtype dt, float scale, int causal, int window_left, int window_right,
                                 float softcap, int num_splits, fa_stream_t stream);

/*
 * Waits for `stream`, then returns and clears the device status word of the
 * current device: FA_OK, FA_ERR_TIMEOUT (a bounded wait ran out) or
 * FA_ERR_INVALID_ARG (a device-side argument check failed, e.g. a cache
 * overflow).  Returns FA_ERR_CUDA if the synchronisation itself fails.
 */
fa_status fa_last_device_status(fa_stream_t stream);

/* Bit of fa_build_flags(): kernels compiled with -DFA_DEBUG_BOUNDS. */
#define FA_BUILD_DEBUG_BOUNDS 1

/*
 * How this copy of the library was compiled: FA_BUILD_DEBUG_BOUNDS is set in
 * the bounds-checked test build (libfa_debug.so), whose kernels check every
 * buffer index they compute against the buffer's extent, record
 * FA_ERR_BOUNDS in the device status word and skip the access on a miss; it
 * is clear in the library proper (libfa.so).  No arguments, no errors.
 */
int fa_build_flags(void);

/*
 * Which forward kernel fa_fwd runs: 0 = automatic, 1 = the warp-level
 * mma.sync kernel, 2 = the tensor-memory tcgen05 kernel (fa_fwd returns
 * FA_ERR_UNSUPPORTED where it does not apply).  The calls that exist on the
 * tcgen05 kernel only (strided, varlen, ALiBi) return FA_ERR_UNSUPPORTED
 * under 1 rather than run another kernel.  Process wide; meant for tests
 * and benchmarks that compare the two.
 */
void fa_set_fwd_kernel(int which);

/*
 * Which main backward kernel fa_bwd runs: 0 = automatic, 1 = the warp-level
 * mma.sync kernel, 2 = the tensor-memory tcgen05 kernel (head dim 64 and
 * 128, atomic and ordered dQ).  The tcgen05-only calls (strided, varlen,
 * ALiBi) return FA_ERR_UNSUPPORTED under 1.  Process wide; meant for tests
 * and benchmarks.
 */
void fa_set_bwd_kernel(int which);

/*
 * Diagnostic for the failure-detection path: one kernel spins (bounded, with
 * the same helper the ordered backward uses) until the int32 at device
 * address `flag` equals `expected` or `limit_ns` nanoseconds pass; on timeout
 * it records FA_ERR_TIMEOUT in the status word and returns.  Never faults or
 * hangs: the wait always ends.
 */
fa_status fa_selftest_bounded_wait(const int* flag, int expected, long long limit_ns, fa_stream_t stream);

/*
 * Timing hook: when set (non-NULL cudaEvent_t handles), every later fa_fwd,
 * fa_bwd and fa_fwd_kvcache call records `start_event` immediately before its
 * dominant kernel (the forward kernel, the main backward kernel, the split
 * decode kernel) and `stop_event` immediately after it, on the call's stream.
 * Pass NULL, NULL to switch it off.  The events stay owned by the caller.
 */
void fa_set_trace_events(void* start_event, void* stop_event);

/*
 * Diagnostic: y[i] = 2^x[i] for n device floats, computed with the FMA-pipe
 * polynomial that the forward kernel can use for a share of its softmax
 * exponentials (compile-time FA_POLY_PAIRS; off by default because it
 * measured slower).  Arguments below -125 are clamped to -125.  x and y are
 * device pointers the caller owns; returns FA_ERR_INVALID_ARG for n < 0 or a
 * null pointer with n > 0.  For tests that hold it to its error bound
 * against float64.
 */
fa_status fa_selftest_exp2_poly(const float* x, float* y, int n, fa_stream_t stream);

/* Number of kernels the last fa_* call launched (for launch accounting). */
int fa_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
