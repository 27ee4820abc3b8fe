// Parameter blocks and launchers shared between the host layer (fa_api.cu)
// and the kernel translation units.  Host code only; no torch types.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fa.h"

namespace fa {

// Forward problem after validation: window extents already have causal folded
// in (negative = unbounded), scale already resolved.
struct FwdParams {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, Sq, Sk, Hq, Hkv, D, G;
  int wl, wr;            // effective window extents, -1 = unbounded
  float scale_log2;      // scale * log2(e)
  float softcap;         // > 0 enables the tanh cap
  float cap_in;          // scale / softcap: raw dot product -> tanh argument
  float cap_log2;        // softcap * log2(e)
  int* status;           // device status word
  // packed variable-length batch: (B+1) token offsets, else null; Sq/Sk are
  // then the longest sequence and total_q the packed query tokens
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  // element strides (batch, token, head) of q, k, v, out; the head dimension
  // is contiguous.  Packed batches have batch stride 0.
  long long st_q[3], st_k[3], st_v[3], st_o[3];
  // ALiBi: slope of (batch b, q-head h) at alibi[b * alibi_bstride + h]
  // (bstride 0: one slope per head for the whole batch); null = off
  const float* alibi;
  int alibi_bstride;
  // FP8 (E4M3) inputs: one float32 factor per (batch, kv-head) for q, k, v
  // ((B, Hkv) arrays, null = 1); out is then bf16
  const float* descale_q;
  const float* descale_k;
  const float* descale_v;
  // element extents (largest offset + 1) of out and of the LSE array; read
  // only by the bounds-checked build
  long long ext_o, n_stat;
};

struct BwdParams {
  const void* dout;
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* dq_accum;       // (B, Sq, Hq, D) fp32
  float* delta;          // (B, Hq, Sq) fp32
  int* sem;              // (B, Hq, n_qblocks) ordering counters (deterministic)
  int* work_counter;     // dynamic work index (deterministic)
  int B, Sq, Sk, Hq, Hkv, D, G;
  int wl, wr;
  float scale;
  float scale_log2;
  float softcap, cap_in, cap_log2;
  int deterministic;
  int kernel_choice;     // 0 automatic, 1 mma.sync main kernel, 2 tcgen05 main kernel
  int* status;
  // packed variable-length batch (see FwdParams); dq_accum is then
  // (total_q, Hq, D) and delta (Hq, total_q)
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  // element strides (batch, token, head) of every (B, S, H, D) tensor; the
  // workspace tensors (dq_accum, delta) are always packed
  long long st_do[3], st_q[3], st_k[3], st_v[3], st_o[3], st_dq[3], st_dk[3], st_dv[3];
  int rows_packed;       // dout, out and dq are packed (token, head) rows: plain indexing
  const float* alibi;    // ALiBi slopes as in FwdParams; null = off
  int alibi_bstride;
  // element extents (largest offset + 1) of dout, out, dq, dk, dv, of the
  // LSE / Delta arrays and of the dQ accumulator; read only by the
  // bounds-checked build
  long long ext_do, ext_o, ext_dq, ext_dk, ext_dv, n_stat, n_accum;
};

struct DecodeParams {
  const void* q;
  void* k_cache;
  void* v_cache;
  const void* k_new;
  const void* v_new;
  const int* cache_seqlens;
  const int* block_table;
  int page_size, max_pages_per_seq, capacity_pages;  // paged layout
  int max_seqlen;                                    // contiguous layout
  int paged;
  void* out;
  float* lse;
  float* o_part;   // (splits, B, Hq, Sq, D)
  float* lse_part; // (splits, B, Hq, Sq)
  int B, Sq, Snew, Hq, Hkv, D, G;
  int num_splits;
  int wl, wr;
  float scale_log2, softcap, cap_in, cap_log2;
  int* status;
  // rotary position embedding (rot_cos == null: off): float32 tables
  // (rot_len, rot_half); q is rotated into q_rot, which the attention
  // kernels then read as q, and k_new is rotated on its way into the cache
  const float* rot_cos;
  const float* rot_sin;
  int rot_half, rot_len, rot_inter;
  void* q_rot;
  // TMA split kernel only.  box_rows: cache rows per TMA box (32, or 16 / 8
  // for pages smaller than or not a multiple of 32 tokens).  fuse_append: the
  // split kernel writes k_new / v_new into the cache itself and takes the new
  // rows from k_new / v_new (no separate append kernel).
  int box_rows;
  int fuse_append;
  // element counts of q / out (B*Sq*Hq*D), of the caches and of the split
  // partial rows; read only by the bounds-checked build
  long long n_out, ext_cache, n_part;
};

// Optional timing hooks around the dominant kernel of each call (events set
// with fa_set_trace_events; no-ops when unset).
void trace_begin(cudaStream_t s);
void trace_end(cudaStream_t s);

// Launchers: return the first CUDA error (cudaSuccess on success) and add the
// number of kernels launched to *launches.
cudaError_t launch_fwd_mma(const FwdParams& p, fa_dtype dt, cudaStream_t s, int* launches);
bool fwd_tc_supported(const FwdParams& p);
cudaError_t launch_fwd_tc(const FwdParams& p, fa_dtype dt, cudaStream_t s, int* launches);
// E4M3 q, k, v (head dim 128, dense batch), bf16 out
cudaError_t launch_fwd_tc_fp8(const FwdParams& p, cudaStream_t s, int* launches);
cudaError_t launch_bwd(const BwdParams& p, fa_dtype dt, cudaStream_t s, int* launches);
bool bwd_tc_supported(const BwdParams& p);
cudaError_t launch_bwd_main_tc(const BwdParams& p, fa_dtype dt, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams& p, fa_dtype dt, cudaStream_t s, int* launches);
// Split count the kvcache calls use when the caller passes num_splits <= 0.
int kvcache_auto_splits(int B, int Sq, int Hq, int Hkv, int page_size, int paged, int max_pages_per_seq,
                        int num_pages_or_max_seqlen);
bool decode_tma_supported(const DecodeParams& p);
cudaError_t launch_decode_split_tma(const DecodeParams& p, fa_dtype dt, cudaStream_t s);

}  // namespace fa
