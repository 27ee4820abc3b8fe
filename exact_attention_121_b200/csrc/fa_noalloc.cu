// fa_fwd_kvcache_noalloc: the paged KV-cache decode of fa_fwd_kvcache for
// callers that cannot allocate device memory themselves -- for example a
// plugin running inside a host runtime that owns every device allocation, or
// a serving loop whose device-memory footprint is fixed once it has started.
// The split-KV partial results, which fa_fwd_kvcache keeps in a caller-owned
// workspace, live here in a file-scope device array of fixed size instead.
//
// Nothing in this file allocates: no cudaMalloc, no cudaFree, no allocating
// library routine.  The array is part of the library's device image, so every
// GPU that loads libfa.so holds its FA_STATIC_SCRATCH_BYTES until the process
// exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "fa.h"
#include "fa_kernels.h"

namespace {

// Split-KV partials (partial outputs, then partial LSEs) of the most recent
// call on this device.  In host code this name is only a host-side stand-in
// for the device symbol: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Atomic slots: first calls made at the same time from several host threads
// all store the same address, without a data race.
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
fa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  void* ptr = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (ptr == nullptr) {
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return FA_ERR_CUDA;
    g_scratch_addr[dev].store(ptr, std::memory_order_release);
  }
  *out = ptr;
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_fwd_kvcache_noalloc(const void* q, void* k_cache, void* v_cache, const void* k_new,
                                            const void* v_new, const int* cache_seqlens, const int* block_table,
                                            int page_size, int max_pages_per_seq, int num_pages_or_max_seqlen,
                                            void* out, float* lse, int B, int Sq, int Snew, int Hq, int Hkv, int D,
                                            fa_dtype dt, float scale, int causal, int window_left,
                                            int window_right, float softcap, int num_splits, fa_stream_t stream) {
  // Requests whose partials do not fit the fixed array are refused up front.
  if (num_splits > 0 && fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits) > (size_t)FA_STATIC_SCRATCH_BYTES)
    return FA_ERR_INVALID_ARG;
  // No split count given: the workspace call's choice, lowered to the
  // largest count whose partials fit the array (one split needs none).
  if (num_splits <= 0 && B > 0 && Sq > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0) {
    int n = fa::kvcache_auto_splits(B, Sq, Hq, Hkv, page_size, block_table != nullptr, max_pages_per_seq,
                                    num_pages_or_max_seqlen);
    while (n > 1 && fa_kvcache_workspace_size(B, Sq, Hq, D, n) > (size_t)FA_STATIC_SCRATCH_BYTES) --n;
    num_splits = n;
  }
  void* scratch = nullptr;
  if (B > 0 && Sq > 0) {
    const fa_status st = scratch_address(&scratch);
    if (st != FA_OK) return st;
  }
  // Same validation and kernels as fa_fwd_kvcache.
  return fa_fwd_kvcache(q, k_cache, v_cache, k_new, v_new, cache_seqlens, block_table, page_size,
                        max_pages_per_seq, num_pages_or_max_seqlen, out, lse, B, Sq, Snew, Hq, Hkv, D, dt, scale,
                        causal, window_left, window_right, softcap, num_splits, scratch,
                        (size_t)FA_STATIC_SCRATCH_BYTES, stream);
}
