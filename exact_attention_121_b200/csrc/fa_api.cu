// Host side of the C ABI declared in include/fa.h: argument validation,
// workspace sizing and carving, the device status word, and kernel dispatch.
// Nothing here allocates, frees or synchronises (except fa_last_device_status,
// whose job is to wait and read the status word).
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "fa.h"
#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
int bwd_num_qblocks(int Sq);
}

namespace {

// Device status word: bounded waits and device-side argument checks record
// their failure here; fa_last_device_status reads and clears it.
__device__ int g_fa_status = 0;

constexpr int kMaxDevices = 64;
// Device address of the status word per device, looked up once (with that
// device current).  Atomic slots: concurrent first calls from several host
// threads store the same address.
std::atomic<int*> g_status_ptr[kMaxDevices];
int g_fwd_kernel_choice = 0;
int g_bwd_kernel_choice = 0;
// Whether the automatic choice uses the tcgen05 forward kernel.
constexpr bool kTcAuto = true;
cudaEvent_t g_trace_start = nullptr, g_trace_stop = nullptr;
thread_local int g_last_launches = 0;

int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  int* ptr = g_status_ptr[dev].load(std::memory_order_acquire);
  if (!ptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_status) != cudaSuccess) return nullptr;
    ptr = static_cast<int*>(p);
    g_status_ptr[dev].store(ptr, std::memory_order_release);
  }
  return ptr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Largest element offset + 1 of a (B, S, H, D) tensor with (batch, token,
// head) strides; 0 when it is empty.
long long extent(long long B, long long S, long long H, int D, const long long st[3]) {
  if (B <= 0 || S <= 0 || H <= 0) return 0;
  return (B - 1) * st[0] + (S - 1) * st[1] + (H - 1) * st[2] + D;
}
size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

fa_status check_common(int B, int Sq, int Hq, int Hkv, int D, fa_dtype dt, float scale, float softcap) {
  if (B < 0 || Sq < 0 || Hq <= 0 || Hkv <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_FP16 && dt != FA_BF16) return FA_ERR_INVALID_ARG;
  if (isnan(scale) || isinf(scale) || isnan(softcap) || isinf(softcap)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

void fold_window(int causal, int window_left, int window_right, int* wl, int* wr) {
  *wl = window_left < 0 ? -1 : window_left;
  *wr = window_right < 0 ? -1 : window_right;
  if (causal) *wr = 0;
}

float resolve_scale(float scale, int D) { return scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D)); }

void fill_cap(float scale, float softcap, float* cap, float* cap_in, float* cap_log2, float* scale_log2) {
  const float log2e = 1.4426950408889634f;
  *scale_log2 = scale * log2e;
  if (softcap > 0.f) {
    *cap = softcap;
    *cap_in = scale / softcap;
    *cap_log2 = softcap * log2e;
  } else {
    *cap = 0.f;
    *cap_in = 0.f;
    *cap_log2 = 0.f;
  }
}

// Waits (bounded) for *flag == expected with the same helper the ordered
// backward uses; records FA_ERR_TIMEOUT in the status word when it runs out.
__global__ void selftest_wait_kernel(const int* flag, int expected, unsigned long long limit_ns, int* status) {
  if (threadIdx.x == 0 && !fa::wait_eq_bounded(flag, expected, limit_ns)) fa::report_status(status, FA_ERR_TIMEOUT);
}

__global__ void selftest_exp2_kernel(const float* x, float* y, int n) {
  const long long i = 2 * (blockIdx.x * (long long)blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    fa::exp2_poly2(x[i], x[i + 1], y[i], y[i + 1]);
  } else if (i < n) {
    float unused;
    fa::exp2_poly2(x[i], 0.f, y[i], unused);
  }
}

}  // namespace

extern "C" fa_status fa_selftest_exp2_poly(const float* x, float* y, int n, fa_stream_t stream) {
  g_last_launches = 0;
  if (n < 0 || (n > 0 && (!x || !y))) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  const int threads = 256;
  const long long pairs = (n + 1) / 2;
  selftest_exp2_kernel<<<(unsigned)((pairs + threads - 1) / threads), threads, 0, stream>>>(x, y, n);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  g_last_launches = 1;
  return FA_OK;
}

namespace fa {
void trace_begin(cudaStream_t s) {
  if (g_trace_start) cudaEventRecord(g_trace_start, s);
}
void trace_end(cudaStream_t s) {
  if (g_trace_stop) cudaEventRecord(g_trace_stop, s);
}
}  // namespace fa

extern "C" {

void fa_set_trace_events(void* start_event, void* stop_event) {
  g_trace_start = static_cast<cudaEvent_t>(start_event);
  g_trace_stop = static_cast<cudaEvent_t>(stop_event);
}

fa_status fa_selftest_bounded_wait(const int* flag, int expected, long long limit_ns, fa_stream_t stream) {
  g_last_launches = 0;
  if (!flag || limit_ns < 0 || (reinterpret_cast<uintptr_t>(flag) & 3u)) return FA_ERR_INVALID_ARG;
  int* st = status_ptr();
  if (!st) return FA_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, stream>>>(flag, expected, static_cast<unsigned long long>(limit_ns), st);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  g_last_launches = 1;
  return FA_OK;
}


const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_BOUNDS: return "FA_ERR_BOUNDS";
  }
  return "FA_ERR_UNKNOWN";
}

void fa_set_fwd_kernel(int which) { g_fwd_kernel_choice = which; }

void fa_set_bwd_kernel(int which) { g_bwd_kernel_choice = which; }

int fa_last_launch_count(void) { return g_last_launches; }

int fa_build_flags(void) {
#ifdef FA_DEBUG_BOUNDS
  return FA_BUILD_DEBUG_BOUNDS;
#else
  return 0;
#endif
}

// (batch, token, head) element strides of a packed (B, S, H, D) tensor
static void contiguous_strides(long long st[3], int S, int H, int D) {
  st[0] = (long long)S * H * D;
  st[1] = (long long)H * D;
  st[2] = D;
}
// user strides: non-negative multiples of 8 elements (16-byte rows for TMA)
static bool strides_ok(const long long* st, int n) {
  for (int i = 0; i < n; ++i)
    if (st[i] < 0 || st[i] % 8 != 0) return false;
  return true;
}

// ALiBi slopes: null (off), else 4-byte aligned with batch stride 0 (one
// slope per head) or >= Hq (one row of Hq slopes per batch element)
static bool alibi_ok(const float* a, int bstride, int Hq) {
  if (!a) return true;
  if (reinterpret_cast<uintptr_t>(a) & 3u) return false;
  return bstride == 0 || bstride >= Hq;
}

// strides: NULL (packed tensors) or 12 values, (batch, token, head) of q, k, v, out
static fa_status fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk,
                          int Hq, int Hkv, int D, fa_dtype dt, float scale, int causal, int window_left,
                          int window_right, float softcap, const long long* strides, const float* alibi,
                          int alibi_bstride, fa_stream_t stream) {
  g_last_launches = 0;
  fa_status st = check_common(B, Sq, Hq, Hkv, D, dt, scale, softcap);
  if (st != FA_OK) return st;
  if (Sk < 0) return FA_ERR_INVALID_ARG;
  if (!alibi_ok(alibi, alibi_bstride, Hq)) return FA_ERR_INVALID_ARG;
  if (B == 0 || Sq == 0) return FA_OK;
  if (!q || !out || !lse) return FA_ERR_INVALID_ARG;
  if (Sk > 0 && (!k || !v)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  if (strides && !strides_ok(strides, 12)) return FA_ERR_INVALID_ARG;
  fa::FwdParams p{};
  p.q = q; p.k = k; p.v = v; p.o = out; p.lse = lse;
  p.B = B; p.Sq = Sq; p.Sk = Sk; p.Hq = Hq; p.Hkv = Hkv; p.D = D; p.G = Hq / Hkv;
  contiguous_strides(p.st_q, Sq, Hq, D);
  contiguous_strides(p.st_k, Sk, Hkv, D);
  contiguous_strides(p.st_v, Sk, Hkv, D);
  contiguous_strides(p.st_o, Sq, Hq, D);
  if (strides) {
    long long* dst[4] = {p.st_q, p.st_k, p.st_v, p.st_o};
    for (int t = 0; t < 4; ++t)
      for (int i = 0; i < 3; ++i) dst[t][i] = strides[3 * t + i];
  }
  fold_window(causal, window_left, window_right, &p.wl, &p.wr);
  scale = resolve_scale(scale, D);
  fill_cap(scale, softcap, &p.softcap, &p.cap_in, &p.cap_log2, &p.scale_log2);
  p.alibi = alibi;
  p.alibi_bstride = alibi_bstride;
  p.ext_o = extent(B, Sq, Hq, D, p.st_o);
  p.n_stat = (long long)B * Hq * Sq;
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  int launches = 0;
  cudaError_t e;
  // strided tensors and ALiBi run on the tcgen05 kernel only: refused when
  // the mma.sync kernel is forced
  const bool tc_only = strides || alibi;
  if (tc_only && g_fwd_kernel_choice == 1) return FA_ERR_UNSUPPORTED;
  const bool tc = (g_fwd_kernel_choice == 2) || (g_fwd_kernel_choice == 0 && kTcAuto) || tc_only;
  if (tc && fa::fwd_tc_supported(p)) {
    e = fa::launch_fwd_tc(p, dt, stream, &launches);
  } else {
    if (g_fwd_kernel_choice == 2 || tc_only) return FA_ERR_UNSUPPORTED;
    e = fa::launch_fwd_mma(p, dt, stream, &launches);
  }
  g_last_launches = launches;
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk,
                 int Hq, int Hkv, int D, fa_dtype dt, float scale, int causal, int window_left, int window_right,
                 float softcap, fa_stream_t stream) {
  return fwd_impl(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, D, dt, scale, causal, window_left, window_right, softcap,
                  nullptr, nullptr, 0, stream);
}

fa_status fa_fwd_strided(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk,
                         int Hq, int Hkv, int D, fa_dtype dt, float scale, int causal, int window_left,
                         int window_right, float softcap, const long long* strides, fa_stream_t stream) {
  if (!strides) return FA_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, D, dt, scale, causal, window_left, window_right, softcap,
                  strides, nullptr, 0, stream);
}

fa_status fa_fwd_alibi(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk,
                       int Hq, int Hkv, int D, fa_dtype dt, float scale, int causal, int window_left,
                       int window_right, float softcap, const long long* strides, const float* alibi_slopes,
                       int alibi_batch_stride, fa_stream_t stream) {
  if (!alibi_slopes) return FA_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, D, dt, scale, causal, window_left, window_right, softcap,
                  strides, alibi_slopes, alibi_batch_stride, stream);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk,
                     int Hq, int Hkv, int D, const float* descale_q, const float* descale_k,
                     const float* descale_v, float scale, int causal, int window_left, int window_right,
                     float softcap, fa_stream_t stream) {
  g_last_launches = 0;
  fa_status st = check_common(B, Sq, Hq, Hkv, D, FA_BF16, scale, softcap);
  if (st != FA_OK) return st;
  if (Sk < 0) return FA_ERR_INVALID_ARG;
  for (const float* d : {descale_q, descale_k, descale_v})
    if (reinterpret_cast<uintptr_t>(d) & 3u) return FA_ERR_INVALID_ARG;
  if (B == 0 || Sq == 0) return FA_OK;
  if (Sk == 0) return FA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  if (g_fwd_kernel_choice == 1) return FA_ERR_UNSUPPORTED;  // tcgen05 kernel only
  fa::FwdParams p{};
  p.q = q; p.k = k; p.v = v; p.o = out; p.lse = lse;
  p.B = B; p.Sq = Sq; p.Sk = Sk; p.Hq = Hq; p.Hkv = Hkv; p.D = D; p.G = Hq / Hkv;
  contiguous_strides(p.st_q, Sq, Hq, D);
  contiguous_strides(p.st_k, Sk, Hkv, D);
  contiguous_strides(p.st_v, Sk, Hkv, D);
  contiguous_strides(p.st_o, Sq, Hq, D);
  p.descale_q = descale_q; p.descale_k = descale_k; p.descale_v = descale_v;
  p.ext_o = extent(B, Sq, Hq, D, p.st_o);
  p.n_stat = (long long)B * Hq * Sq;
  fold_window(causal, window_left, window_right, &p.wl, &p.wr);
  scale = resolve_scale(scale, D);
  fill_cap(scale, softcap, &p.softcap, &p.cap_in, &p.cap_log2, &p.scale_log2);
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  if (!fa::fwd_tc_supported(p)) return FA_ERR_UNSUPPORTED;
  int launches = 0;
  const cudaError_t e = fa::launch_fwd_tc_fp8(p, stream, &launches);
  g_last_launches = launches;
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_size(int B, int Sq, int Sk, int Hq, int Hkv, int D, int deterministic) {
  if (B < 0 || Sq < 0 || Sk < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || (D != 64 && D != 128)) return 0;
  size_t n = round256((size_t)B * Sq * Hq * D * sizeof(float));   // dQ accumulator
  n += round256((size_t)B * Hq * Sq * sizeof(float));               // Delta
  if (deterministic) n += round256(((size_t)B * Hq * fa::bwd_num_qblocks(Sq) + 1) * sizeof(int));
  return n;
}

// strides: NULL (packed tensors) or 24 values, (batch, token, head) of dout,
// q, k, v, out, dq, dk, dv
static fa_status bwd_impl(const void* dout, const void* q, const void* k, const void* v, const void* out,
                          const float* lse, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int Hq, int Hkv,
                          int D, fa_dtype dt, float scale, int causal, int window_left, int window_right,
                          float softcap, int deterministic, void* workspace, size_t ws_bytes,
                          const long long* strides, const float* alibi, int alibi_bstride, fa_stream_t stream) {
  g_last_launches = 0;
  fa_status st = check_common(B, Sq, Hq, Hkv, D, dt, scale, softcap);
  if (st != FA_OK) return st;
  if (Sk < 0) return FA_ERR_INVALID_ARG;
  if (!alibi_ok(alibi, alibi_bstride, Hq)) return FA_ERR_INVALID_ARG;
  if (B == 0 || (Sq == 0 && Sk == 0)) return FA_OK;
  const void* ptrs[] = {dout, q, k, v, out, lse, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if (Sq > 0 && (!dout || !q || !out || !lse || !dq)) return FA_ERR_INVALID_ARG;
  if (Sk > 0 && (!k || !v || !dk || !dv)) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_workspace_size(B, Sq, Sk, Hq, Hkv, D, deterministic);
  if (ws_bytes < need || (need > 0 && !workspace)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  fa::BwdParams p{};
  p.dout = dout; p.q = q; p.k = k; p.v = v; p.o = out; p.lse = lse; p.dq = dq; p.dk = dk; p.dv = dv;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.dq_accum = reinterpret_cast<float*>(ws);
  ws += round256((size_t)B * Sq * Hq * D * sizeof(float));
  p.delta = reinterpret_cast<float*>(ws);
  ws += round256((size_t)B * Hq * Sq * sizeof(float));
  if (deterministic) {
    p.sem = reinterpret_cast<int*>(ws);
    p.work_counter = p.sem + (size_t)B * Hq * fa::bwd_num_qblocks(Sq);
  }
  p.B = B; p.Sq = Sq; p.Sk = Sk; p.Hq = Hq; p.Hkv = Hkv; p.D = D; p.G = Hq / Hkv;
  if (strides && !strides_ok(strides, 24)) return FA_ERR_INVALID_ARG;
  if ((long long)B * Sq * Hq >= (1LL << 31)) return FA_ERR_UNSUPPORTED;  // row index of the dQ accumulator
  {
    long long* dst[8] = {p.st_do, p.st_q, p.st_k, p.st_v, p.st_o, p.st_dq, p.st_dk, p.st_dv};
    const bool is_q[8] = {true, true, false, false, true, true, false, false};
    for (int t = 0; t < 8; ++t) {
      if (strides)
        for (int i = 0; i < 3; ++i) dst[t][i] = strides[3 * t + i];
      else
        contiguous_strides(dst[t], is_q[t] ? Sq : Sk, is_q[t] ? Hq : Hkv, D);
    }
  }
  {
    long long c[3];
    contiguous_strides(c, Sq, Hq, D);
    p.rows_packed = 1;
    for (const long long* st : {p.st_do, p.st_o, p.st_dq})
      if (st[0] != c[0] || st[1] != c[1] || st[2] != c[2]) p.rows_packed = 0;
  }
  fold_window(causal, window_left, window_right, &p.wl, &p.wr);
  scale = resolve_scale(scale, D);
  p.scale = scale;
  fill_cap(scale, softcap, &p.softcap, &p.cap_in, &p.cap_log2, &p.scale_log2);
  p.deterministic = deterministic ? 1 : 0;
  p.kernel_choice = g_bwd_kernel_choice;
  p.ext_do = extent(B, Sq, Hq, D, p.st_do);
  p.ext_o = extent(B, Sq, Hq, D, p.st_o);
  p.ext_dq = extent(B, Sq, Hq, D, p.st_dq);
  p.ext_dk = extent(B, Sk, Hkv, D, p.st_dk);
  p.ext_dv = extent(B, Sk, Hkv, D, p.st_dv);
  p.n_stat = (long long)B * Hq * Sq;
  p.n_accum = (long long)B * Sq * Hq * D;
  p.alibi = alibi;
  p.alibi_bstride = alibi_bstride;
  // strided tensors and ALiBi run on the tcgen05 kernel only
  if (strides || alibi) {
    if (g_bwd_kernel_choice == 1) return FA_ERR_UNSUPPORTED;
    p.kernel_choice = 2;
  }
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  int launches = 0;
  cudaError_t e = fa::launch_bwd(p, dt, stream, &launches);
  g_last_launches = launches;
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_bwd(const void* dout, const void* q, const void* k, const void* v, const void* out, const float* lse,
                 void* dq, void* dk, void* dv, int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                 float scale, int causal, int window_left, int window_right, float softcap, int deterministic,
                 void* workspace, size_t ws_bytes, fa_stream_t stream) {
  return bwd_impl(dout, q, k, v, out, lse, dq, dk, dv, B, Sq, Sk, Hq, Hkv, D, dt, scale, causal, window_left,
                  window_right, softcap, deterministic, workspace, ws_bytes, nullptr, nullptr, 0, stream);
}

fa_status fa_bwd_strided(const void* dout, const void* q, const void* k, const void* v, const void* out,
                         const float* lse, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int Hq, int Hkv,
                         int D, fa_dtype dt, float scale, int causal, int window_left, int window_right,
                         float softcap, int deterministic, void* workspace, size_t ws_bytes,
                         const long long* strides, fa_stream_t stream) {
  if (!strides) return FA_ERR_INVALID_ARG;
  return bwd_impl(dout, q, k, v, out, lse, dq, dk, dv, B, Sq, Sk, Hq, Hkv, D, dt, scale, causal, window_left,
                  window_right, softcap, deterministic, workspace, ws_bytes, strides, nullptr, 0, stream);
}

fa_status fa_bwd_alibi(const void* dout, const void* q, const void* k, const void* v, const void* out,
                       const float* lse, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int Hq, int Hkv, int D,
                       fa_dtype dt, float scale, int causal, int window_left, int window_right, float softcap,
                       int deterministic, void* workspace, size_t ws_bytes, const long long* strides,
                       const float* alibi_slopes, int alibi_batch_stride, fa_stream_t stream) {
  if (!alibi_slopes) return FA_ERR_INVALID_ARG;
  return bwd_impl(dout, q, k, v, out, lse, dq, dk, dv, B, Sq, Sk, Hq, Hkv, D, dt, scale, causal, window_left,
                  window_right, softcap, deterministic, workspace, ws_bytes, strides, alibi_slopes,
                  alibi_batch_stride, stream);
}

// ---------------------------------------------------------------- packed batches

static fa_status check_varlen(const int* cu_q, const int* cu_k, int B, int max_q, int max_k, int total_q,
                              int total_k) {
  if (max_q < 0 || max_k < 0 || total_q < 0 || total_k < 0) return FA_ERR_INVALID_ARG;
  if (B > 0 && (!cu_q || !cu_k)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_k) & 3u)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                        int Hq, int Hkv, int D, fa_dtype dt, float scale, int causal, int window_left,
                        int window_right, float softcap, fa_stream_t stream) {
  g_last_launches = 0;
  fa_status st = check_common(B, max_seqlen_q, Hq, Hkv, D, dt, scale, softcap);
  if (st != FA_OK) return st;
  st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k);
  if (st != FA_OK) return st;
  if (B == 0 || total_q == 0 || max_seqlen_q == 0) return FA_OK;
  if (!q || !out || !lse) return FA_ERR_INVALID_ARG;
  if (total_k > 0 && (!k || !v)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  fa::FwdParams p{};
  p.q = q; p.k = k; p.v = v; p.o = out; p.lse = lse;
  p.B = B; p.Sq = max_seqlen_q; p.Sk = max_seqlen_k; p.Hq = Hq; p.Hkv = Hkv; p.D = D; p.G = Hq / Hkv;
  p.cu_q = cu_seqlens_q; p.cu_k = cu_seqlens_k; p.total_q = total_q; p.total_k = total_k;
  // packed tensors: one batch of tokens (batch stride 0)
  for (long long* st : {p.st_q, p.st_o}) { st[0] = 0; st[1] = (long long)Hq * D; st[2] = D; }
  for (long long* st : {p.st_k, p.st_v}) { st[0] = 0; st[1] = (long long)Hkv * D; st[2] = D; }
  p.ext_o = extent(1, total_q, Hq, D, p.st_o);
  p.n_stat = (long long)Hq * total_q;
  fold_window(causal, window_left, window_right, &p.wl, &p.wr);
  scale = resolve_scale(scale, D);
  fill_cap(scale, softcap, &p.softcap, &p.cap_in, &p.cap_log2, &p.scale_log2);
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  // packed batches run on the tcgen05 kernel only
  if (g_fwd_kernel_choice == 1 || !fa::fwd_tc_supported(p)) return FA_ERR_UNSUPPORTED;
  int launches = 0;
  const cudaError_t e = fa::launch_fwd_tc(p, dt, stream, &launches);
  g_last_launches = launches;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_varlen_workspace_size(int B, int max_seqlen_q, int total_q, int Hq, int D, int deterministic) {
  if (B < 0 || max_seqlen_q < 0 || total_q < 0 || Hq <= 0 || (D != 64 && D != 128)) return 0;
  size_t n = round256((size_t)total_q * Hq * D * sizeof(float));  // dQ accumulator (total_q, Hq, D)
  n += round256((size_t)Hq * total_q * sizeof(float));              // Delta (Hq, total_q)
  if (deterministic) n += round256(((size_t)B * Hq * fa::bwd_num_qblocks(max_seqlen_q) + 1) * sizeof(int));
  return n;
}

fa_status fa_bwd_varlen(const void* dout, const void* q, const void* k, const void* v, const void* out,
                        const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                        int Hq, int Hkv, int D, fa_dtype dt, float scale, int causal, int window_left,
                        int window_right, float softcap, int deterministic, void* workspace, size_t ws_bytes,
                        fa_stream_t stream) {
  g_last_launches = 0;
  fa_status st = check_common(B, max_seqlen_q, Hq, Hkv, D, dt, scale, softcap);
  if (st != FA_OK) return st;
  st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k);
  if (st != FA_OK) return st;
  if (B == 0 || (total_q == 0 && total_k == 0)) return FA_OK;
  const void* ptrs[] = {dout, q, k, v, out, lse, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if (total_q > 0 && (!dout || !q || !out || !lse || !dq)) return FA_ERR_INVALID_ARG;
  if (total_k > 0 && (!k || !v || !dk || !dv)) return FA_ERR_INVALID_ARG;
  if ((long long)total_q * Hq >= (1LL << 31)) return FA_ERR_UNSUPPORTED;  // row index of the dQ accumulator
  const size_t need = fa_bwd_varlen_workspace_size(B, max_seqlen_q, total_q, Hq, D, deterministic);
  if (ws_bytes < need || (need > 0 && !workspace)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  fa::BwdParams p{};
  p.dout = dout; p.q = q; p.k = k; p.v = v; p.o = out; p.lse = lse; p.dq = dq; p.dk = dk; p.dv = dv;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.dq_accum = reinterpret_cast<float*>(ws);
  ws += round256((size_t)total_q * Hq * D * sizeof(float));
  p.delta = reinterpret_cast<float*>(ws);
  ws += round256((size_t)Hq * total_q * sizeof(float));
  if (deterministic) {
    p.sem = reinterpret_cast<int*>(ws);
    p.work_counter = p.sem + (size_t)B * Hq * fa::bwd_num_qblocks(max_seqlen_q);
  }
  p.B = B; p.Sq = max_seqlen_q; p.Sk = max_seqlen_k; p.Hq = Hq; p.Hkv = Hkv; p.D = D; p.G = Hq / Hkv;
  p.cu_q = cu_seqlens_q; p.cu_k = cu_seqlens_k; p.total_q = total_q; p.total_k = total_k;
  // packed tensors: one batch of tokens (batch stride 0)
  for (long long* st : {p.st_do, p.st_q, p.st_o, p.st_dq}) { st[0] = 0; st[1] = (long long)Hq * D; st[2] = D; }
  for (long long* st : {p.st_k, p.st_v, p.st_dk, p.st_dv}) { st[0] = 0; st[1] = (long long)Hkv * D; st[2] = D; }
  p.rows_packed = 1;
  p.ext_do = extent(1, total_q, Hq, D, p.st_do);
  p.ext_o = extent(1, total_q, Hq, D, p.st_o);
  p.ext_dq = extent(1, total_q, Hq, D, p.st_dq);
  p.ext_dk = extent(1, total_k, Hkv, D, p.st_dk);
  p.ext_dv = extent(1, total_k, Hkv, D, p.st_dv);
  p.n_stat = (long long)Hq * total_q;
  p.n_accum = (long long)total_q * Hq * D;
  fold_window(causal, window_left, window_right, &p.wl, &p.wr);
  scale = resolve_scale(scale, D);
  p.scale = scale;
  fill_cap(scale, softcap, &p.softcap, &p.cap_in, &p.cap_log2, &p.scale_log2);
  p.deterministic = deterministic ? 1 : 0;
  // packed batches run on the tcgen05 kernel only
  if (g_bwd_kernel_choice == 1) return FA_ERR_UNSUPPORTED;
  p.kernel_choice = 2;
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  int launches = 0;
  const cudaError_t e = fa::launch_bwd(p, dt, stream, &launches);
  g_last_launches = launches;
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"

namespace fa {
// Split count of the kvcache calls when the caller gives none: enough
// (b, kv-head, split) work items for about seven CTAs per SM (three and a
// half waves of two), never more splits than pages of the longest sequence.
// Fewer, longer splits amortise each CTA's pipeline start; more waves even
// out uneven sequence lengths.  On 32k-token paged caches (B=8, 8 kv-heads)
// this gives 17 splits, 5% faster over five length draws than the 33 that
// twice as many waves give.
int kvcache_auto_splits(int B, int Sq, int Hq, int Hkv, int page_size, int paged, int max_pages_per_seq,
                        int num_pages_or_max_seqlen) {
  if (B <= 0 || Sq <= 0 || Hkv <= 0 || Hq <= 0 || page_size <= 0) return 1;
  const long long cap_tokens = paged ? (long long)max_pages_per_seq * page_size : num_pages_or_max_seqlen;
  const long long max_units = (cap_tokens + page_size - 1) / page_size;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int nrt = (Sq * (Hq / Hkv) + 15) / 16;
  const long long units = (long long)B * Hkv * nrt;
  long long n = (7LL * sms + units - 1) / units;  // ~7 CTAs per SM
  if (n > FA_MAX_SPLITS) n = FA_MAX_SPLITS;
  if (n > max_units) n = max_units;
  return n < 1 ? 1 : (int)n;
}
}  // namespace fa

extern "C" {

size_t fa_kvcache_workspace_size(int B, int Sq, int Hq, int D, int num_splits) {
  if (B < 0 || Sq < 0 || Hq <= 0 || (D != 64 && D != 128)) return 0;
  if (num_splits <= 0 || num_splits > FA_MAX_SPLITS) num_splits = FA_MAX_SPLITS;
  if (num_splits == 1) return 0;
  const size_t rows = (size_t)num_splits * B * Hq * Sq;
  return round256(rows * D * sizeof(float)) + round256(rows * sizeof(float));
}

struct RotaryArgs {
  const float* cos;
  const float* sin;
  int dim, len, interleaved;
};

// rot: NULL, or rotary tables; their q copy takes the first
// round256(B*Sq*Hq*D*2) bytes of the workspace
static fa_status kvcache_impl(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                              const int* cache_seqlens, const int* block_table, int page_size, int max_pages_per_seq,
                              int num_pages_or_max_seqlen, void* out, float* lse, int B, int Sq, int Snew, int Hq,
                              int Hkv, int D, fa_dtype dt, float scale, int causal, int window_left,
                              int window_right, float softcap, int num_splits, void* workspace, size_t ws_bytes,
                              const RotaryArgs* rot, fa_stream_t stream) {
  g_last_launches = 0;
  fa_status st = check_common(B, Sq, Hq, Hkv, D, dt, scale, softcap);
  if (st != FA_OK) return st;
  if (Snew < 0 || page_size <= 0 || num_pages_or_max_seqlen < 0) return FA_ERR_INVALID_ARG;
  if (num_splits > FA_MAX_SPLITS) return FA_ERR_INVALID_ARG;
  if (B == 0 || Sq == 0) return FA_OK;
  if (!q || !k_cache || !v_cache || !cache_seqlens || !out) return FA_ERR_INVALID_ARG;
  if (Snew > 0 && (!k_new || !v_new)) return FA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k_cache, v_cache, k_new, v_new, out, lse};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u))
    return FA_ERR_INVALID_ARG;
  const bool paged = block_table != nullptr;
  if (paged && max_pages_per_seq <= 0) return FA_ERR_INVALID_ARG;
  fa::DecodeParams p{};
  p.q = q; p.k_cache = k_cache; p.v_cache = v_cache; p.k_new = k_new; p.v_new = v_new;
  p.cache_seqlens = cache_seqlens; p.block_table = block_table;
  p.page_size = page_size; p.paged = paged ? 1 : 0;
  p.max_pages_per_seq = paged ? max_pages_per_seq : 0;
  p.capacity_pages = paged ? num_pages_or_max_seqlen : 0;
  p.max_seqlen = paged ? 0 : num_pages_or_max_seqlen;
  p.out = out; p.lse = lse;
  p.B = B; p.Sq = Sq; p.Snew = Snew; p.Hq = Hq; p.Hkv = Hkv; p.D = D; p.G = Hq / Hkv;
  p.n_out = (long long)B * Sq * Hq * D;
  p.ext_cache = paged ? (long long)num_pages_or_max_seqlen * page_size * Hkv * D
                      : (long long)B * num_pages_or_max_seqlen * Hkv * D;
  fold_window(causal, window_left, window_right, &p.wl, &p.wr);
  scale = resolve_scale(scale, D);
  fill_cap(scale, softcap, &p.softcap, &p.cap_in, &p.cap_log2, &p.scale_log2);
  if (num_splits <= 0) num_splits = fa::kvcache_auto_splits(B, Sq, Hq, Hkv, page_size, paged, max_pages_per_seq,
                                                           num_pages_or_max_seqlen);
  p.num_splits = num_splits;
  if (rot) {
    if (!rot->cos || !rot->sin || rot->dim <= 0 || rot->dim % 2 || rot->dim > D || rot->len <= 0)
      return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(rot->cos) & 3u) || (reinterpret_cast<uintptr_t>(rot->sin) & 3u))
      return FA_ERR_INVALID_ARG;
    const size_t qbytes = round256((size_t)B * Sq * Hq * D * 2);
    if (!workspace || ws_bytes < qbytes || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return FA_ERR_INVALID_ARG;
    p.rot_cos = rot->cos; p.rot_sin = rot->sin; p.rot_half = rot->dim / 2; p.rot_len = rot->len;
    p.rot_inter = rot->interleaved ? 1 : 0;
    p.q_rot = workspace;
    workspace = static_cast<uint8_t*>(workspace) + qbytes;
    ws_bytes -= qbytes;
  }
  if (num_splits > 1) {
    const size_t rows = (size_t)num_splits * B * Hq * Sq;
    const size_t need = fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits);
    if (!workspace || ws_bytes < need) return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.o_part = reinterpret_cast<float*>(ws);
    ws += round256(rows * D * sizeof(float));
    p.lse_part = reinterpret_cast<float*>(ws);
    p.n_part = (long long)rows;
  }
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  int launches = 0;
  cudaError_t e = fa::launch_decode(p, dt, stream, &launches);
  g_last_launches = launches;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_kvcache(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                         const int* cache_seqlens, const int* block_table, int page_size, int max_pages_per_seq,
                         int num_pages_or_max_seqlen, void* out, float* lse, int B, int Sq, int Snew, int Hq,
                         int Hkv, int D, fa_dtype dt, float scale, int causal, int window_left, int window_right,
                         float softcap, int num_splits, void* workspace, size_t ws_bytes, fa_stream_t stream) {
  return kvcache_impl(q, k_cache, v_cache, k_new, v_new, cache_seqlens, block_table, page_size, max_pages_per_seq,
                      num_pages_or_max_seqlen, out, lse, B, Sq, Snew, Hq, Hkv, D, dt, scale, causal, window_left,
                      window_right, softcap, num_splits, workspace, ws_bytes, nullptr, stream);
}

size_t fa_kvcache_rotary_workspace_size(int B, int Sq, int Hq, int D, int num_splits) {
  if (B < 0 || Sq < 0 || Hq <= 0 || (D != 64 && D != 128)) return 0;
  return round256((size_t)B * Sq * Hq * D * 2) + fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits);
}

fa_status fa_fwd_kvcache_rotary(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                                const int* cache_seqlens, const int* block_table, int page_size,
                                int max_pages_per_seq, int num_pages_or_max_seqlen, void* out, float* lse, int B,
                                int Sq, int Snew, int Hq, int Hkv, int D, fa_dtype dt, float scale, int causal,
                                int window_left, int window_right, float softcap, const float* rotary_cos,
                                const float* rotary_sin, int rotary_dim, int seqlen_ro, int rotary_interleaved,
                                int num_splits, void* workspace, size_t ws_bytes, fa_stream_t stream) {
  const RotaryArgs rot{rotary_cos, rotary_sin, rotary_dim, seqlen_ro, rotary_interleaved};
  return kvcache_impl(q, k_cache, v_cache, k_new, v_new, cache_seqlens, block_table, page_size, max_pages_per_seq,
                      num_pages_or_max_seqlen, out, lse, B, Sq, Snew, Hq, Hkv, D, dt, scale, causal, window_left,
                      window_right, softcap, num_splits, workspace, ws_bytes, &rot, stream);
}

fa_status fa_last_device_status(fa_stream_t stream) {
  int* ptr = status_ptr();
  if (!ptr) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fa_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  return static_cast<fa_status>(v);
}

}  // extern "C"
