// Device helpers shared by the attention kernels: 16-bit element traits,
// cp.async / ldmatrix / mma.sync wrappers, swizzled shared-memory addressing,
// and the device status word that bounded waits report into.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa.h"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Status word codes written by kernels (same values as fa_status).
constexpr int kStatusTimeout = FA_ERR_TIMEOUT;
constexpr int kStatusBadArg = FA_ERR_INVALID_ARG;
constexpr int kStatusBounds = FA_ERR_BOUNDS;

// Default time limit of every device-side wait.
constexpr unsigned long long kWaitLimitNs = 10ull * 1000ull * 1000ull * 1000ull;

__device__ __forceinline__ void report_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Index checks of the bounds-checked build (compiled with -DFA_DEBUG_BOUNDS):
// FA_IN_BOUNDS(cond, status) is `cond`, and a false `cond` records
// FA_ERR_BOUNDS in the status word; callers skip the access it guards.  In
// the normal build it is the constant `true` and costs nothing.
#ifdef FA_DEBUG_BOUNDS
__device__ __forceinline__ bool in_bounds_checked(bool ok, int* status) {
  if (!ok) report_status(status, kStatusBounds);
  return ok;
}
#define FA_IN_BOUNDS(cond, status) (::fa::in_bounds_checked((cond), (status)))
#else
#define FA_IN_BOUNDS(cond, status) (true)
#endif

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Spin until *p == expected or limit_ns elapses; false on timeout.
__device__ __forceinline__ bool wait_eq_bounded(const int* p, int expected, unsigned long long limit_ns) {
  const unsigned long long t0 = globaltimer_ns();
  while (ld_acquire_gpu(p) != expected) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
    __nanosleep(32);
  }
  return true;
}

// ---------------------------------------------------------------------------
// 16-bit element traits
// ---------------------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<__half> {
  static constexpr bool kBf16 = false;
  __device__ static __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ static __forceinline__ float2 unpack(uint32_t v) {
    __half2 h = *reinterpret_cast<__half2*>(&v);
    return __half22float2(h);
  }
  __device__ static __forceinline__ __half from_float(float x) { return __float2half_rn(x); }
  __device__ static __forceinline__ float to_float(__half x) { return __half2float(x); }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr bool kBf16 = true;
  __device__ static __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ static __forceinline__ float2 unpack(uint32_t v) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v);
    return __bfloat1622float2(h);
  }
  __device__ static __forceinline__ __nv_bfloat16 from_float(float x) { return __float2bfloat16_rn(x); }
  __device__ static __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
};

// ---------------------------------------------------------------------------
// PTX wrappers (warp-level tensor-core path)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global->shared copy; src_bytes = 0 zero-fills.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D, fp32 accumulate.
template <typename T>
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1);

template <>
__device__ __forceinline__ void mma16816<__half>(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <>
__device__ __forceinline__ void mma16816<__nv_bfloat16>(float* d, const uint32_t* a, uint32_t b0,
                                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for a pair of arguments on the FMA pipe (packed f32x2 arithmetic):
// x = n + f with n = round(x) (adding and subtracting 1.5 * 2^23 rounds to the
// nearest integer), 2^f ~ p(f) on |f| <= 1/2 by a degree-4 polynomial fitted
// for minimum relative error (exp2_poly_fit.py: max relative error 2.9e-6 in
// float32), and 2^n applied by adding n to the exponent field.  Arguments are
// clamped to >= -125 so the result stays a normal float; callers use it only
// where no argument is -inf (a masked score must give exactly 0).
constexpr float kExp2C1 = 0.693124175f;
constexpr float kExp2C2 = 0.240240991f;
constexpr float kExp2C3 = 0.0559063703f;
constexpr float kExp2C4 = 0.00958281849f;

__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long f2_sub(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
  const float kRound = 12582912.0f;  // 1.5 * 2^23
  const unsigned long long x = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const unsigned long long rnd = f2_pack(kRound, kRound);
  const unsigned long long t = f2_add(x, rnd);      // low mantissa bits hold round(x)
  const unsigned long long f = f2_sub(x, f2_sub(t, rnd));
  unsigned long long p = f2_fma(f2_pack(kExp2C4, kExp2C4), f, f2_pack(kExp2C3, kExp2C3));
  p = f2_fma(p, f, f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_pack(1.0f, 1.0f));
  float t0, t1, p0, p1;
  f2_unpack(t, t0, t1);
  f2_unpack(p, p0, p1);
  // bits(t) = 0x4B400000 + n and 0x4B400000 << 23 == 0 (mod 2^32): bits(t) << 23 == n << 23
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Order of CTAs over (work item, head) pairs for a 1-D grid of
// n_items * n_heads blocks.  Heads go in groups of kHeadGroup; inside a group
// every head's item of one rank comes before the next rank.  A wave of CTAs
// then covers few heads (their K/V stays in L2), and with `reverse` the
// highest item index comes first, so that the items that see the most keys
// (causal masks make them uneven) start first and the last wave is light.
constexpr int kHeadGroup = 8;
__device__ __forceinline__ void group_order(int L, int n_items, int n_heads, bool reverse, int& item, int& head) {
  const int per_group = kHeadGroup * n_items;
  const int grp = L / per_group;
  const int r = L - grp * per_group;
  const int gsz = min(kHeadGroup, n_heads - grp * kHeadGroup);
  const int rank = r / gsz;
  head = grp * kHeadGroup + (r - rank * gsz);
  item = reverse ? n_items - 1 - rank : rank;
}

// Where sequence b of a batch lives.  Dense batches: every sequence has Sq
// query and Sk key rows, token row t of sequence b is b*S + t and the TMA
// batch coordinate is b.  Packed (variable-length) batches: lengths and first
// rows come from the cu_seqlens offsets, and the TMA maps cover all tokens as
// a single batch.
struct SeqView {
  int sq, sk;              // query / key rows of the sequence
  long long qtok, ktok;    // token index of its first query / key row
  int qtma, ktma, tb;      // TMA row offset of the sequence, TMA batch coordinate
};
template <class P>
__device__ __forceinline__ SeqView seq_view(const P& p, int b) {
  SeqView v;
  if (p.cu_q) {
    // offsets outside [0, total] or lengths above the stated maxima are the
    // caller's error: clamp them so every access stays inside the tensors,
    // and record FA_ERR_INVALID_ARG in the status word
    const int a0 = p.cu_q[b], a1 = p.cu_q[b + 1], c0 = p.cu_k[b], c1 = p.cu_k[b + 1];
    const int q0 = min(max(a0, 0), p.total_q), k0 = min(max(c0, 0), p.total_k);
    v.sq = min(min(max(a1, q0), p.total_q) - q0, p.Sq);
    v.sk = min(min(max(c1, k0), p.total_k) - k0, p.Sk);
    if (q0 != a0 || k0 != c0 || v.sq != a1 - a0 || v.sk != c1 - c0) report_status(p.status, kStatusBadArg);
    v.qtok = q0;
    v.ktok = k0;
    v.qtma = q0;
    v.ktma = k0;
    v.tb = 0;
  } else {
    v.sq = p.Sq;
    v.sk = p.Sk;
    v.qtok = (long long)b * p.Sq;
    v.ktok = (long long)b * p.Sk;
    v.qtma = 0;
    v.ktma = 0;
    v.tb = b;
  }
  return v;
}
// Offset of the row statistics (LSE, Delta) of (b, h): dense layout
// (B, Hq, Sq), packed layout (Hq, total_q).
template <class P>
__device__ __forceinline__ long long stat_base(const P& p, const SeqView& v, int b, int h) {
  return p.cu_q ? (long long)h * p.total_q + v.qtok : ((long long)b * p.Hq + h) * p.Sq;
}

// max(a, b, c) in one instruction (three-operand form, sm_100 and later).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// tanh(x) from the identity tanh(x) = 1 - 2 / (e^{2x} + 1); absolute error
// ~1e-7, far tighter than the hardware tanh approximation.
__device__ __forceinline__ float tanh_exp(float x) {
  float e = fast_exp2(x * (2.0f * kLog2e));
  return 1.0f - __fdividef(2.0f, e + 1.0f);
}

// ---------------------------------------------------------------------------
// Swizzled row-major tiles in shared memory: a row of D 16-bit elements is
// D/8 chunks of 16 bytes; chunk c of row r is stored at c ^ (r & 7).  Eight
// consecutive rows touching the same logical chunk land on eight distinct
// bank groups, so ldmatrix and 16-byte cp.async are conflict-free.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ uint32_t swz_offset(int row, int chunk) {
  return static_cast<uint32_t>((row * (D / 8) + (chunk ^ (row & 7))) * 16);
}

}  // namespace fa
