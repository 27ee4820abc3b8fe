// Backward attention by recomputation ("FlashAttention 实战指南" (mhpq.cn),
// the three techniques: the backward pass does not keep the attention matrix,
// it recomputes it from the saved row log-sum-exp when it is needed; and the
// `deterministic` parameter, reproducible gradients at some cost).
//
//   bwd_preprocess_kernel  Delta = rowsum(dO * O); zero the fp32 dQ accumulator
//                          and the ordering counters
//   bwd_main_kernel        one CTA per (64-key block, kv-head, batch): for every
//                          q-head of the GQA group and every query block that
//                          can see these keys, recompute S^T = K Q^T and
//                          P^T = exp(S^T - LSE), then
//                            dV += P^T dO ; dP^T = V dO^T ;
//                            dS^T = P^T (dP^T - Delta) [* (1 - tanh^2)] ;
//                            dK += dS^T Q ; dQ += dS K  (fp32, atomic or ordered)
//   bwd_convert_kernel     dQ = scale * dQaccum rounded to 16 bits
//
// Warp-level tensor-core path (mma.sync m16n8k16).  Each of the 4 warps owns
// 16 keys of the block, so P^T and dS^T come out of the accumulators already in
// the A-operand layout of the dV and dK products.
#include <math.h>

#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {

namespace {

constexpr int kKB = 64;   // keys per CTA
constexpr int kQB = 64;   // query rows per iteration
constexpr int kBwdThreads = 128;

// Delta_i = sum_d dO_id O_id for every (b, i, h) row, the fp32 dQ
// accumulator zeroed, and (deterministic mode) the ordering counters reset.
// A row is D/8 lanes with 16-byte loads; a warp takes 32/(D/8) rows per step
// and keeps kPreSteps steps of loads in flight (the kernel is HBM-bound).
constexpr int kPreSteps = 4;

// Element offset of row r = (token, head) of a (B, S, H, D) tensor with
// strides st (batch, token, head); packed batches have one batch of total_q
// tokens.
// Row counts stay below 2^31 (checked on the host): 32-bit division.
__device__ __forceinline__ long long row_offset(const BwdParams& p, const long long st[3], unsigned r) {
  const unsigned tok = r / (unsigned)p.Hq, h = r - tok * (unsigned)p.Hq;
  if (p.cu_q) return (long long)tok * st[1] + (long long)h * st[2];
  const unsigned b = tok / (unsigned)p.Sq, i = tok - b * (unsigned)p.Sq;
  return (long long)b * st[0] + (long long)i * st[1] + (long long)h * st[2];
}
template <typename T, int D, bool kPacked>
__global__ void bwd_preprocess_kernel(const BwdParams p, int n_sem) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerStep = 32 / kLanesPerRow;
  // (token, h) order; a packed batch has total_q tokens
  const long long rows = (p.cu_q ? (long long)p.total_q : (long long)p.B * p.Sq) * p.Hq;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow, l = lane % kLanesPerRow;
  const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  constexpr int kRowsPerWarp = kRowsPerStep * kPreSteps;
  for (long long base = warp0 * kRowsPerWarp; base < rows; base += nwarps * kRowsPerWarp) {
    uint4 a[kPreSteps], c[kPreSteps];
#pragma unroll
    for (int u = 0; u < kPreSteps; ++u) {
      const long long r = base + u * kRowsPerStep + sub;
      const long long off_do = r < rows ? (kPacked ? r * D : row_offset(p, p.st_do, (unsigned)r)) + l * 8 : 0;
      const long long off_o = r < rows ? (kPacked ? r * D : row_offset(p, p.st_o, (unsigned)r)) + l * 8 : 0;
      if (r < rows && FA_IN_BOUNDS(off_do >= 0 && off_do + 8 <= p.ext_do && off_o >= 0 && off_o + 8 <= p.ext_o,
                                   p.status)) {
        a[u] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.dout) + off_do));
        c[u] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.o) + off_o));
      } else {
        a[u] = c[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kPreSteps; ++u) {
      const long long r = base + u * kRowsPerStep + sub;
      const uint32_t av[4] = {a[u].x, a[u].y, a[u].z, a[u].w}, cv[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 x = Elem<T>::unpack(av[j]), y = Elem<T>::unpack(cv[j]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
#pragma unroll
      for (int o = kLanesPerRow / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (r < rows && FA_IN_BOUNDS((r + 1) * D <= p.n_accum, p.status)) {
        float4* z = reinterpret_cast<float4*>(p.dq_accum + r * D + l * 8);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (l == 0) {
          const int h = (int)(r % p.Hq);
          const long long tok = r / p.Hq;
          const long long di = p.cu_q ? (long long)h * p.total_q + tok  // (Hq, total_q)
                                      : ((long long)(tok / p.Sq) * p.Hq + h) * p.Sq + tok % p.Sq;
          if (FA_IN_BOUNDS(di >= 0 && di < p.n_stat, p.status)) p.delta[di] = acc;
        }
      }
    }
  }
  if (p.deterministic) {
    const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long nthreads = (long long)gridDim.x * blockDim.x;
    for (long long i = tid; i < n_sem; i += nthreads) p.sem[i] = 0;
    if (tid == 0) *p.work_counter = 0;
  }
}

template <int D>
constexpr int bwd_smem_bytes() {
  // K, V, 2 stages x (Q, dO), dS^T (64x64 16-bit), 2 stages x (LSE, Delta)
  return 2 * kKB * D * 2 + 2 * 2 * kQB * D * 2 + kKB * kQB * 2 + 2 * 2 * kQB * 4;
}

template <typename T, int D, bool kCap, bool kDet>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_main_kernel(const BwdParams p) {
  constexpr int CH = D / 8;
  constexpr int KSTEPS = D / 16;
  constexpr int NT_Q = kQB / 8;  // n-tiles over the 64 query columns
  constexpr int NT_O = D / 8;
  constexpr int TILE = kKB * D * 2;
  constexpr int QTILE = kQB * D * 2;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sK = smem;
  uint8_t* sV = sK + TILE;
  uint8_t* sQ = sV + TILE;              // 2 stages
  uint8_t* sdO = sQ + 2 * QTILE;        // 2 stages
  uint8_t* sdS = sdO + 2 * QTILE;       // [key][q] 64 x 64
  float* sL = reinterpret_cast<float*>(sdS + kKB * kQB * 2);  // [stage][64] LSE*log2e
  float* sDl = sL + 2 * kQB;                                    // [stage][64] Delta
  __shared__ int s_item;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nkb = (p.Sk + kKB - 1) / kKB;
  const int nqb = (p.Sq + kQB - 1) / kQB;
  int item = blockIdx.x;
  if (kDet) {
    // Dynamic work index: every item with a smaller index has already been
    // claimed by a running CTA, so the ordered waits below always progress.
    if (tid == 0) s_item = atomicAdd(p.work_counter, 1);
    __syncthreads();
    item = s_item;
  }
  const int kb = item % nkb;
  const int hkv = (item / nkb) % p.Hkv;
  const int b = item / (nkb * p.Hkv);
  const int off = p.Sk - p.Sq;
  const int k0 = kb * kKB;
  const int k1 = min(k0 + kKB, p.Sk) - 1;

  // Query rows that see at least one key of [k0, k1].
  int i_min = 0, i_max = p.Sq - 1;
  if (p.wr >= 0) i_min = max(i_min, k0 - off - p.wr);
  if (p.wl >= 0) i_max = min(i_max, k1 - off + p.wl);
  const int qb_lo = i_min / kQB;
  const int n_qb = (i_max >= i_min) ? (i_max / kQB - qb_lo + 1) : 0;
  const int n_iter = n_qb * p.G;

  const size_t qs = (size_t)p.Hq * D;
  const size_t ks = (size_t)p.Hkv * D;
  const T* Kg = reinterpret_cast<const T*>(p.k) + (size_t)b * p.Sk * ks + (size_t)hkv * D;
  const T* Vg = reinterpret_cast<const T*>(p.v) + (size_t)b * p.Sk * ks + (size_t)hkv * D;
  const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV), sQa = smem_u32(sQ), sdOa = smem_u32(sdO);
  const uint32_t sdSa = smem_u32(sdS);

  for (int i = tid; i < kKB * CH; i += kBwdThreads) {
    const int r = i / CH, c = i % CH;
    const int kr = k0 + r;
    const bool ok = kr < p.Sk;
    const size_t src = (size_t)(ok ? kr : 0) * ks + c * 8;
    cp_async_16(sKa + swz_offset<D>(r, c), Kg + src, ok ? 16 : 0);
    cp_async_16(sVa + swz_offset<D>(r, c), Vg + src, ok ? 16 : 0);
  }
  // iteration it -> (q-head in group, query block)
  auto load_q = [&](int it, int stage) {
    const int hg = it / n_qb;
    const int qb = qb_lo + it % n_qb;
    const int h = hkv * p.G + hg;
    const int q0 = qb * kQB;
    const T* Qg = reinterpret_cast<const T*>(p.q) + (size_t)b * p.Sq * qs + (size_t)h * D;
    const T* dOg = reinterpret_cast<const T*>(p.dout) + (size_t)b * p.Sq * qs + (size_t)h * D;
    for (int i = tid; i < kQB * CH; i += kBwdThreads) {
      const int r = i / CH, c = i % CH;
      const int qi = q0 + r;
      const bool ok = qi < p.Sq;
      const size_t src = (size_t)(ok ? qi : 0) * qs + c * 8;
      cp_async_16(sQa + stage * QTILE + swz_offset<D>(r, c), Qg + src, ok ? 16 : 0);
      cp_async_16(sdOa + stage * QTILE + swz_offset<D>(r, c), dOg + src, ok ? 16 : 0);
    }
    if (tid < kQB) {
      const int qi = q0 + tid;
      float l2 = INFINITY, dl = 0.f;
      if (qi < p.Sq) {
        const float l = p.lse[((size_t)b * p.Hq + h) * p.Sq + qi];
        l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;
        dl = p.delta[((size_t)b * p.Hq + h) * p.Sq + qi];
      }
      sL[stage * kQB + tid] = l2;
      sDl[stage * kQB + tid] = dl;
    }
  };
  if (n_iter > 0) load_q(0, 0);
  cp_async_commit();

  float dk[NT_O][4], dv[NT_O][4];
#pragma unroll
  for (int i = 0; i < NT_O; ++i) {
    dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
    dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  }
  const int key_a = k0 + warp * 16 + (lane >> 2);  // this thread's two key rows
  const int key_b = key_a + 8;

  for (int it = 0; it < n_iter; ++it) {
    const int stage = it & 1;
    if (it + 1 < n_iter) {
      load_q(it + 1, stage ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int hg = it / n_qb;
    const int qb = qb_lo + it % n_qb;
    const int h = hkv * p.G + hg;
    const int q0 = qb * kQB;
    const uint32_t qbase = sQa + stage * QTILE;
    const uint32_t obase = sdOa + stage * QTILE;
    const float* L2 = sL + stage * kQB;
    const float* Dl = sDl + stage * kQB;

    // ---- S^T = K Q^T and dP^T = V dO^T (16 keys x 64 queries per warp)
    float sT[NT_Q][4], dpT[NT_Q][4];
#pragma unroll
    for (int i = 0; i < NT_Q; ++i) {
      sT[i][0] = sT[i][1] = sT[i][2] = sT[i][3] = 0.f;
      dpT[i][0] = dpT[i][1] = dpT[i][2] = dpT[i][3] = 0.f;
    }
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      uint32_t ka[4], va[4];
      const int r = warp * 16 + (lane & 15);
      ldmatrix_x4(sKa + swz_offset<D>(r, kk * 2 + (lane >> 4)), ka[0], ka[1], ka[2], ka[3]);
      ldmatrix_x4(sVa + swz_offset<D>(r, kk * 2 + (lane >> 4)), va[0], va[1], va[2], va[3]);
#pragma unroll
      for (int np = 0; np < NT_Q / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        const int qr = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = kk * 2 + ((lane >> 3) & 1);
        ldmatrix_x4(qbase + swz_offset<D>(qr, ch), b0, b1, b2, b3);
        mma16816<T>(sT[2 * np], ka, b0, b1);
        mma16816<T>(sT[2 * np + 1], ka, b2, b3);
        ldmatrix_x4(obase + swz_offset<D>(qr, ch), b0, b1, b2, b3);
        mma16816<T>(dpT[2 * np], va, b0, b1);
        mma16816<T>(dpT[2 * np + 1], va, b2, b3);
      }
    }

    // ---- P^T and dS^T, element by element
    const int qpos0 = q0 + off;
    const bool full = (k1 - k0 + 1 == kKB) && (p.wl < 0 || k0 >= q0 + kQB - 1 + off - p.wl) &&
                      (p.wr < 0 || k1 <= qpos0 + p.wr) && (q0 + kQB <= p.Sq);
#pragma unroll
    for (int nt = 0; nt < NT_Q; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qc = nt * 8 + (lane & 3) * 2 + (e & 1);
        const int key = (e < 2) ? key_a : key_b;
        float x, dfac = 1.f;
        if (kCap) {
          const float t = tanh_exp(sT[nt][e] * p.cap_in);
          x = p.cap_log2 * t;
          dfac = 1.f - t * t;
        } else {
          x = sT[nt][e] * p.scale_log2;
        }
        float pr = fast_exp2(x - L2[qc]);
        if (!full) {
          const int qp = qpos0 + qc;
          const bool vis = key <= k1 && (q0 + qc) < p.Sq && (p.wl < 0 || key >= qp - p.wl) &&
                           (p.wr < 0 || key <= qp + p.wr);
          if (!vis) pr = 0.f;
        }
        sT[nt][e] = pr;
        dpT[nt][e] = pr * (dpT[nt][e] - Dl[qc]) * dfac;
      }
    }

    // ---- dV += P^T dO ; dK += dS^T Q  (A operands straight from registers)
#pragma unroll
    for (int kk = 0; kk < kQB / 16; ++kk) {
      uint32_t pa[4], sa[4];
      pa[0] = Elem<T>::pack(sT[2 * kk][0], sT[2 * kk][1]);
      pa[1] = Elem<T>::pack(sT[2 * kk][2], sT[2 * kk][3]);
      pa[2] = Elem<T>::pack(sT[2 * kk + 1][0], sT[2 * kk + 1][1]);
      pa[3] = Elem<T>::pack(sT[2 * kk + 1][2], sT[2 * kk + 1][3]);
      sa[0] = Elem<T>::pack(dpT[2 * kk][0], dpT[2 * kk][1]);
      sa[1] = Elem<T>::pack(dpT[2 * kk][2], dpT[2 * kk][3]);
      sa[2] = Elem<T>::pack(dpT[2 * kk + 1][0], dpT[2 * kk + 1][1]);
      sa[3] = Elem<T>::pack(dpT[2 * kk + 1][2], dpT[2 * kk + 1][3]);
      // dS^T (16-bit) to shared memory for the dQ product
      {
        const int kr = warp * 16 + (lane >> 2);
        *reinterpret_cast<uint32_t*>(sdS + swz_offset<64>(kr, 2 * kk) + (lane & 3) * 4) = sa[0];
        *reinterpret_cast<uint32_t*>(sdS + swz_offset<64>(kr + 8, 2 * kk) + (lane & 3) * 4) = sa[1];
        *reinterpret_cast<uint32_t*>(sdS + swz_offset<64>(kr, 2 * kk + 1) + (lane & 3) * 4) = sa[2];
        *reinterpret_cast<uint32_t*>(sdS + swz_offset<64>(kr + 8, 2 * kk + 1) + (lane & 3) * 4) = sa[3];
      }
#pragma unroll
      for (int dp = 0; dp < NT_O / 2; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int qr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int ch = dp * 2 + (lane >> 4);
        ldmatrix_x4_trans(obase + swz_offset<D>(qr, ch), b0, b1, b2, b3);
        mma16816<T>(dv[2 * dp], pa, b0, b1);
        mma16816<T>(dv[2 * dp + 1], pa, b2, b3);
        ldmatrix_x4_trans(qbase + swz_offset<D>(qr, ch), b0, b1, b2, b3);
        mma16816<T>(dk[2 * dp], sa, b0, b1);
        mma16816<T>(dk[2 * dp + 1], sa, b2, b3);
      }
    }
    __syncthreads();  // dS^T complete

    // ---- dQ(64 x D) += dS K ; warp w owns query rows w*16 .. w*16+15
    int* sem = nullptr;
    if (kDet) {
      sem = p.sem + ((size_t)b * p.Hq + h) * nqb + qb;
      int kb_lo = 0;
      if (p.wl >= 0) kb_lo = max(0, q0 + off - p.wl) / kKB;
      const int expected = kb - kb_lo;
      if (tid == 0 && !wait_eq_bounded(sem, expected, kWaitLimitNs)) report_status(p.status, kStatusTimeout);
      __syncthreads();
    }
    const int qrow_a = q0 + warp * 16 + (lane >> 2);
    float* dQa = p.dq_accum + ((size_t)b * p.Sq + qrow_a) * qs + (size_t)h * D;
    float* dQb = dQa + 8 * qs;
#pragma unroll
    for (int half = 0; half < D / 64; ++half) {
      float dq[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < kKB / 16; ++kk) {
        uint32_t a[4];
        const int m = lane >> 3;
        ldmatrix_x4_trans(sdSa + swz_offset<64>(kk * 16 + (lane & 7) + ((m >> 1) << 3), warp * 2 + (m & 1)), a[0],
                          a[1], a[2], a[3]);
#pragma unroll
        for (int dp = 0; dp < 4; ++dp) {
          uint32_t b0, b1, b2, b3;
          const int kr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          ldmatrix_x4_trans(sKa + swz_offset<D>(kr, half * 8 + dp * 2 + (lane >> 4)), b0, b1, b2, b3);
          mma16816<T>(dq[2 * dp], a, b0, b1);
          mma16816<T>(dq[2 * dp + 1], a, b2, b3);
        }
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int col = half * 64 + nt * 8 + (lane & 3) * 2;
        if (qrow_a < p.Sq) atomicAdd(reinterpret_cast<float2*>(dQa + col), make_float2(dq[nt][0], dq[nt][1]));
        if (qrow_a + 8 < p.Sq) atomicAdd(reinterpret_cast<float2*>(dQb + col), make_float2(dq[nt][2], dq[nt][3]));
      }
    }
    if (kDet) {
      __threadfence();
      __syncthreads();
      if (tid == 0) atomicAdd(sem, 1);
    }
    __syncthreads();  // sdS and this stage are reused next iteration
  }
  cp_async_wait<0>();

  // ---- dK (scaled) and dV for this key block
  T* dKg = reinterpret_cast<T*>(p.dk) + (size_t)b * p.Sk * ks + (size_t)hkv * D;
  T* dVg = reinterpret_cast<T*>(p.dv) + (size_t)b * p.Sk * ks + (size_t)hkv * D;
#pragma unroll
  for (int nt = 0; nt < NT_O; ++nt) {
    const int col = nt * 8 + (lane & 3) * 2;
    if (key_a <= k1) {
      *reinterpret_cast<uint32_t*>(dKg + (size_t)key_a * ks + col) = Elem<T>::pack(dk[nt][0] * p.scale, dk[nt][1] * p.scale);
      *reinterpret_cast<uint32_t*>(dVg + (size_t)key_a * ks + col) = Elem<T>::pack(dv[nt][0], dv[nt][1]);
    }
    if (key_b <= k1) {
      *reinterpret_cast<uint32_t*>(dKg + (size_t)key_b * ks + col) = Elem<T>::pack(dk[nt][2] * p.scale, dk[nt][3] * p.scale);
      *reinterpret_cast<uint32_t*>(dVg + (size_t)key_b * ks + col) = Elem<T>::pack(dv[nt][2], dv[nt][3]);
    }
  }
}

template <typename T, bool kPacked>
__global__ void bwd_convert_kernel(const BwdParams p) {
  // D/4 lanes per (token, head) row of the packed accumulator, four
  // consecutive elements per lane; a warp takes 32/(D/4) rows per step
  const unsigned rows = (unsigned)((p.cu_q ? (long long)p.total_q : (long long)p.B * p.Sq) * p.Hq);
  const int lane = threadIdx.x & 31;
  const int lanes_per_row = p.D / 4, rows_per_step = 32 / lanes_per_row;
  const int sub = lane / lanes_per_row, l = lane - sub * lanes_per_row;
  const unsigned warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, nwarps = (gridDim.x * blockDim.x) >> 5;
  T* dq = reinterpret_cast<T*>(p.dq);
  if (kPacked) {
    const long long n4 = (long long)rows * p.D / 4;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
      if (!FA_IN_BOUNDS(4 * i + 4 <= p.n_accum && 4 * i + 4 <= p.ext_dq, p.status)) continue;
      const float4 a = reinterpret_cast<const float4*>(p.dq_accum)[i];
      uint2 v;
      v.x = Elem<T>::pack(a.x * p.scale, a.y * p.scale);
      v.y = Elem<T>::pack(a.z * p.scale, a.w * p.scale);
      reinterpret_cast<uint2*>(dq)[i] = v;
    }
    return;
  }
  for (unsigned base = warp0 * rows_per_step; base < rows; base += nwarps * rows_per_step) {
    const unsigned r = base + sub;
    if (r >= rows) continue;
    const long long dq_off = row_offset(p, p.st_dq, r) + l * 4;
    if (!FA_IN_BOUNDS(((long long)r + 1) * p.D <= p.n_accum && dq_off >= 0 && dq_off + 4 <= p.ext_dq, p.status))
      continue;
    const float4 a = reinterpret_cast<const float4*>(p.dq_accum + (size_t)r * p.D)[l];
    uint2 v;
    v.x = Elem<T>::pack(a.x * p.scale, a.y * p.scale);
    v.y = Elem<T>::pack(a.z * p.scale, a.w * p.scale);
    *reinterpret_cast<uint2*>(dq + dq_off) = v;
  }
}

template <typename T, int D, bool kCap, bool kDet>
cudaError_t launch_main(const BwdParams& p, cudaStream_t s) {
  auto kern = bwd_main_kernel<T, D, kCap, kDet>;
  constexpr int smem = bwd_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int nkb = (p.Sk + kKB - 1) / kKB;
  const long long items = (long long)nkb * p.Hkv * p.B;
  if (items == 0) return cudaSuccess;  // no keys: dQ stays zero, dK/dV are empty
  trace_begin(s);
  kern<<<(unsigned)items, kBwdThreads, smem, s>>>(p);
  trace_end(s);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_main_d(const BwdParams& p, cudaStream_t s) {
  const bool cap = p.softcap > 0.f;
  if (p.deterministic) return cap ? launch_main<T, D, true, true>(p, s) : launch_main<T, D, false, true>(p, s);
  return cap ? launch_main<T, D, true, false>(p, s) : launch_main<T, D, false, false>(p, s);
}

template <typename T>
cudaError_t launch_bwd_t(const BwdParams& p, cudaStream_t s, int* launches) {
  const int nqb = (p.Sq + kQB - 1) / kQB;
  const int n_sem = p.B * p.Hq * nqb;
  // packed dout/out rows: plain indexing (fewer registers, full occupancy)
  if (p.D == 64)
    p.rows_packed ? bwd_preprocess_kernel<T, 64, true><<<148 * 8, 256, 0, s>>>(p, n_sem)
                  : bwd_preprocess_kernel<T, 64, false><<<148 * 8, 256, 0, s>>>(p, n_sem);
  else
    p.rows_packed ? bwd_preprocess_kernel<T, 128, true><<<148 * 8, 256, 0, s>>>(p, n_sem)
                  : bwd_preprocess_kernel<T, 128, false><<<148 * 8, 256, 0, s>>>(p, n_sem);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ++*launches;
  const bool tc = (p.kernel_choice == 0 || p.kernel_choice == 2) && bwd_tc_supported(p);
  if (p.kernel_choice == 2 && !tc) return cudaErrorNotSupported;
  if (tc)
    e = launch_bwd_main_tc(p, Elem<T>::kBf16 ? FA_BF16 : FA_FP16, s);
  else
    e = (p.D == 64) ? launch_main_d<T, 64>(p, s) : launch_main_d<T, 128>(p, s);
  if (e != cudaSuccess) return e;
  ++*launches;
  p.rows_packed ? bwd_convert_kernel<T, true><<<148 * 8, 256, 0, s>>>(p)
                : bwd_convert_kernel<T, false><<<148 * 8, 256, 0, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ++*launches;
  return cudaSuccess;
}

}  // namespace

int bwd_num_qblocks(int Sq) { return (Sq + kQB - 1) / kQB; }

cudaError_t launch_bwd(const BwdParams& p, fa_dtype dt, cudaStream_t s, int* launches) {
  return dt == FA_BF16 ? launch_bwd_t<__nv_bfloat16>(p, s, launches) : launch_bwd_t<__half>(p, s, launches);
}

}  // namespace fa
