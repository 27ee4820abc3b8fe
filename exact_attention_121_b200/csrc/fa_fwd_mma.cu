// Forward attention on the warp-level tensor-core path (mma.sync m16n8k16).
//
// Tiling and online softmax as described in "FlashAttention 实战指南"
// (mhpq.cn), the three techniques: Q, K, V are cut into blocks, each block is
// brought on chip, QK^T and the softmax of that block are computed there, and
// the running row maximum / running sum are updated block by block.
//
// One CTA = 4 warps = 64 query rows of one (batch, q-head); each warp owns 16
// rows.  K/V tiles of 64 keys stream through a two-stage cp.async pipeline in
// swizzled shared memory.  Scores live in registers; P is re-packed from the
// accumulator layout straight into the A-operand layout of the P.V product.
// This kernel serves every shape fa_fwd accepts; the tcgen05 kernel replaces
// it where that one applies.
#include <math.h>

#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {

namespace {

constexpr int kBR = 64;
constexpr int kBC = 64;
constexpr int kThreads = 128;

template <int D>
constexpr int fwd_mma_smem_bytes() {
  return (kBR + 4 * kBC) * D * 2;  // Q + 2 stages of (K, V)
}

template <typename T, int D, bool kCap>
__global__ void __launch_bounds__(kThreads) fwd_mma_kernel(const FwdParams p) {
  constexpr int CH = D / 8;
  constexpr int KSTEPS = D / 16;
  constexpr int NT_S = kBC / 8;
  constexpr int NT_O = D / 8;
  constexpr int TILE_BYTES = kBC * D * 2;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kBR * D * 2;
  uint8_t* sV = sK + 2 * TILE_BYTES;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int nqb = (p.Sq + kBR - 1) / kBR;
  // Heaviest query blocks first when the key range grows with the row index.
  const int qb = (p.wr >= 0) ? (nqb - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int g = h / p.G;
  const int q0 = qb * kBR;
  const int off = p.Sk - p.Sq;

  const size_t qs = (size_t)p.Hq * D;
  const size_t ks = (size_t)p.Hkv * D;
  const T* Q = reinterpret_cast<const T*>(p.q) + (size_t)b * p.Sq * qs + (size_t)h * D;
  const T* K = reinterpret_cast<const T*>(p.k) + (size_t)b * p.Sk * ks + (size_t)g * D;
  const T* V = reinterpret_cast<const T*>(p.v) + (size_t)b * p.Sk * ks + (size_t)g * D;
  T* O = reinterpret_cast<T*>(p.o) + (size_t)b * p.Sq * qs + (size_t)h * D;

  // Key range that any row of this block can see.
  const int qlast = min(q0 + kBR, p.Sq) - 1;
  int kmin = 0, kmax = p.Sk - 1;
  if (p.wl >= 0) kmin = max(kmin, q0 + off - p.wl);
  if (p.wr >= 0) kmax = min(kmax, qlast + off + p.wr);
  const int kt_begin = kmin / kBC;
  const int n_tiles = (kmax >= kmin) ? (kmax / kBC + 1 - kt_begin) : 0;

  const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);

  // ---- Q tile (rows past Sq are zero-filled)
  for (int i = tid; i < kBR * CH; i += kThreads) {
    const int r = i / CH, c = i % CH;
    const int qi = q0 + r;
    const bool ok = qi < p.Sq;
    cp_async_16(sQa + swz_offset<D>(r, c), Q + (size_t)(ok ? qi : 0) * qs + c * 8, ok ? 16 : 0);
  }
  auto load_kv = [&](int tile, int stage) {
    const int k0 = (kt_begin + tile) * kBC;
    for (int i = tid; i < kBC * CH; i += kThreads) {
      const int r = i / CH, c = i % CH;
      const int kr = k0 + r;
      const bool ok = kr < p.Sk;
      const size_t src = (size_t)(ok ? kr : 0) * ks + c * 8;
      const uint32_t dst = swz_offset<D>(r, c) + stage * TILE_BYTES;
      cp_async_16(sKa + dst, K + src, ok ? 16 : 0);
      cp_async_16(sVa + dst, V + src, ok ? 16 : 0);
    }
  };
  if (n_tiles > 0) load_kv(0, 0);
  cp_async_commit();

  float o_acc[NT_O][4];
#pragma unroll
  for (int i = 0; i < NT_O; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  uint32_t qf[KSTEPS][4];

  const int row_a = warp * 16 + (lane >> 2);  // local rows owned by this thread
  const int qpos_a = q0 + row_a + off;         // absolute positions of those rows
  const int qpos_b = qpos_a + 8;
  const int qpos_first = q0 + off, qpos_last = qlast + off;

  for (int t = 0; t < n_tiles; ++t) {
    const int stage = t & 1;
    if (t + 1 < n_tiles) {
      load_kv(t + 1, stage ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int r = warp * 16 + (lane & 15);
        ldmatrix_x4(sQa + swz_offset<D>(r, kk * 2 + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const uint32_t kbase = sKa + stage * TILE_BYTES;
    const uint32_t vbase = sVa + stage * TILE_BYTES;
    const int k0 = (kt_begin + t) * kBC;

    // ---- S = Q K^T
    float s[NT_S][4];
#pragma unroll
    for (int i = 0; i < NT_S; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
      for (int np = 0; np < NT_S / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        ldmatrix_x4(kbase + swz_offset<D>(r, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma16816<T>(s[2 * np], qf[kk], b0, b1);
        mma16816<T>(s[2 * np + 1], qf[kk], b2, b3);
      }
    }

    // ---- score transform (scale, softcap) into the log2 domain, then mask
    const bool full = (k0 + kBC <= p.Sk) && (p.wl < 0 || k0 >= qpos_last - p.wl) &&
                      (p.wr < 0 || k0 + kBC - 1 <= qpos_first + p.wr);
#pragma unroll
    for (int nt = 0; nt < NT_S; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x;
        if (kCap) {
          x = p.cap_log2 * tanh_exp(s[nt][e] * p.cap_in);
        } else {
          x = s[nt][e] * p.scale_log2;
        }
        if (!full) {
          const int key = k0 + nt * 8 + (lane & 3) * 2 + (e & 1);
          const int qp = (e < 2) ? qpos_a : qpos_b;
          const bool vis = key < p.Sk && (p.wl < 0 || key >= qp - p.wl) && (p.wr < 0 || key <= qp + p.wr);
          if (!vis) x = -INFINITY;
        }
        s[nt][e] = x;
      }
    }

    // ---- online softmax
    float mx[2] = {m_run[0], m_run[1]};
#pragma unroll
    for (int nt = 0; nt < NT_S; ++nt) {
      mx[0] = fmaxf(mx[0], fmaxf(s[nt][0], s[nt][1]));
      mx[1] = fmaxf(mx[1], fmaxf(s[nt][2], s[nt][3]));
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float m_use[2], alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      m_use[r] = (mx[r] == -INFINITY) ? 0.f : mx[r];
      alpha[r] = fast_exp2(m_run[r] - m_use[r]);
      m_run[r] = mx[r];
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < NT_S; ++nt) {
      s[nt][0] = fast_exp2(s[nt][0] - m_use[0]);
      s[nt][1] = fast_exp2(s[nt][1] - m_use[0]);
      s[nt][2] = fast_exp2(s[nt][2] - m_use[1]);
      s[nt][3] = fast_exp2(s[nt][3] - m_use[1]);
      rs[0] += s[nt][0] + s[nt][1];
      rs[1] += s[nt][2] + s[nt][3];
    }
    l_run[0] = l_run[0] * alpha[0] + rs[0];
    l_run[1] = l_run[1] * alpha[1] + rs[1];
#pragma unroll
    for (int nt = 0; nt < NT_O; ++nt) {
      o_acc[nt][0] *= alpha[0];
      o_acc[nt][1] *= alpha[0];
      o_acc[nt][2] *= alpha[1];
      o_acc[nt][3] *= alpha[1];
    }

    // ---- O += P V
#pragma unroll
    for (int kk = 0; kk < kBC / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = Elem<T>::pack(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = Elem<T>::pack(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = Elem<T>::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = Elem<T>::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < NT_O / 2; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int r = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        ldmatrix_x4_trans(vbase + swz_offset<D>(r, dp * 2 + (lane >> 4)), b0, b1, b2, b3);
        mma16816<T>(o_acc[2 * dp], pa, b0, b1);
        mma16816<T>(o_acc[2 * dp + 1], pa, b2, b3);
      }
    }
    __syncthreads();  // stage is overwritten by the next iteration's prefetch
  }
  cp_async_wait<0>();

  // ---- epilogue: normalise, LSE, stage through shared memory, store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
  const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
  if ((lane & 3) == 0) {
    float* L = p.lse + ((size_t)b * p.Hq + h) * p.Sq;
    const int qa = q0 + row_a, qb2 = qa + 8;
    if (qa < p.Sq) L[qa] = l_run[0] > 0.f ? (m_run[0] + log2f(l_run[0])) * kLn2 : -INFINITY;
    if (qb2 < p.Sq) L[qb2] = l_run[1] > 0.f ? (m_run[1] + log2f(l_run[1])) * kLn2 : -INFINITY;
  }
  __syncthreads();  // every warp is done with sQ before it is reused for O
#pragma unroll
  for (int nt = 0; nt < NT_O; ++nt) {
    const uint32_t va = Elem<T>::pack(o_acc[nt][0] * inv0, o_acc[nt][1] * inv0);
    const uint32_t vb = Elem<T>::pack(o_acc[nt][2] * inv1, o_acc[nt][3] * inv1);
    *reinterpret_cast<uint32_t*>(sQ + swz_offset<D>(row_a, nt) + (lane & 3) * 4) = va;
    *reinterpret_cast<uint32_t*>(sQ + swz_offset<D>(row_a + 8, nt) + (lane & 3) * 4) = vb;
  }
  __syncwarp();
#pragma unroll
  for (int i = lane; i < 16 * CH; i += 32) {
    const int r = warp * 16 + i / CH, c = i % CH;
    const int qi = q0 + r;
    if (qi < p.Sq) {
      const uint4 val = *reinterpret_cast<const uint4*>(sQ + swz_offset<D>(r, c));
      *reinterpret_cast<uint4*>(O + (size_t)qi * qs + c * 8) = val;
    }
  }
}

template <typename T, int D, bool kCap>
cudaError_t launch_typed(const FwdParams& p, cudaStream_t s) {
  auto kern = fwd_mma_kernel<T, D, kCap>;
  constexpr int smem = fwd_mma_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.Sq + kBR - 1) / kBR, p.Hq, p.B);
  trace_begin(s);
  kern<<<grid, kThreads, smem, s>>>(p);
  trace_end(s);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dt(const FwdParams& p, cudaStream_t s) {
  const bool cap = p.softcap > 0.f;
  if (p.D == 64) return cap ? launch_typed<T, 64, true>(p, s) : launch_typed<T, 64, false>(p, s);
  return cap ? launch_typed<T, 128, true>(p, s) : launch_typed<T, 128, false>(p, s);
}

}  // namespace

cudaError_t launch_fwd_mma(const FwdParams& p, fa_dtype dt, cudaStream_t s, int* launches) {
  cudaError_t e = (dt == FA_BF16) ? launch_dt<__nv_bfloat16>(p, s) : launch_dt<__half>(p, s);
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace fa
