// Incremental decoding with a paged KV cache ("FlashAttention 实战指南"
// (mhpq.cn), section on flash_attn_with_kvcache): the new keys/values are
// appended into the cache, then the queries attend over the whole cache in
// place; the KV range of each sequence is cut into num_splits page-aligned
// splits whose partial results are merged by a log-sum-exp combine.
//
// Kernels:
//   kvcache_append_kernel  writes k_new/v_new through the block table
//   decode_split_kernel    one CTA per (split, kv-head, packed row tile, batch)
//   decode_combine_kernel  merges the splits (skipped when num_splits == 1)
//
// The decode step is bound by HBM bandwidth: every cached K/V byte of the
// attended range is read once.  The q-heads of a GQA group (and the Sq query
// rows) are packed into the 16 rows of one mma.sync tile so that each K/V tile
// is read once for the whole group.
#include <math.h>

#include <type_traits>

#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {

namespace {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = 4;
constexpr int kTok = 32;  // tokens per warp tile

template <int D>
constexpr int decode_smem_bytes() {
  // Q tile (16 rows) + per warp 2 stages of (K, V) 32-token tiles.
  return 16 * D * 2 + kDecWarps * 2 * 2 * kTok * D * 2;
}

// Capacity in tokens of one sequence's cache.
__device__ __forceinline__ int seq_capacity(const DecodeParams& p) {
  return p.paged ? p.max_pages_per_seq * p.page_size : p.max_seqlen;
}

// Element offset of token t of sequence b, kv-head g; -1 if the block table
// entry is out of range.
__device__ __forceinline__ long long cache_row(const DecodeParams& p, int b, int t, int g) {
  long long row;
  if (p.paged) {
    const int page = __ldg(p.block_table + (size_t)b * p.max_pages_per_seq + t / p.page_size);
    if (page < 0 || page >= p.capacity_pages) return -1;
    row = (long long)page * p.page_size + (t % p.page_size);
  } else {
    row = (long long)b * p.max_seqlen + t;
  }
  return (row * p.Hkv + g) * p.D;
}

template <typename T>
__global__ void kvcache_append_kernel(const DecodeParams p) {
  const int chunks = p.D / 8;
  const long long total = (long long)p.B * p.Snew * p.Hkv * chunks;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(i % chunks);
    long long r = i / chunks;
    const int g = (int)(r % p.Hkv);
    r /= p.Hkv;
    const int t = (int)(r % p.Snew);
    const int b = (int)(r / p.Snew);
    const int pos = __ldg(p.cache_seqlens + b) + t;
    if (pos < 0 || pos >= seq_capacity(p)) {
      report_status(p.status, kStatusBadArg);
      continue;
    }
    const long long dst = cache_row(p, b, pos, g);
    if (dst < 0) {
      report_status(p.status, kStatusBadArg);
      continue;
    }
    const size_t src = (((size_t)b * p.Snew + t) * p.Hkv + g) * p.D + c * 8;
    *reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.k_cache) + dst + c * 8) =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.k_new) + src);
    *reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.v_cache) + dst + c * 8) =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.v_new) + src);
  }
}

// Element d of a row of x rotated at table row `pos` (rotary position
// embedding): pairs (j, j + half), or (2j, 2j + 1) when interleaved, turn by
// the angle whose cosine and sine the tables hold; dims past 2 * half are
// copied.  Computed in float32 from the 16-bit inputs.
template <typename T>
__device__ __forceinline__ float rotate_elem(const DecodeParams& p, const T* x, int d, int pos) {
  const int half = p.rot_half;
  const float xd = Elem<T>::to_float(x[d]);
  if (d >= 2 * half) return xd;
  int j, partner;
  float sign;
  if (p.rot_inter) {
    j = d >> 1;
    partner = d ^ 1;
    sign = (d & 1) ? 1.f : -1.f;
  } else {
    j = d < half ? d : d - half;
    partner = d < half ? d + half : d - half;
    sign = d < half ? -1.f : 1.f;
  }
  const float c = __ldg(p.rot_cos + (size_t)pos * half + j), s = __ldg(p.rot_sin + (size_t)pos * half + j);
  return xd * c + sign * Elem<T>::to_float(x[partner]) * s;
}

// q row (b, i, h) rotated at position cache_seqlens[b] + i into q_rot.
template <typename T>
__global__ void rotary_q_kernel(const DecodeParams p) {
  const long long total = (long long)p.B * p.Sq * p.Hq * p.D;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int d = (int)(e % p.D);
    const long long row = e / p.D;  // (b, i, h)
    const int i = (int)((row / p.Hq) % p.Sq);
    const int b = (int)(row / ((long long)p.Hq * p.Sq));
    const T* x = reinterpret_cast<const T*>(p.q) + row * p.D;
    int pos = __ldg(p.cache_seqlens + b) + i;
    if (pos < 0 || pos >= p.rot_len) {
      report_status(p.status, kStatusBadArg);
      pos = min(max(pos, 0), p.rot_len - 1);
    }
    reinterpret_cast<T*>(p.q_rot)[e] = Elem<T>::from_float(rotate_elem<T>(p, x, d, pos));
  }
}

// kvcache_append_kernel with k_new rotated at its position on the way in.
template <typename T>
__global__ void kvcache_append_rotary_kernel(const DecodeParams p) {
  const long long total = (long long)p.B * p.Snew * p.Hkv * p.D;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int d = (int)(e % p.D);
    long long r = e / p.D;
    const int g = (int)(r % p.Hkv);
    r /= p.Hkv;
    const int t = (int)(r % p.Snew);
    const int b = (int)(r / p.Snew);
    const int pos = __ldg(p.cache_seqlens + b) + t;
    if (pos < 0 || pos >= seq_capacity(p) || pos >= p.rot_len) {
      report_status(p.status, kStatusBadArg);
      continue;
    }
    const long long dst = cache_row(p, b, pos, g);
    if (dst < 0) {
      report_status(p.status, kStatusBadArg);
      continue;
    }
    const size_t src = (((size_t)b * p.Snew + t) * p.Hkv + g) * p.D;
    reinterpret_cast<T*>(p.k_cache)[dst + d] =
        Elem<T>::from_float(rotate_elem<T>(p, reinterpret_cast<const T*>(p.k_new) + src, d, pos));
    reinterpret_cast<T*>(p.v_cache)[dst + d] = reinterpret_cast<const T*>(p.v_new)[src + d];
  }
}

template <typename T, int D, bool kCap>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecodeParams p) {
  constexpr int CH = D / 8;
  constexpr int KSTEPS = D / 16;
  constexpr int NT_S = kTok / 8;
  constexpr int NT_O = D / 8;
  constexpr int TILE = kTok * D * 2;          // bytes of one K or V tile
  constexpr int WARP_BYTES = 2 * 2 * TILE;    // 2 stages x (K, V)

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* sW = smem + 16 * D * 2 + warp * WARP_BYTES;

  const int split = blockIdx.x;
  const int nrt = (p.Sq * p.G + 15) / 16;
  const int g = blockIdx.y / nrt;
  const int rt = blockIdx.y % nrt;
  const int b = blockIdx.z;
  const int rows = p.Sq * p.G;

  int L = __ldg(p.cache_seqlens + b) + p.Snew;
  if (L > seq_capacity(p) || L < 0) {
    if (tid == 0) report_status(p.status, kStatusBadArg);
    L = 0;
  }
  // Page-aligned split of [0, L).
  const int P = (L + p.page_size - 1) / p.page_size;
  const int u0 = (int)(((long long)split * P + p.num_splits - 1) / p.num_splits);
  const int u1 = (int)(((long long)(split + 1) * P + p.num_splits - 1) / p.num_splits);
  const int t0 = min(L, u0 * p.page_size);
  const int t1 = min(L, u1 * p.page_size);
  const int n_tt = (t1 - t0 + kTok - 1) / kTok;

  // ---- Q tile: packed row r = sq * G + gi  ->  query sq, q-head g*G + gi
  for (int i = tid; i < 16 * CH; i += kDecThreads) {
    const int r = i / CH, c = i % CH;
    const int pr = rt * 16 + r;
    const bool ok = pr < rows;
    const int sq = ok ? pr / p.G : 0;
    const int h = g * p.G + (ok ? pr % p.G : 0);
    const T* src = reinterpret_cast<const T*>(p.q) + (((size_t)b * p.Sq + sq) * p.Hq + h) * D + c * 8;
    cp_async_16(smem_u32(sQ) + swz_offset<D>(r, c), src, ok ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  uint32_t qf[KSTEPS][4];
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk)
    ldmatrix_x4(smem_u32(sQ) + swz_offset<D>(lane & 15, kk * 2 + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2],
                qf[kk][3]);

  const T* Kc = reinterpret_cast<const T*>(p.k_cache);
  const T* Vc = reinterpret_cast<const T*>(p.v_cache);
  const uint32_t wbase = smem_u32(sW);
  auto load_tile = [&](int tt, int stage) {
    const int tb = t0 + tt * kTok;
    for (int i = lane; i < kTok * CH; i += 32) {
      const int r = i / CH, c = i % CH;
      const int t = tb + r;
      long long off = -1;
      if (t < t1) {
        off = cache_row(p, b, t, g);
        if (off < 0) report_status(p.status, kStatusBadArg);
      }
      const bool ok = off >= 0;
      const uint32_t dst = wbase + stage * 2 * TILE + swz_offset<D>(r, c);
      cp_async_16(dst, Kc + (ok ? off : 0) + c * 8, ok ? 16 : 0);
      cp_async_16(dst + TILE, Vc + (ok ? off : 0) + c * 8, ok ? 16 : 0);
    }
  };

  float o_acc[NT_O][4];
#pragma unroll
  for (int i = 0; i < NT_O; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};

  // Absolute query positions of this thread's two packed rows.
  const int pr_a = rt * 16 + (lane >> 2), pr_b = pr_a + 8;
  const int qpos_a = pr_a / p.G + L - p.Sq;
  const int qpos_b = pr_b / p.G + L - p.Sq;

  int it = 0;
  if (warp < n_tt) load_tile(warp, 0);
  cp_async_commit();
  for (int tt = warp; tt < n_tt; tt += kDecWarps, ++it) {
    const int stage = it & 1;
    if (tt + kDecWarps < n_tt) {
      load_tile(tt + kDecWarps, stage ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint32_t kb = wbase + stage * 2 * TILE;
    const uint32_t vb = kb + TILE;
    const int tb = t0 + tt * kTok;

    float s[NT_S][4];
#pragma unroll
    for (int i = 0; i < NT_S; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
      for (int np = 0; np < NT_S / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        ldmatrix_x4(kb + swz_offset<D>(r, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma16816<T>(s[2 * np], qf[kk], b0, b1);
        mma16816<T>(s[2 * np + 1], qf[kk], b2, b3);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT_S; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x = kCap ? p.cap_log2 * tanh_exp(s[nt][e] * p.cap_in) : s[nt][e] * p.scale_log2;
        const int key = tb + nt * 8 + (lane & 3) * 2 + (e & 1);
        const int qp = (e < 2) ? qpos_a : qpos_b;
        const bool vis = key < t1 && (p.wl < 0 || key >= qp - p.wl) && (p.wr < 0 || key <= qp + p.wr);
        s[nt][e] = vis ? x : -INFINITY;
      }
    }
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
#pragma unroll
    for (int kk = 0; kk < kTok / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = Elem<T>::pack(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = Elem<T>::pack(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = Elem<T>::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = Elem<T>::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < NT_O / 2; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int r = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        ldmatrix_x4_trans(vb + swz_offset<D>(r, dp * 2 + (lane >> 4)), b0, b1, b2, b3);
        mma16816<T>(o_acc[2 * dp], pa, b0, b1);
        mma16816<T>(o_acc[2 * dp + 1], pa, b2, b3);
      }
    }
    __syncwarp();  // the stage is refilled by the next prefetch
  }
  cp_async_wait<0>();
  __syncwarp();

  // ---- merge the four warps' running states through shared memory
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  float* wO = reinterpret_cast<float*>(sW);            // 16 x D fp32
  float* wML = reinterpret_cast<float*>(sW + 16 * D * 4);  // m[16], l[16]
  const int ra = lane >> 2;
#pragma unroll
  for (int nt = 0; nt < NT_O; ++nt) {
    const int col = nt * 8 + (lane & 3) * 2;
    wO[ra * D + col] = o_acc[nt][0];
    wO[ra * D + col + 1] = o_acc[nt][1];
    wO[(ra + 8) * D + col] = o_acc[nt][2];
    wO[(ra + 8) * D + col + 1] = o_acc[nt][3];
  }
  if ((lane & 3) == 0) {
    wML[ra] = m_run[0];
    wML[ra + 8] = m_run[1];
    wML[16 + ra] = l_run[0];
    wML[16 + ra + 8] = l_run[1];
  }
  __syncthreads();

  // Thread -> (row, column group): 16 rows x D columns over 128 threads.
  constexpr int COLS_PER_THREAD = 16 * D / kDecThreads;  // 8 or 16
  const int r = tid / (kDecThreads / 16);
  const int c0 = (tid % (kDecThreads / 16)) * COLS_PER_THREAD;
  float mw[kDecWarps], lw[kDecWarps];
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kDecWarps; ++w) {
    const float* ml = reinterpret_cast<const float*>(smem + 16 * D * 2 + w * WARP_BYTES + 16 * D * 4);
    mw[w] = ml[r];
    lw[w] = ml[16 + r];
    M = fmaxf(M, mw[w]);
  }
  float fw[kDecWarps], lsum = 0.f;
#pragma unroll
  for (int w = 0; w < kDecWarps; ++w) {
    fw[w] = (M == -INFINITY) ? 0.f : fast_exp2(mw[w] - M);
    lsum += lw[w] * fw[w];
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  const float lse_nat = lsum > 0.f ? (M + log2f(lsum)) * kLn2 : -INFINITY;

  const int pr = rt * 16 + r;
  if (pr >= rows) return;
  const int sq = pr / p.G;
  const int h = g * p.G + pr % p.G;
  float acc[COLS_PER_THREAD];
#pragma unroll
  for (int j = 0; j < COLS_PER_THREAD; ++j) acc[j] = 0.f;
#pragma unroll
  for (int w = 0; w < kDecWarps; ++w) {
    const float* o = reinterpret_cast<const float*>(smem + 16 * D * 2 + w * WARP_BYTES) + r * D + c0;
#pragma unroll
    for (int j = 0; j < COLS_PER_THREAD; ++j) acc[j] += o[j] * fw[w];
  }
  if (p.num_splits == 1) {
    T* out = reinterpret_cast<T*>(p.out) + (((size_t)b * p.Sq + sq) * p.Hq + h) * D + c0;
#pragma unroll
    for (int j = 0; j < COLS_PER_THREAD; j += 8) {
      uint4 v;
      v.x = Elem<T>::pack(acc[j] * inv, acc[j + 1] * inv);
      v.y = Elem<T>::pack(acc[j + 2] * inv, acc[j + 3] * inv);
      v.z = Elem<T>::pack(acc[j + 4] * inv, acc[j + 5] * inv);
      v.w = Elem<T>::pack(acc[j + 6] * inv, acc[j + 7] * inv);
      *reinterpret_cast<uint4*>(out + j) = v;
    }
    if (p.lse && c0 == 0) p.lse[((size_t)b * p.Hq + h) * p.Sq + sq] = lse_nat;
  } else {
    const size_t row = (((size_t)split * p.B + b) * p.Hq + h) * p.Sq + sq;
    float* out = p.o_part + row * D + c0;
#pragma unroll
    for (int j = 0; j < COLS_PER_THREAD; j += 4)
      *reinterpret_cast<float4*>(out + j) = make_float4(acc[j] * inv, acc[j + 1] * inv, acc[j + 2] * inv, acc[j + 3] * inv);
    if (c0 == 0) p.lse_part[row] = lse_nat;
  }
}

// One 4-warp block per (b, q-head, query row): LSE = ln sum_s e^{LSE_s},
// O = sum_s e^{LSE_s - LSE} O_s.  Warp w takes splits w, w+4, ...; every
// lane loads its D/32 contiguous floats of O_s as one vector, and the loads
// do not depend on the split's weight (an empty split's weight 0 selects
// nothing), so consecutive splits' loads are in flight together; the four
// partial sums meet in shared memory.
constexpr int kCombineWarps = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kCombineWarps * 32) decode_combine_kernel(const DecodeParams p) {
  constexpr int PER_LANE = D / 32;  // 4 at head dim 128, 2 at 64
  using Vec = typename std::conditional<PER_LANE == 4, float4, float2>::type;
  __shared__ float s_acc[kCombineWarps][D];
  __shared__ float s_w[kCombineWarps], s_m[kCombineWarps];
  // launched as a programmatic dependent of the split kernel: wait until
  // that grid has completed and its partials are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t split_stride = (size_t)p.B * p.Hq * p.Sq;
  // largest split LSE (num_splits <= FA_MAX_SPLITS < the block's threads)
  float m = (int)threadIdx.x < p.num_splits ? p.lse_part[threadIdx.x * split_stride + row] : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_m[warp] = m;
  __syncthreads();
  float M = s_m[0];
#pragma unroll
  for (int w = 1; w < kCombineWarps; ++w) M = fmaxf(M, s_m[w]);
  float acc[PER_LANE];
#pragma unroll
  for (int j = 0; j < PER_LANE; ++j) acc[j] = 0.f;
  float wsum = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int sp = warp; sp < p.num_splits; sp += kCombineWarps) {
      const float ls = p.lse_part[sp * split_stride + row];
      const Vec v = *reinterpret_cast<const Vec*>(p.o_part + (sp * split_stride + row) * D + lane * PER_LANE);
      const float w = fast_exp2((ls - M) * kLog2e);  // 0 for an empty split (LSE -inf)
      const float* vf = reinterpret_cast<const float*>(&v);
      wsum += w;
#pragma unroll
      for (int j = 0; j < PER_LANE; ++j) acc[j] = w > 0.f ? fmaf(w, vf[j], acc[j]) : acc[j];
    }
  }
#pragma unroll
  for (int j = 0; j < PER_LANE; ++j) s_acc[warp][lane * PER_LANE + j] = acc[j];
  if (lane == 0) s_w[warp] = wsum;
  __syncthreads();
  if (warp != 0) return;
  float W = 0.f;
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) W += s_w[w];
#pragma unroll
  for (int j = 0; j < PER_LANE; ++j) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) a += s_acc[w][lane * PER_LANE + j];
    acc[j] = a;
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  // row = (b * Hq + h) * Sq + sq
  const int sq = (int)(row % p.Sq);
  const long long bh = row / p.Sq;
  const int h = (int)(bh % p.Hq);
  const int b = (int)(bh / p.Hq);
  T* out = reinterpret_cast<T*>(p.out) + (((size_t)b * p.Sq + sq) * p.Hq + h) * D + lane * PER_LANE;
#pragma unroll
  for (int j = 0; j < PER_LANE; j += 2) {
    const uint32_t v = Elem<T>::pack(acc[j] * inv, acc[j + 1] * inv);
    *reinterpret_cast<uint32_t*>(out + j) = v;
  }
  if (p.lse && lane == 0) p.lse[row] = W > 0.f ? M + logf(W) : -INFINITY;
}

template <typename T, int D, bool kCap>
cudaError_t launch_split(const DecodeParams& p, cudaStream_t s) {
  auto kern = decode_split_kernel<T, D, kCap>;
  constexpr int smem = decode_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int nrt = (p.Sq * p.G + 15) / 16;
  dim3 grid(p.num_splits, p.Hkv * nrt, p.B);
  trace_begin(s);
  kern<<<grid, kDecThreads, smem, s>>>(p);
  trace_end(s);
  return cudaGetLastError();
}

// Write k_new / v_new (rotated with rotary tables) into the cache.
template <typename T>
cudaError_t launch_append(const DecodeParams& p, cudaStream_t s, int* launches) {
  const int threads = 256;
  if (p.rot_cos) {
    const long long total = (long long)p.B * p.Snew * p.Hkv * p.D;
    const int blocks = (int)((total + threads - 1) / threads < 4096 ? (total + threads - 1) / threads : 4096);
    kvcache_append_rotary_kernel<T><<<blocks, threads, 0, s>>>(p);
  } else {
    const long long total = (long long)p.B * p.Snew * p.Hkv * (p.D / 8);
    const int blocks = (int)((total + threads - 1) / threads < 4096 ? (total + threads - 1) / threads : 4096);
    kvcache_append_kernel<T><<<blocks, threads, 0, s>>>(p);
  }
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

// The combine pass as a programmatic dependent launch: its blocks may be
// scheduled while the split kernel's last CTAs still run (the TMA split
// kernel signals this at its start) and wait in griddepcontrol.wait until
// that grid has completed and its partials are visible.
template <typename T>
cudaError_t launch_combine(const DecodeParams& p, cudaStream_t s, int* launches) {
  const long long rows = (long long)p.B * p.Hq * p.Sq;
  if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;  // one block per row
  static_assert(FA_MAX_SPLITS <= kCombineWarps * 32, "one thread per split for the LSE maximum");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(kCombineWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = p.D == 64 ? cudaLaunchKernelEx(&cfg, decode_combine_kernel<T, 64>, p)
                                  : cudaLaunchKernelEx(&cfg, decode_combine_kernel<T, 128>, p);
  if (e == cudaSuccess) ++*launches;
  return e;
}

template <typename T>
cudaError_t launch_decode_t(const DecodeParams& p_in, cudaStream_t s, int* launches) {
  cudaError_t e;
  DecodeParams p = p_in;
  p.fuse_append = 0;
  if (p.rot_cos) {
    // rotate q into the scratch copy the attention kernels then read
    const long long total = (long long)p.B * p.Sq * p.Hq * p.D;
    const int threads = 256;
    const int blocks = (int)((total + threads - 1) / threads < 4096 ? (total + threads - 1) / threads : 4096);
    rotary_q_kernel<T><<<blocks, threads, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
    p.q = p.q_rot;
  }
  bool appended = false;
  if (decode_tma_supported(p)) {
    // The TMA split kernel appends the new rows itself (not with rotary
    // tables: those rows are rotated by the append kernel first); the
    // combine follows as its programmatic dependent.
    if (p.Snew > 0 && p.rot_cos) {
      e = launch_append<T>(p, s, launches);
      if (e != cudaSuccess) return e;
      appended = true;
    }
    DecodeParams pf = p;
    pf.fuse_append = p.Snew > 0 && !p.rot_cos;
    e = launch_decode_split_tma(pf, Elem<T>::kBf16 ? FA_BF16 : FA_FP16, s);
    if (e == cudaSuccess) {
      ++*launches;
      return p.num_splits > 1 ? launch_combine<T>(p, s, launches) : cudaSuccess;
    }
    if (e != cudaErrorNotSupported) return e;
  }
  // pages the TMA boxes cannot follow: append, the cp.async gather kernel,
  // then the combine pass
  if (p.Snew > 0 && !appended) {
    e = launch_append<T>(p, s, launches);
    if (e != cudaSuccess) return e;
  }
  const bool cap = p.softcap > 0.f;
  if (p.D == 64)
    e = cap ? launch_split<T, 64, true>(p, s) : launch_split<T, 64, false>(p, s);
  else
    e = cap ? launch_split<T, 128, true>(p, s) : launch_split<T, 128, false>(p, s);
  if (e != cudaSuccess) return e;
  ++*launches;
  return p.num_splits > 1 ? launch_combine<T>(p, s, launches) : cudaSuccess;
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, fa_dtype dt, cudaStream_t s, int* launches) {
  return dt == FA_BF16 ? launch_decode_t<__nv_bfloat16>(p, s, launches) : launch_decode_t<__half>(p, s, launches);
}

}  // namespace fa
