// Split-KV paged decode with a TMA-fed pipeline ("FlashAttention 实战指南"
// (mhpq.cn), section on flash_attn_with_kvcache: append, then attend over the
// cache in place, the KV range split into num_splits parts).
//
// The step is bound by HBM bandwidth, so the kernel is built around keeping
// enough bytes in flight: one producer warp looks up the block table once per
// TMA box (a 32-token tile is one box, or two / four boxes when pages hold 16
// or 8 tokens) and issues one box per 64 head-dim columns of K and V into a
// 6-stage shared-memory ring (96 KB per CTA, two CTAs per SM); three consumer
// warps each own two stages, so every warp computes on one tile while its
// next tile lands.  The q-heads of the GQA group (times the query rows) are
// packed into the 16 rows of an mma.sync tile, so each K/V byte is read from
// HBM once for the whole group.
//
// The append and the launch gap of the combine are folded in:
//   * append (fuse_append): the CTAs of the first row tile write the new
//     rows k_new / v_new into the cache, spread over the splits, and every
//     CTA whose tile covers a new row takes that row from k_new / v_new in
//     shared memory, so no CTA depends on another's cache write;
//   * combine: the partials go to the workspace; the combine kernel that
//     merges them is launched as a programmatic dependent of this kernel
//     (each CTA signals it at its start), so it is scheduled during this
//     kernel's tail and only waits for the grid to complete.
#include <math.h>

#include "fa_common.cuh"
#include "fa_kernels.h"
#include "fa_sm100.cuh"
#include "fa_tma.h"

namespace fa {

namespace {

using namespace sm100;

constexpr int kTokT = 32;        // tokens per tile (one TMA box row count)
constexpr int kConsumers = 3;
constexpr int kStages = 2 * kConsumers;  // stage s belongs to consumer warp s % kConsumers
constexpr int kThreadsD = 32 * (kConsumers + 1);
constexpr unsigned long long kDecWaitNs = kWaitLimitNs;

template <int D>
struct DecCfg {
  static constexpr int NCH = D / 64;
  static constexpr int CHUNK = kTokT * 128;          // 32 rows x 64 columns, 16-bit, swizzled
  static constexpr int KT = NCH * CHUNK;             // one K (or V) tile
  static constexpr int STAGE = 2 * KT;
  static constexpr int OFF_Q = 0;                    // 16 x D, XOR-swizzled (cp.async)
  static constexpr int OFF_ST = 16 * D * 2 > 1024 ? 16 * D * 2 : 1024;
  static constexpr int OFF_BAR = OFF_ST + kStages * STAGE;
  static constexpr int OFF_FLAG = OFF_BAR + 2 * kStages * 8;
  static constexpr int SMEM = OFF_FLAG + kStages * 4 + 1024;
};

// Byte offset of logical 16-byte chunk j of row r inside a TMA-swizzled tile
// made of 64-column chunks of `rows` rows.
template <int ROWS>
__device__ __forceinline__ uint32_t tma_sw(int r, int j) {
  return (uint32_t)((j >> 3) * ROWS * 128 + r * 128 + (((j & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ int cap_tokens(const DecodeParams& p) {
  return p.paged ? p.max_pages_per_seq * p.page_size : p.max_seqlen;
}

// Element offset of (sequence b, position pos, kv-head g) in the cache, or -1
// when the position or its page is outside the cache.
__device__ __forceinline__ long long cache_elem(const DecodeParams& p, int b, int pos, int g) {
  if (pos < 0 || pos >= cap_tokens(p)) return -1;
  long long row;
  if (p.paged) {
    const int page = __ldg(p.block_table + (size_t)b * p.max_pages_per_seq + pos / p.page_size);
    if (page < 0 || page >= p.capacity_pages) return -1;
    row = (long long)page * p.page_size + pos % p.page_size;
  } else {
    row = (long long)b * p.max_seqlen + pos;
  }
  return (row * p.Hkv + g) * p.D;
}

template <typename T, int D, bool kCap>
__global__ void __launch_bounds__(kThreadsD, 1)
    decode_tma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const DecodeParams p) {
  using C = DecCfg<D>;
  constexpr int CH = D / 8;
  constexpr int KSTEPS = D / 16;
  constexpr int NT_S = kTokT / 8;
  constexpr int NT_O = D / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto full = [&](int st) -> uint32_t { return sb + C::OFF_BAR + 8 * st; };
  auto empty = [&](int st) -> uint32_t { return sb + C::OFF_BAR + 8 * (kStages + st); };
  volatile int* flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);

  // the combine kernel (a programmatic dependent launch) may be scheduled
  // once every CTA of this grid has started; it waits for the grid to finish
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int nrt = (p.Sq * p.G + 15) / 16;
  const int g = blockIdx.y / nrt;
  const int rt = blockIdx.y % nrt;
  const int b = blockIdx.z;
  const int rows = p.Sq * p.G;

  int L = __ldg(p.cache_seqlens + b) + p.Snew;
  if (L > cap_tokens(p) || L < 0) {
    if (threadIdx.x == 0) report_status(p.status, kStatusBadArg);
    L = 0;
  }
  const int P = (L + p.page_size - 1) / p.page_size;
  const int u0 = (int)(((long long)split * P + p.num_splits - 1) / p.num_splits);
  const int u1 = (int)(((long long)(split + 1) * P + p.num_splits - 1) / p.num_splits);
  const int t0 = min(L, u0 * p.page_size);
  const int t1 = min(L, u1 * p.page_size);
  const int n_tt = (t1 - t0 + kTokT - 1) / kTokT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      volatile int never = 0;
      for (int tt = 0; tt < n_tt; ++tt) {
        const int st = tt % kStages, u = tt / kStages;
        if (tt >= kStages && !mbar_wait(empty(st), (u - 1) & 1, &never, kDecWaitNs)) {
          report_status(p.status, kStatusTimeout);
          break;
        }
        const int t = t0 + tt * kTokT;
        const uint32_t kst = sb + C::OFF_ST + st * C::STAGE;
        if (p.box_rows == kTokT) {
          // one box per tile: the tile lies inside one page
          int c2 = t, c3 = b;
          bool ok = true;
          if (p.paged) {
            const int page = __ldg(p.block_table + (size_t)b * p.max_pages_per_seq + t / p.page_size);
            ok = page >= 0 && page < p.capacity_pages;
            c2 = t % p.page_size;
            c3 = page;
          }
          flag[st] = ok ? 1 : 0;
          if (!ok) {
            report_status(p.status, kStatusBadArg);
            mbar_arrive(full(st));
            continue;
          }
          mbar_expect_tx(full(st), C::STAGE);
          for (int c = 0; c < C::NCH; ++c) {
            tma_load_4d(kst + c * C::CHUNK, &tmK, c * 64, g, c2, c3, full(st));
            tma_load_4d(kst + C::KT + c * C::CHUNK, &tmV, c * 64, g, c2, c3, full(st));
          }
          continue;
        }
        // boxes of R = 16 or 8 rows; each lies inside one page (R divides the
        // page size and t0 starts a page); boxes past the split end are not
        // loaded
        const int R = p.box_rows;
        const int nbox = min(kTokT / R, (t1 - t + R - 1) / R);
        int c2[kTokT / 8], c3[kTokT / 8];  // unrolled: registers
        bool ok = true;
#pragma unroll
        for (int x = 0; x < kTokT / 8; ++x) {
          const int tx = t + x * R;
          c2[x] = tx;
          c3[x] = b;
          if (x < nbox && p.paged) {
            const int page = __ldg(p.block_table + (size_t)b * p.max_pages_per_seq + tx / p.page_size);
            ok = ok && page >= 0 && page < p.capacity_pages;
            c2[x] = tx % p.page_size;
            c3[x] = page;
          }
        }
        flag[st] = ok ? 1 : 0;
        if (!ok) {
          report_status(p.status, kStatusBadArg);
          mbar_arrive(full(st));
          continue;
        }
        mbar_expect_tx(full(st), (uint32_t)(nbox * R * 128 * C::NCH * 2));
#pragma unroll
        for (int x = 0; x < kTokT / 8; ++x)
          if (x < nbox)
#pragma unroll
            for (int c = 0; c < C::NCH; ++c) {
              tma_load_4d(kst + c * C::CHUNK + x * R * 128, &tmK, c * 64, g, c2[x], c3[x], full(st));
              tma_load_4d(kst + C::KT + c * C::CHUNK + x * R * 128, &tmV, c * 64, g, c2[x], c3[x], full(st));
            }
      }
    }
    return;  // the consumers never wait on this warp again
  }

  // -------------------------------------------------------------- consumers
  uint8_t* sQ = smem + C::OFF_Q;
  for (int i = threadIdx.x; i < 16 * CH; i += 32 * kConsumers) {
    const int r = i / CH, c = i % CH;
    const int pr = rt * 16 + r;
    const bool okr = pr < rows;
    const int sq = okr ? pr / p.G : 0;
    const int h = g * p.G + (okr ? pr % p.G : 0);
    const long long qi = (((long long)b * p.Sq + sq) * p.Hq + h) * D + c * 8;
    const bool ld = okr && FA_IN_BOUNDS(qi >= 0 && qi + 8 <= p.n_out, p.status);
    const T* src = reinterpret_cast<const T*>(p.q) + (ld ? qi : 0);
    cp_async_16(smem_u32(sQ) + swz_offset<D>(r, c), src, ld ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  named_bar_sync(1, 32 * kConsumers);

  if (p.fuse_append && rt == 0) {
    // the cache write of this call's new rows for (b, g): split s takes rows
    // s, s + num_splits, ...; positions outside the cache are reported and
    // skipped (as the separate append kernel does)
    const int base = __ldg(p.cache_seqlens + b);
    for (int tn = split; tn < p.Snew; tn += p.num_splits) {
      const long long dst = cache_elem(p, b, base + tn, g);
      if (dst < 0) {
        if (threadIdx.x == 0) report_status(p.status, kStatusBadArg);
        continue;
      }
      if (!FA_IN_BOUNDS(dst + D <= p.ext_cache, p.status)) continue;
      const size_t src = (((size_t)b * p.Snew + tn) * p.Hkv + g) * D;
      for (int c = threadIdx.x; c < CH; c += 32 * kConsumers) {
        *reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.k_cache) + dst + c * 8) =
            *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.k_new) + src + c * 8);
        *reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.v_cache) + dst + c * 8) =
            *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.v_new) + src + c * 8);
      }
    }
  }

  uint32_t qf[KSTEPS][4];
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk)
    ldmatrix_x4(smem_u32(sQ) + swz_offset<D>(lane & 15, kk * 2 + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2],
                qf[kk][3]);

  float o_acc[NT_O][4];
#pragma unroll
  for (int i = 0; i < NT_O; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  const int pr_a = rt * 16 + (lane >> 2), pr_b = pr_a + 8;
  const int qpos_a = pr_a / p.G + L - p.Sq;
  const int qpos_b = pr_b / p.G + L - p.Sq;
  volatile int never = 0;
  bool alive = true;

  for (int tt = warp; alive && tt < n_tt; tt += kConsumers) {
    const int st = tt % kStages, u = tt / kStages;
    if (!__all_sync(0xffffffffu, mbar_wait(full(st), u & 1, &never, kDecWaitNs))) {
      if (lane == 0) report_status(p.status, kStatusTimeout);
      alive = false;
      break;
    }
    const int tb = t0 + tt * kTokT;
    uint8_t* kst = smem + C::OFF_ST + st * C::STAGE;
    const uint32_t kb = sb + C::OFF_ST + st * C::STAGE;
    const uint32_t vb = kb + C::KT;
    if (flag[st]) {
      // rows past the split end may hold anything (even NaN): zero their V
      const int valid = t1 - tb;
      bool patched = false;
      if (valid < kTokT) {
        for (int i = lane; i < (kTokT - valid) * CH; i += 32) {
          const int r = valid + i / CH, j = i % CH;
          *reinterpret_cast<uint4*>(kst + C::KT + tma_sw<kTokT>(r, j)) = make_uint4(0, 0, 0, 0);
        }
        patched = true;
      }
      if (p.fuse_append) {
        // this call's new rows (positions L - Snew .. L - 1) come from
        // k_new / v_new: the cache write of another CTA may not have landed
        const int n0 = max(tb, L - p.Snew), n1 = min(tb + kTokT, t1);
        for (int i = lane; i < (n1 - n0) * CH; i += 32) {
          const int r = n0 - tb + i / CH, j = i % CH;
          const size_t src = (((size_t)b * p.Snew + (n0 + i / CH - (L - p.Snew))) * p.Hkv + g) * D + j * 8;
          if (!FA_IN_BOUNDS(r >= 0 && r < kTokT && src + 8 <= (size_t)p.B * p.Snew * p.Hkv * D, p.status)) continue;
          *reinterpret_cast<uint4*>(kst + tma_sw<kTokT>(r, j)) =
              *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.k_new) + src);
          *reinterpret_cast<uint4*>(kst + C::KT + tma_sw<kTokT>(r, j)) =
              *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.v_new) + src);
        }
        patched = patched || n0 < n1;
      }
      if (patched) {
        // the next TMA write into this stage must come after these stores
        fence_proxy_async_smem();
        __syncwarp();
      }
      float s[NT_S][4];
#pragma unroll
      for (int i = 0; i < NT_S; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
        for (int np = 0; np < NT_S / 2; ++np) {
          uint32_t b0, b1, b2, b3;
          const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          ldmatrix_x4(kb + tma_sw<kTokT>(r, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
          mma16816<T>(s[2 * np], qf[kk], b0, b1);
          mma16816<T>(s[2 * np + 1], qf[kk], b2, b3);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT_S; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = kCap ? p.cap_log2 * tanh_exp(s[nt][e] * p.cap_in) : s[nt][e] * p.scale_log2;
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
      for (int kk = 0; kk < kTokT / 16; ++kk) {
        uint32_t pa[4];
        pa[0] = Elem<T>::pack(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = Elem<T>::pack(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = Elem<T>::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = Elem<T>::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int dp = 0; dp < NT_O / 2; ++dp) {
          uint32_t b0, b1, b2, b3;
          const int r = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          ldmatrix_x4_trans(vb + tma_sw<kTokT>(r, dp * 2 + (lane >> 4)), b0, b1, b2, b3);
          mma16816<T>(o_acc[2 * dp], pa, b0, b1);
          mma16816<T>(o_acc[2 * dp + 1], pa, b2, b3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(st));
  }

  // ---- merge the consumer warps' states (warp w reuses stage w, which it owns)
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  float* wO = reinterpret_cast<float*>(smem + C::OFF_ST + warp * C::STAGE);  // 16 x D fp32 (<= one stage)
  float* wML = wO + 16 * D;
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
  named_bar_sync(1, 32 * kConsumers);

  // each work item: 8 consecutive columns of one of the 16 packed rows
  constexpr int NT = 32 * kConsumers;
  constexpr int ITEMS = 16 * (D / 8);
  for (int item = threadIdx.x; item < ITEMS; item += NT) {
    const int r = item / (D / 8);
    const int c0 = (item % (D / 8)) * 8;
    const int pr = rt * 16 + r;
    if (pr >= rows) continue;
    float mw[kConsumers], lw[kConsumers], M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      const float* ml = reinterpret_cast<const float*>(smem + C::OFF_ST + w * C::STAGE) + 16 * D;
      mw[w] = ml[r];
      lw[w] = ml[16 + r];
      M = fmaxf(M, mw[w]);
    }
    float fw[kConsumers], lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      fw[w] = (M == -INFINITY) ? 0.f : fast_exp2(mw[w] - M);
      lsum += lw[w] * fw[w];
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    const float lse_nat = lsum > 0.f ? (M + log2f(lsum)) * kLn2 : -INFINITY;
    const int sq = pr / p.G;
    const int h = g * p.G + pr % p.G;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      const float* o = reinterpret_cast<const float*>(smem + C::OFF_ST + w * C::STAGE) + r * D + c0;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += o[j] * fw[w];
    }
    if (p.num_splits == 1) {
      const long long oi = (((long long)b * p.Sq + sq) * p.Hq + h) * D + c0;
      if (!FA_IN_BOUNDS(oi >= 0 && oi + 8 <= p.n_out, p.status)) continue;
      T* out = reinterpret_cast<T*>(p.out) + oi;
      uint4 v;
      v.x = Elem<T>::pack(acc[0] * inv, acc[1] * inv);
      v.y = Elem<T>::pack(acc[2] * inv, acc[3] * inv);
      v.z = Elem<T>::pack(acc[4] * inv, acc[5] * inv);
      v.w = Elem<T>::pack(acc[6] * inv, acc[7] * inv);
      *reinterpret_cast<uint4*>(out) = v;
      if (p.lse && c0 == 0) p.lse[((size_t)b * p.Hq + h) * p.Sq + sq] = lse_nat;
    } else {
      const size_t row = (((size_t)split * p.B + b) * p.Hq + h) * p.Sq + sq;
      if (!FA_IN_BOUNDS((long long)row < p.n_part, p.status)) continue;
      float* out = p.o_part + row * D + c0;
      *reinterpret_cast<float4*>(out) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      *reinterpret_cast<float4*>(out + 4) = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      if (c0 == 0) p.lse_part[row] = lse_nat;
    }
  }
}

template <typename T, int D, bool kCap>
cudaError_t launch_t(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t s) {
  auto kern = decode_tma_kernel<T, D, kCap>;
  constexpr int smem = DecCfg<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int nrt = (p.Sq * p.G + 15) / 16;
  dim3 grid(p.num_splits, p.Hkv * nrt, p.B);
  trace_begin(s);
  kern<<<grid, kThreadsD, smem, s>>>(mk, mv, p);
  trace_end(s);
  return cudaGetLastError();
}

}  // namespace

// Rows per TMA box: a whole 32-token tile, or 16 / 8 rows when pages hold a
// multiple of 16 / 8 tokens but not of 32 (a box must stay inside one page);
// 0 when neither fits (the cp.async kernel takes those pages).
int decode_box_rows(const DecodeParams& p) {
  if (!p.paged || p.page_size % kTokT == 0) return kTokT;
  if (p.page_size % 16 == 0) return 16;
  if (p.page_size % 8 == 0) return 8;
  return 0;
}

bool decode_tma_supported(const DecodeParams& p) {
  return (p.D == 64 || p.D == 128) && decode_box_rows(p) > 0 && tma_available();
}

cudaError_t launch_decode_split_tma(const DecodeParams& p_in, fa_dtype dt, cudaStream_t s) {
  CUtensorMap mk, mv;
  DecodeParams p = p_in;
  p.box_rows = decode_box_rows(p);
  if (p.box_rows == 0) return cudaErrorNotSupported;
  const bool bf = dt == FA_BF16;
  // paged: (D, Hkv, page_size, num_pages); contiguous: (D, Hkv, max_seqlen, B)
  const int S = p.paged ? p.page_size : p.max_seqlen;
  const int N = p.paged ? p.capacity_pages : p.B;
  if (S <= 0 || N <= 0) return cudaErrorNotSupported;
  if (!make_bshd_map(&mk, p.k_cache, bf, p.D, p.Hkv, S, N, p.box_rows) ||
      !make_bshd_map(&mv, p.v_cache, bf, p.D, p.Hkv, S, N, p.box_rows))
    return cudaErrorNotSupported;
  const bool cap = p.softcap > 0.f;
  if (p.D == 64) {
    if (bf) return cap ? launch_t<__nv_bfloat16, 64, true>(p, mk, mv, s) : launch_t<__nv_bfloat16, 64, false>(p, mk, mv, s);
    return cap ? launch_t<__half, 64, true>(p, mk, mv, s) : launch_t<__half, 64, false>(p, mk, mv, s);
  }
  if (bf) return cap ? launch_t<__nv_bfloat16, 128, true>(p, mk, mv, s) : launch_t<__nv_bfloat16, 128, false>(p, mk, mv, s);
  return cap ? launch_t<__half, 128, true>(p, mk, mv, s) : launch_t<__half, 128, false>(p, mk, mv, s);
}

}  // namespace fa
