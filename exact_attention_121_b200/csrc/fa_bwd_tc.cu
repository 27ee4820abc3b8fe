// Backward attention on the Blackwell tensor-memory path (tcgen05 + TMA),
// head dim 64 or 128, float32 dQ accumulation through bulk reductions.
//
// The method: "FlashAttention 实战指南" (mhpq.cn), the three techniques — the
// backward pass recomputes the attention probabilities from the saved row
// log-sum-exp instead of reading a stored matrix.
//
// One CTA owns 128 keys of one (batch, kv-head) and walks every q-head of the
// GQA group and every 64-row query block that can see those keys.  Per
// iteration i (query block Q_i, dO_i, LSE_i, Delta_i):
//   S^T  = K Q_i^T        (M=128 keys, N=64 queries, K=D)      -> TMEM
//   dP^T = V dO_i^T                                            -> TMEM
//   P^T  = exp(S^T - LSE), dS^T = P^T (dP^T - Delta) [* (1 - tanh^2)]
//          (warps 0-7, thread = key = TMEM lane; P^T and dS^T go back to
//           TMEM in 16 bits, dS^T also to shared memory)
//   dV  += P^T dO_i       (A = P^T from TMEM)                  -> TMEM
//   dK  += dS^T Q_i       (A = dS^T from TMEM)                 -> TMEM
//   dQ^T = K^T dS^T       (M=128 head dims, N=64 queries)      -> TMEM
//   dQ  += dQ^T^T         (warps 8-11, thread = head-dim index: TMEM ->
//                          shared memory -> bulk fp32 add into the dQ
//                          accumulator in global memory)
// S^T/dP^T live in two TMEM buffers, so the elementwise work of iteration i
// overlaps the products of iteration i+1.  TMEM (512 columns): buffer x at
// [128x, 128x+128) holds S^T [0,64) | dP^T [64,128); the warps that handle
// query half h write P^T (16-bit pairs) to [32h, 32h+16) and dS^T to
// [64+32h, 64+32h+16).  Head dim 128: dQ^T goes over [64,128) once dK has
// read dS^T; dV [256,384), dK [384,512).  Head dim 64: dV [256,320), dK
// [320,384), and one N = 128 product per pair of blocks writes dQ^T of both
// to [384,512).  Warps 0-7 do the elementwise step (two warps
// per TMEM lane quarter, one per query half), warps 8-11 drain dQ, warp 12
// loads (TMA for K, V, Q_i, dO_i; plain loads for LSE/Delta), warp 13 issues
// the MMAs.  Every wait is bounded.
#include <math.h>

#include "fa_common.cuh"
#include "fa_kernels.h"
#include "fa_sm100.cuh"
#include "fa_tma.h"

namespace fa {

namespace {

using namespace sm100;

constexpr int kKeys = 128;
constexpr int kQ = 64;
constexpr int kThreadsB = 448;
constexpr int kDqWarp0 = 8;   // warps 0-7: P^T/dS^T (two per TMEM lane quarter), 8-11: dQ drain
constexpr int kLoadWarp = 12;
constexpr int kMmaWarpB = 13;
constexpr unsigned long long kWaitNs = kWaitLimitNs;

template <int D_>
struct BwdTcCfg {
  static constexpr int D = D_;
  static constexpr int NCH = D / 64;              // 64-column (128-byte) chunks per row
  static constexpr int KV_CHUNK = kKeys * 128;    // 128 rows x 64 columns, 16-bit, swizzled
  static constexpr int KV_TILE = NCH * KV_CHUNK;
  static constexpr int Q_CHUNK = kQ * 128;        // 64 rows x 64 columns
  static constexpr int Q_TILE = NCH * Q_CHUNK;
  static constexpr int DS_TILE = kKeys * kQ * 2;  // [128 keys][64 queries] 16-bit, swizzled
  static constexpr int DQ_TILE = kQ * D * 4;      // [64 queries][D] fp32, dense (TMA reduce box)
  // Head dim 64: dQ^T of two consecutive blocks comes from one N = 128
  // product, so dS keeps four buffers (a pair is two adjacent ones) and the
  // drain stages two dQ tiles.
  static constexpr bool PAIR = (D == 64);
  static constexpr int NDS = PAIR ? 4 : 2;
  static constexpr int NDQ = PAIR ? 2 : 1;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;
  static constexpr int NQS = 3;                        // Q/dO/LSE/Delta stages
  static constexpr int OFF_Q = OFF_V + KV_TILE;        // NQS stages
  static constexpr int OFF_DO = OFF_Q + NQS * Q_TILE;  // NQS stages
  static constexpr int OFF_DS = OFF_DO + NQS * Q_TILE;  // NDS buffers
  static constexpr int OFF_DQ = OFF_DS + NDS * DS_TILE; // NDQ tiles
  static constexpr int OFF_ROW = OFF_DQ + NDQ * DQ_TILE;  // [stage][LSE*log2e 64 | Delta 64]
  static constexpr int OFF_BAR = OFF_ROW + NQS * 2 * kQ * 4;
  enum { B_KV = 0, B_QF = 1, B_QE = B_QF + NQS, B_SDP = B_QE + NQS, B_PDS = B_SDP + 2, B_DQF = B_PDS + 2,
         B_TMF = B_DQF + 2, B_FIN = B_TMF + 2, B_DRAIN = B_FIN + 1, B_DQT_FULL = B_DRAIN + 1,
         B_DQT_FREE = B_DQT_FULL + 1, NBAR = B_DQT_FREE + 1 };
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int OFF_ITEM = OFF_ABORT + 4;  // claimed work item (deterministic mode)
  static constexpr int SMEM = OFF_ITEM + 4 + 1024;
};

__device__ __forceinline__ float f32(uint32_t u) { return __uint_as_float(u); }

template <typename T, int D_, bool kCap, bool kAlibi>
__global__ void __launch_bounds__(kThreadsB, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BwdTcCfg<D_>;
  constexpr int D = C::D;
  constexpr bool kPair = C::PAIR;
  static_assert(C::SMEM <= 227 * 1024, "shared memory per CTA");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
  const uint32_t* tmem_slot = reinterpret_cast<const uint32_t*>(smem + C::OFF_TMEM);
  float* rows = reinterpret_cast<float*>(smem + C::OFF_ROW);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_KV), 1);
    for (int x = 0; x < C::NQS; ++x) {
      mbar_init(bar(C::B_QF + x), 1);
      mbar_init(bar(C::B_QE + x), 1);
    }
    mbar_init(bar(C::B_DQT_FULL), 128);
    mbar_init(bar(C::B_DQT_FREE), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(C::B_SDP + x), 1);
      mbar_init(bar(C::B_PDS + x), 256);
      mbar_init(bar(C::B_DQF + x), 1);
      mbar_init(bar(C::B_TMF + x), 128);
    }
    mbar_init(bar(C::B_FIN), 1);
    mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    // Deterministic mode: items are claimed in order from a global counter,
    // key block major, so every key block a CTA waits for below belongs to
    // a CTA that is already running or done.
    if (p.deterministic) *reinterpret_cast<volatile int*>(smem + C::OFF_ITEM) = atomicAdd(p.work_counter, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarpB) {
    tmem_alloc(sb + C::OFF_TMEM, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    *abort_flag = 1;
    report_status(p.status, kStatusTimeout);
  };

  const int nkb = (p.Sk + kKeys - 1) / kKeys;
  int kb, hb;
  if (p.deterministic) {
    const int item = *reinterpret_cast<volatile int*>(smem + C::OFF_ITEM);
    kb = item / (p.Hkv * p.B);
    hb = item - kb * (p.Hkv * p.B);
  } else {
    // a right bound (causal) gives early key blocks the most query blocks, a
    // left bound alone the late ones: those go first
    group_order((int)blockIdx.x, nkb, p.Hkv * p.B, p.wr < 0 && p.wl >= 0, kb, hb);
  }
  const int hkv = hb % p.Hkv;
  const int b = hb / p.Hkv;
  // this sequence's lengths and rows (packed batches: its own lengths)
  const SeqView seq = seq_view(p, b);
  const int Sq = seq.sq, Sk = seq.sk;
  const int off = Sk - Sq;
  const int k0 = kb * kKeys;
  const int k1 = min(k0 + kKeys, Sk) - 1;  // < k0: no keys of this sequence here
  int i_min = 0, i_max = Sq - 1;
  if (p.wr >= 0) i_min = max(i_min, k0 - off - p.wr);
  if (p.wl >= 0) i_max = min(i_max, k1 - off + p.wl);
  const int qb_lo = i_min / kQ;
  const int n_qb = (k1 >= k0 && i_max >= i_min) ? (i_max / kQ - qb_lo + 1) : 0;
  // bounds-checked build: a CTA whose coordinates fall outside the tensors
  // does no work (it has allocated TMEM already, so it still runs the
  // common teardown)
  const bool coords_ok = FA_IN_BOUNDS(hkv < p.Hkv && b < p.B && hkv * p.G + p.G <= p.Hq, p.status);
  const int n_iter = coords_ok ? n_qb * p.G : 0;
  auto iter_q = [&](int it, int& h, int& q0) {
    h = hkv * p.G + it / n_qb;
    q0 = (qb_lo + it % n_qb) * kQ;
  };

  if (warp == kLoadWarp) {
    // -------------------------------------------------------------- loads
    if (n_iter > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        mbar_expect_tx(bar(C::B_KV), 2 * C::KV_TILE);
        for (int c = 0; c < C::NCH; ++c) {
          tma_load_4d(sb + C::OFF_K + c * C::KV_CHUNK, &tmK, c * 64, hkv, seq.ktma + k0, seq.tb, bar(C::B_KV));
          tma_load_4d(sb + C::OFF_V + c * C::KV_CHUNK, &tmV, c * 64, hkv, seq.ktma + k0, seq.tb, bar(C::B_KV));
        }
      }
      // LSE and Delta of a block's 64 rows (two per lane), read into
      // registers one block ahead so that their global-memory latency
      // overlaps the wait for the stage instead of delaying the Q/dO copies
      constexpr int kRowsPerLane = kQ / 32;
      float nl_next[kRowsPerLane], dl_next[kRowsPerLane];
      auto fetch_rows = [&](int it) {
        int h, q0;
        iter_q(it, h, q0);
        const long long sbase = stat_base(p, seq, b, h);
#pragma unroll
        for (int j = 0; j < kRowsPerLane; ++j) {
          const int q = q0 + lane + 32 * j;
          float l2 = INFINITY, dl = 0.f;
          // rows past the sequence: P = 0, Delta = 0
          if (q < Sq && FA_IN_BOUNDS(sbase + q >= 0 && sbase + q < p.n_stat, p.status)) {
            const float l = p.lse[sbase + q];
            l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;
            dl = p.delta[sbase + q];
          }
          nl_next[j] = -l2;  // x - LSE*log2e becomes one fma: s * scale_log2 + (-LSE*log2e)
          dl_next[j] = dl;
        }
      };
      fetch_rows(0);
      int issued = 0;
      for (int it = 0; it < n_iter; ++it) {
        const int st = it % C::NQS, u = it / C::NQS;
        if (it >= C::NQS &&
            !__all_sync(0xffffffffu, mbar_wait(bar(C::B_QE + st), (u - 1) & 1, abort_flag, kWaitNs))) {
          if (lane == 0) fail();
          break;
        }
        int h, q0;
        iter_q(it, h, q0);
        float* r = rows + st * 2 * kQ;
#pragma unroll
        for (int j = 0; j < kRowsPerLane; ++j) {
          r[lane + 32 * j] = nl_next[j];
          r[kQ + lane + 32 * j] = dl_next[j];
        }
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(bar(C::B_QF + st), 2 * C::Q_TILE);
          for (int c = 0; c < C::NCH; ++c) {
            tma_load_4d(sb + C::OFF_Q + st * C::Q_TILE + c * C::Q_CHUNK, &tmQ, c * 64, h, seq.qtma + q0, seq.tb,
                        bar(C::B_QF + st));
            tma_load_4d(sb + C::OFF_DO + st * C::Q_TILE + c * C::Q_CHUNK, &tmdO, c * 64, h, seq.qtma + q0, seq.tb,
                        bar(C::B_QF + st));
          }
        }
        issued = it + 1;
        if (it + 1 < n_iter) fetch_rows(it + 1);
      }
      if (*abort_flag && lane == 0) {
        volatile int never = 0;
        mbar_wait(bar(C::B_KV), 0, &never, kWaitNs);
        for (int it = max(0, issued - C::NQS); it < issued; ++it)
          mbar_wait(bar(C::B_QF + it % C::NQS), (it / C::NQS) & 1, &never, kWaitNs);
      }
    }
  } else if (warp == kMmaWarpB) {
    // -------------------------------------------------------------- MMA issue
    if (lane == 0 && n_iter > 0) {
      constexpr bool kBf = Elem<T>::kBf16;
      constexpr uint32_t idesc_s = make_idesc(kBf, 128, kQ, false, false);
      constexpr uint32_t idesc_kv = make_idesc(kBf, 128, D, true, false);
      constexpr uint32_t idesc_dq = make_idesc(kBf, 128, kQ, true, true);
      constexpr uint32_t idesc_dq2 = make_idesc(kBf, 128, 2 * kQ, true, true);
      // head dim 64: dV [256,320), dK [320,384), dQ^T of a block pair [384,512)
      const uint32_t tdV = tmem + 256, tdK = tmem + (kPair ? 320 : 384);
      // S^T(it) into [0,64) of buffer it&1, dP^T(it) into [64,128)
      auto issue_s = [&](int it) {
        const int x = it & 1, st = it % C::NQS;
        const uint32_t tb = tmem + x * 128;
        const uint64_t a0 = make_sdesc_sw128(sb + C::OFF_K, 16, 1024);
        const uint64_t b0 = make_sdesc_sw128(sb + C::OFF_Q + st * C::Q_TILE, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
          mma_ss(tb, desc_advance(a0, okv), desc_advance(b0, oq), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_dp = [&](int it) {
        const int x = it & 1, st = it % C::NQS;
        const uint32_t tb = tmem + x * 128;
        const uint64_t a0 = make_sdesc_sw128(sb + C::OFF_V, 16, 1024);
        const uint64_t b0 = make_sdesc_sw128(sb + C::OFF_DO + st * C::Q_TILE, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
          mma_ss(tb + 64, desc_advance(a0, okv), desc_advance(b0, oq), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_grads = [&](int it) {
        const int x = it & 1, st = it % C::NQS;
        const uint32_t tb = tmem + x * 128;
        const uint32_t q_st = sb + C::OFF_Q + st * C::Q_TILE, do_st = sb + C::OFF_DO + st * C::Q_TILE;
        const uint32_t ds = sb + C::OFF_DS + (it % C::NDS) * C::DS_TILE;
        const bool acc = it > 0;
        const uint64_t bv = make_sdesc_sw128(do_st, C::Q_CHUNK, 1024);
        const uint64_t bk = make_sdesc_sw128(q_st, C::Q_CHUNK, 1024);
#pragma unroll
        for (int kk = 0; kk < kQ / 16; ++kk)
          // 16-query k-step kk of P^T sits at column 32*(kk/2) + 8*(kk%2)
          mma_ts(tdV, tb + (kk >> 1) * 32 + (kk & 1) * 8, desc_advance(bv, kk * 16 * 128), idesc_kv,
                 (acc || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kQ / 16; ++kk)
          mma_ts(tdK, tb + 64 + (kk >> 1) * 32 + (kk & 1) * 8, desc_advance(bk, kk * 16 * 128), idesc_kv,
                 (acc || kk > 0) ? 1u : 0u);
        if (kPair) return;
        const uint64_t aq = make_sdesc_sw128(sb + C::OFF_K, C::NCH > 1 ? C::KV_CHUNK : 0, 1024);
        const uint64_t bq = make_sdesc_sw128(ds, C::KV_CHUNK, 1024);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_ss(tb + 64, desc_advance(aq, kk * 16 * 128), desc_advance(bq, kk * 16 * 128), idesc_dq,
                 kk > 0 ? 1u : 0u);
      };
      // Head dim 64: dQ^T of blocks (it0, it0 + n - 1), n = 2 (or 1 for a
      // last unpaired block) into [384, 384 + 64n): M = 128 head dims, where
      // the second 64-row half of K^T points back at the first (LBO 0) and
      // those TMEM lanes are unused; N = 64n queries from n adjacent dS
      // buffers (LBO = one buffer).
      auto issue_dq_pair = [&](int it0, int n) {
        const uint32_t ds = sb + C::OFF_DS + (it0 % C::NDS) * C::DS_TILE;
        const uint32_t idesc = n == 2 ? idesc_dq2 : idesc_dq;
        const uint64_t aq = make_sdesc_sw128(sb + C::OFF_K, 0, 1024);
        const uint64_t bq = make_sdesc_sw128(ds, C::DS_TILE, 1024);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_ss(tmem + 384, desc_advance(aq, kk * 16 * 128), desc_advance(bq, kk * 16 * 128), idesc,
                 kk > 0 ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(C::B_KV), 0, abort_flag, kWaitNs) && mbar_wait(bar(C::B_QF), 0, abort_flag, kWaitNs);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        mma_commit(bar(C::B_SDP));
      }
      for (int it = 0; ok && it < n_iter; ++it) {
        const int x = it & 1, u = it >> 1;
        if (it + 1 < n_iter) {
          const int x1 = (it + 1) & 1, u1 = (it + 1) >> 1;
          const int s1 = (it + 1) % C::NQS, v1 = (it + 1) / C::NQS;
          ok = mbar_wait(bar(C::B_QF + s1), v1 & 1, abort_flag, kWaitNs);
          if (!ok) break;
          tc_fence_after();
          issue_s(it + 1);
          // head dim 128: dQ^T(it-1) sits over the dP^T columns of buffer x1
          // (not the S^T ones): only dP^T(it+1) waits for its drain
          if (!kPair && it + 1 >= 2) {
            ok = mbar_wait(bar(C::B_TMF + x1), (u1 - 1) & 1, abort_flag, kWaitNs);
            if (!ok) break;
            tc_fence_after();
          }
          issue_dp(it + 1);
          mma_commit(bar(C::B_SDP + x1));
        }
        ok = mbar_wait(bar(C::B_PDS + x), u & 1, abort_flag, kWaitNs);
        if (!ok) break;
        tc_fence_after();
        issue_grads(it);
        if (!kPair) {
          mma_commit(bar(C::B_DQF + x));
        } else if ((it & 1) || it == n_iter - 1) {
          // pair m = it / 2 complete (or the last block alone): its dQ^T
          // region is free once the drain has read pair m - 1
          const int m = it >> 1;
          if (m >= 1 && !mbar_wait(bar(C::B_TMF), (m - 1) & 1, abort_flag, kWaitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_dq_pair(2 * m, (it & 1) ? 2 : 1);
          mma_commit(bar(C::B_DQF));
        }
        mma_commit(bar(C::B_QE + it % C::NQS));
      }
      if (ok) mma_commit(bar(C::B_FIN));
      if (!ok) fail();
      mma_commit(bar(C::B_DRAIN));
      volatile int never = 0;
      mbar_wait(bar(C::B_DRAIN), 0, &never, kWaitNs);
    }
  } else if (warp < kDqWarp0) {
    // -------------------------------------------------------------- P^T, dS^T
    // warp = (hh, wq): TMEM lane quarter wq (32 keys) and query half hh.
    const int wq = warp & 3, hh = warp >> 2;
    const int r = wq * 32 + lane;
    const int key = k0 + r;
    const bool key_ok = key <= k1;
    const uint32_t lanes = (uint32_t)(wq * 32) << 16;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int x = it & 1, u = it >> 1;
      int h, q0;
      iter_q(it, h, q0);
      // ALiBi slope of (b, h) as a log2-domain factor of |qpos - key|
      const float mb = kAlibi ? -kLog2e * p.alibi[(long long)b * p.alibi_bstride + h] : 0.f;
      // S^T/dP^T(it) ready also means (commit order) that the products of
      // it-2 that read this TMEM buffer and the dQ^T that read this dS
      // buffer are done
      const bool w = mbar_wait(bar(C::B_SDP + x), u & 1, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem + lanes + x * 128;
      const float* rw = rows + (it % C::NQS) * 2 * kQ + 32 * hh;
      const bool full = (k1 - k0 + 1 == kKeys) && (q0 + kQ <= Sq) &&
                        (p.wl < 0 || k0 >= q0 + kQ - 1 + off - p.wl) && (p.wr < 0 || k1 <= q0 + off + p.wr);
      // This warp's 32 queries: S^T columns [32hh, 32hh+32), dP^T columns
      // [64+32hh, ...), taken in two sub-blocks of 16 queries (sb) to keep
      // few registers live.  P^T (16-bit pairs) of sub-block sb goes to
      // [32hh+8sb, +8) and dS^T to [64+32hh+8sb, +8): inside columns this
      // warp has already read.
      const unsigned long long sl2 = f2_pack(p.scale_log2, p.scale_log2);
      uint8_t* dsrow = smem + C::OFF_DS + (it % C::NDS) * C::DS_TILE + r * 128;
#pragma unroll
      for (int sbk = 0; sbk < 2; ++sbk) {
        const int q16 = 32 * hh + 16 * sbk;  // first query of the sub-block
        uint32_t s[16], dp[16];
        tmem_ld16(tb + q16, s);
        tmem_ld16(tb + 64 + q16, dp);
        const float4* nl4 = reinterpret_cast<const float4*>(rw + 16 * sbk);       // -LSE*log2e
        const float4* dl4 = reinterpret_cast<const float4*>(rw + kQ + 16 * sbk);  // Delta
        float nl[16], dlv[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 a4 = nl4[j], b4 = dl4[j];
          nl[4 * j] = a4.x; nl[4 * j + 1] = a4.y; nl[4 * j + 2] = a4.z; nl[4 * j + 3] = a4.w;
          dlv[4 * j] = b4.x; dlv[4 * j + 1] = b4.y; dlv[4 * j + 2] = b4.z; dlv[4 * j + 3] = b4.w;
        }
        if (kAlibi) {
          // the distance bias joins -LSE*log2e: query q0 + q16 + c
          const float d0 = (float)(q0 + q16 + off - key);
#pragma unroll
          for (int c = 0; c < 16; ++c) nl[c] = fmaf(mb, fabsf(d0 + (float)c), nl[c]);
        }
        tmem_wait_ld();
        reg_fence(s);
        reg_fence(dp);
        uint32_t pk[8], dk[8];
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          float pv[2], dv[2];
          if (kCap) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float t = tanh_exp(f32(s[c + e]) * p.cap_in);
              pv[e] = fast_exp2(fmaf(p.cap_log2, t, nl[c + e]));
              dv[e] = (f32(dp[c + e]) - dlv[c + e]) * (1.f - t * t);
            }
          } else {
            // packed f32x2: one instruction per query pair
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(f32(s[c]), f32(s[c + 1])), sl2, f2_pack(nl[c], nl[c + 1])), x0, x1);
            pv[0] = fast_exp2(x0);
            pv[1] = fast_exp2(x1);
            f2_unpack(f2_sub(f2_pack(f32(dp[c]), f32(dp[c + 1])), f2_pack(dlv[c], dlv[c + 1])), dv[0], dv[1]);
          }
          if (!full) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int qp = q0 + q16 + c + e + off;
              const bool vis = key_ok && (p.wl < 0 || key >= qp - p.wl) && (p.wr < 0 || key <= qp + p.wr);
              pv[e] = vis ? pv[e] : 0.f;
            }
          }
          // dS = P (dP - Delta) [* (1 - tanh^2)]
          f2_unpack(f2_mul(f2_pack(pv[0], pv[1]), f2_pack(dv[0], dv[1])), dv[0], dv[1]);
          pk[c / 2] = Elem<T>::pack(pv[0], pv[1]);
          dk[c / 2] = Elem<T>::pack(dv[0], dv[1]);
        }
        tmem_st8(tb + 32 * hh + 8 * sbk, pk);
        tmem_st8(tb + 64 + 32 * hh + 8 * sbk, dk);
        // dS^T row r, these 16 queries -> shared memory, 128-byte swizzle
        // (MN-major operand of dQ^T)
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int gg = 4 * hh + 2 * sbk + g;
          *reinterpret_cast<uint4*>(dsrow + ((gg ^ (r & 7)) << 4)) =
              make_uint4(dk[4 * g], dk[4 * g + 1], dk[4 * g + 2], dk[4 * g + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(C::B_PDS + x));
    }
    if (ok && n_iter > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_FIN), 0, abort_flag, kWaitNs));
    if (!ok) {
      fail();
    } else {
      // ---- dV and dK rows of this warp's keys, head-dim half hh
      tc_fence_after();
      const long long dv_off = (long long)b * p.st_dv[0] + (long long)(seq.ktma + key) * p.st_dv[1] +
                               (long long)hkv * p.st_dv[2] + hh * (D / 2);
      const long long dk_off = (long long)b * p.st_dk[0] + (long long)(seq.ktma + key) * p.st_dk[1] +
                               (long long)hkv * p.st_dk[2] + hh * (D / 2);
      T* dVr = reinterpret_cast<T*>(p.dv) + dv_off;
      T* dKr = reinterpret_cast<T*>(p.dk) + dk_off;
      const bool rows_ok = key_ok && FA_IN_BOUNDS(dv_off >= 0 && dv_off + D / 2 <= p.ext_dv && dk_off >= 0 &&
                                                       dk_off + D / 2 <= p.ext_dk,
                                                   p.status);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const float mul = which ? p.scale : 1.f;
        T* dst = which ? dKr : dVr;
        const uint32_t src = tmem + lanes + (which ? (kPair ? 320 : 384) : 256) + hh * (D / 2);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t v[32];
          if (n_iter > 0) {
            tmem_ld32(src + c * 32, v);
            tmem_wait_ld();
            reg_fence(v);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          if (rows_ok) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              uint4 o;
              o.x = Elem<T>::pack(f32(v[8 * g + 0]) * mul, f32(v[8 * g + 1]) * mul);
              o.y = Elem<T>::pack(f32(v[8 * g + 2]) * mul, f32(v[8 * g + 3]) * mul);
              o.z = Elem<T>::pack(f32(v[8 * g + 4]) * mul, f32(v[8 * g + 5]) * mul);
              o.w = Elem<T>::pack(f32(v[8 * g + 6]) * mul, f32(v[8 * g + 7]) * mul);
              *reinterpret_cast<uint4*>(dst + c * 32 + 8 * g) = o;
            }
          }
        }
      }
    }
  } else {
    // -------------------------------------------------------------- dQ drain
    const int wq = warp - kDqWarp0;          // TMEM lane quarter = head-dim slice
    const bool has_dims = wq * 32 < D;       // D = 64 uses two of the four warps
    const uint32_t lanes = (uint32_t)(wq * 32) << 16;
    // A drain group is one block (head dim 128, dQ^T in TMEM buffer it & 1)
    // or a pair of blocks (head dim 64, dQ^T of both in [384, 512)).  The
    // dQ tile of a block is [64 queries][D] fp32 in shared memory; every
    // drain thread writes its head-dim column, then one thread adds each
    // tile into the global accumulator with a single tiled TMA reduction.
    // Rows past Sq fall outside the tensor and are skipped by the TMA unit.
    const bool issuer = (warp == kDqWarp0) && lane == 0;
    const int n_groups = kPair ? (n_iter + 1) / 2 : n_iter;
    bool ok = true;
    for (int gi = 0; gi < n_groups; ++gi) {
      const int it0 = kPair ? 2 * gi : gi;
      const int cnt = kPair ? min(2, n_iter - it0) : 1;
      const int bx = kPair ? 0 : (gi & 1);
      const int ph = kPair ? (gi & 1) : ((gi >> 1) & 1);
      bool w = mbar_wait(bar(C::B_DQF + bx), ph, abort_flag, kWaitNs);
      // the tiles are free once the reductions of the previous group have read them
      if (gi >= 1) w = w && mbar_wait(bar(C::B_DQT_FREE), (gi - 1) & 1, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (has_dims) {
#pragma unroll
        for (int i = 0; i < C::NDQ; ++i) {
          if (i < cnt) {
            uint32_t v[kQ];
            const uint32_t tb = tmem + lanes + (kPair ? 384 + 64 * i : bx * 128 + 64);
            tmem_ld32(tb, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld32(tb + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
            tmem_wait_ld();
            reg_fence(v);
            if (i == cnt - 1) {
              // dQ^T of the group is in registers: the region may be rewritten
              tc_fence_before();
              mbar_arrive(bar(C::B_TMF + bx));
            }
            float* tile = reinterpret_cast<float*>(smem + C::OFF_DQ + i * C::DQ_TILE);
#pragma unroll
            for (int c = 0; c < kQ; ++c) tile[c * D + wq * 32 + lane] = f32(v[c]);
          }
        }
        fence_proxy_async_smem();
      } else {
        // no head-dim rows here (D = 64): keep the barrier phases in step
        tc_fence_before();
        mbar_arrive(bar(C::B_TMF + bx));
      }
      mbar_arrive(bar(C::B_DQT_FULL));
      if (issuer) {
        if (!mbar_wait(bar(C::B_DQT_FULL), gi & 1, abort_flag, kWaitNs)) ok = false;
        for (int i = 0; ok && i < cnt; ++i) {
          int h, q0;
          iter_q(it0 + i, h, q0);
          int* sem = nullptr;
          if (p.deterministic) {
            // add after the key blocks before this one that see query block
            // q0/64, in ascending order: wait for their count
            sem = p.sem + ((size_t)b * p.Hq + h) * ((p.Sq + kQ - 1) / kQ) + q0 / kQ;
            const int kb_lo = (p.wl >= 0) ? max(0, q0 + off - p.wl) / kKeys : 0;
            if (!wait_eq_bounded(sem, kb - kb_lo, kWaitNs)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
          }
          // a reduction may not start at a negative coordinate: skipped
          // (and reported) by the bounds-checked build
          if (FA_IN_BOUNDS(q0 >= 0 && h < p.Hq && seq.qtma + q0 >= 0, p.status))
            tma_reduce_add_4d(&tmDQ, 0, h, seq.qtma + q0, seq.tb, sb + C::OFF_DQ + i * C::DQ_TILE);
          bulk_commit();
          if (sem) {
            // the additions are complete in global memory before the count moves
            bulk_wait_all();
            fence_proxy_async_global();
            red_release_add(sem, 1);
          }
        }
        // the tiles may be rewritten once the reductions have read them
        bulk_wait_read_all();
        mbar_arrive(bar(C::B_DQT_FREE));
      }
      if (!__all_sync(0xffffffffu, ok)) break;
    }
    if (issuer) bulk_wait_all();
    if (!ok) fail();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarpB) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <typename T, int D, bool kCap, bool kAlibi>
cudaError_t launch_t(const BwdParams& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mdo, const CUtensorMap& mdq, cudaStream_t s) {
  auto kern = bwd_tc_kernel<T, D, kCap, kAlibi>;
  constexpr int smem = BwdTcCfg<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int nkb = (p.Sk + kKeys - 1) / kKeys;
  const long long items = (long long)nkb * p.Hkv * p.B;
  if (items == 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;  // block index is an int
  trace_begin(s);
  kern<<<(unsigned)items, kThreadsB, smem, s>>>(mq, mk, mv, mdo, mdq, p);
  trace_end(s);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_d(const BwdParams& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mdo, const CUtensorMap& mdq, cudaStream_t s) {
  const bool cap = p.softcap > 0.f;
  if (p.alibi) {
    if (p.D == 64)
      return cap ? launch_t<T, 64, true, true>(p, mq, mk, mv, mdo, mdq, s)
                 : launch_t<T, 64, false, true>(p, mq, mk, mv, mdo, mdq, s);
    return cap ? launch_t<T, 128, true, true>(p, mq, mk, mv, mdo, mdq, s)
               : launch_t<T, 128, false, true>(p, mq, mk, mv, mdo, mdq, s);
  }
  if (p.D == 64)
    return cap ? launch_t<T, 64, true, false>(p, mq, mk, mv, mdo, mdq, s)
               : launch_t<T, 64, false, false>(p, mq, mk, mv, mdo, mdq, s);
  return cap ? launch_t<T, 128, true, false>(p, mq, mk, mv, mdo, mdq, s)
             : launch_t<T, 128, false, false>(p, mq, mk, mv, mdo, mdq, s);
}

}  // namespace

bool bwd_tc_supported(const BwdParams& p) {
  return (p.D == 64 || p.D == 128) && p.Sq >= 1 && p.Sk >= 1 && tma_available();
}

cudaError_t launch_bwd_main_tc(const BwdParams& p, fa_dtype dt, cudaStream_t s) {
  CUtensorMap mq, mk, mv, mdo, mdq;
  const bool bf = dt == FA_BF16;
  // a packed batch is one batch of total_q / total_k token rows
  const int mq_s = p.cu_q ? p.total_q : p.Sq, mk_s = p.cu_q ? p.total_k : p.Sk, mb = p.cu_q ? 1 : p.B;
  if (!make_bshd_map_strided(&mq, p.q, bf, p.D, p.Hq, mq_s, mb, p.st_q, kQ) ||
      !make_bshd_map_strided(&mdo, p.dout, bf, p.D, p.Hq, mq_s, mb, p.st_do, kQ) ||
      !make_bshd_map_strided(&mk, p.k, bf, p.D, p.Hkv, mk_s, mb, p.st_k, kKeys) ||
      !make_bshd_map_strided(&mv, p.v, bf, p.D, p.Hkv, mk_s, mb, p.st_v, kKeys) ||
      !make_bshd_map_f32(&mdq, p.dq_accum, p.D, p.Hq, mq_s, mb, kQ))
    return cudaErrorNotSupported;
  return bf ? launch_d<__nv_bfloat16>(p, mq, mk, mv, mdo, mdq, s) : launch_d<__half>(p, mq, mk, mv, mdo, mdq, s);
}

}  // namespace fa
