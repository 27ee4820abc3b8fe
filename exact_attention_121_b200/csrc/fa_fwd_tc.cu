// Forward attention on the Blackwell tensor-memory path (tcgen05 + TMA).
//
// The method is the one described in "FlashAttention 实战指南" (mhpq.cn), the
// three techniques: tiles of Q, K, V are brought on chip, QK^T and its
// softmax are formed there with a running row maximum and running sum, and the
// n x n score matrix never reaches device memory.
//
// B200 design.  One CTA owns 256 query rows of one (batch, q-head) as two
// 128-row tiles A and B, and 320 threads in four roles:
//   warps 0-3  softmax of tile A  (thread = row = TMEM lane)
//   warps 4-7  softmax of tile B
//   warp  8    TMA producer: Q once, then K/V 128-key tiles through a ring of
//              shared-memory stages (128-byte swizzle, zero fill past the ends)
//   warp  9    MMA issuer: tcgen05.mma with fp32 accumulators in TMEM
// Tensor memory (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+D),
// O_B [384,384+D); P (16-bit) is the A operand of O += P V straight from TMEM.
// Head dim 128: P is written over the first 64 columns of S, and per key tile
// j the MMA warp issues  PV_A(j), S_A(j+1), PV_B(j), S_B(j+1),  so one tile's
// softmax overlaps the other tile's products.  Because a tcgen05.commit tracks
// every earlier MMA of the issuing thread, "S(j+1) is ready" also means "PV(j)
// is done", which is when a softmax warp may rescale its O rows in TMEM.
// Head dim 64: P_t has its own 64 columns after O_t, so S_t(j+1) is issued as
// soon as the softmax warps have read S_t(j) into registers, and the next
// tile's scores are ready when the softmax finishes; the softmax waits for
// PV_t(j-1) only before it writes P_t(j) or rescales O_t.  The running maximum is
// only moved (and O rescaled) when it grows by more than 2^8, which keeps
// every exponent <= 2^8 and makes rescales rare.  O is divided by the sum of
// the 16-bit probabilities the P.V product used (so the rounding of a
// dominant probability cancels), the LSE uses the sum of the fp32 values.
// Every wait is bounded; a timeout records FA_ERR_TIMEOUT and the CTA drains
// its asynchronous work and exits.
#include <math.h>

#include "fa_common.cuh"
#include "fa_kernels.h"
#include "fa_sm100.cuh"
#include "fa_tma.h"

namespace fa {

namespace {

using namespace sm100;

constexpr int kRows = 128;           // rows per Q tile, keys per K/V tile
constexpr int kThreadsTC = 320;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleLog2 = 8.0f;

// Share of the softmax exponentials computed on the FMA pipe instead of the
// MUFU unit: FA_POLY_PAIRS of every 16 element pairs (unmasked tiles only).
// Measured on B200 at S=4096, B=4, non-causal, TFLOP/s (D64 / D128):
// 0 -> 609 / 1004, 2 -> 512 / 817, 4 -> 467 / 770: the extra FMA/ALU
// instructions cost more than the MUFU time they free, so the default is 0.
#ifndef FA_POLY_PAIRS
#define FA_POLY_PAIRS 0
#endif
__host__ __device__ constexpr bool poly_pair(int i) { return ((i * FA_POLY_PAIRS) % 16) < FA_POLY_PAIRS; }

constexpr unsigned long long kTcWaitNs = kWaitLimitNs;

template <int D, bool kF8 = false>
struct TcCfg {
  // A row of a tile is one or two 128-byte swizzle atoms (16-bit elements),
  // or D bytes of E4M3 codes: one 128-byte atom at head dim 128, one 64-byte
  // atom at head dim 64.
  static constexpr int ROWB = (kF8 && D == 64) ? 64 : 128;  // bytes per row of a chunk
  static constexpr int CHUNK = kRows * ROWB;                // one swizzled 128-row chunk
  static constexpr int CHUNK_ELEMS = kF8 ? D : 64;          // head-dim elements per chunk
  static constexpr int NCHUNK = D / CHUNK_ELEMS;
  static constexpr int TILE = CHUNK * NCHUNK;        // one 128-row tile
  // odd stage counts at head dim 64: the loader can then take "stage free"
  // from the S and PV barriers (see the kernel)
  static constexpr int NSK = (D == 128) ? 3 : 5;     // K stages
  static constexpr int NSV = (D == 128) ? 2 : 5;     // V stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE;
  static constexpr int OFF_V = OFF_K + NSK * TILE;
  static constexpr int OFF_BAR = OFF_V + NSV * TILE;
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KF = 1;             // NSK: K tile landed
  static constexpr int B_KE = B_KF + NSK;    // NSK: K stage free (both QK^T products done)
  static constexpr int B_VF = B_KE + NSK;    // NSV: V tile landed
  static constexpr int B_VE = B_VF + NSV;    // NSV: V stage free (both PV products done)
  static constexpr int B_S = B_VE + NSV;     // 2
  static constexpr int B_P = B_S + 2;        // 2
  static constexpr int B_O = B_P + 2;        // 2
  static constexpr int B_SF = B_O + 2;       // 2: S read out of TMEM (separate-P layout)
  static constexpr int B_PV = B_SF + 2;      // 2: PV product done (separate-P layout)
  static constexpr int B_DRAIN = B_PV + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  // E4M3 at head dim 64: 16 KB of unused room after the barriers, so that
  // operand reads cannot leave the CTA's shared memory whatever the rows'
  // swizzle is taken to be
  static constexpr int PAD = ROWB == 64 ? 16384 : 0;
  static constexpr int SMEM = OFF_ABORT + 4 + PAD + 1024;  // + alignment slack
};

__device__ __forceinline__ float f32(uint32_t u) { return __uint_as_float(u); }
// head dim 64 keeps P in its own TMEM columns beside O
__host__ __device__ constexpr bool kSepPLayout(int D) { return D == 64; }

// factor of (batch b, kv-head g) in a (B, Hkv) array; none given = 1
__device__ __forceinline__ float descale_of(const float* d, int b, int g, int Hkv) {
  return d ? d[(long long)b * Hkv + g] : 1.f;
}

// kFp8: q, k, v are E4M3 codes (T is the 16-bit output type), the two
// products run as kind::f8f6f4 and P is quantised to E4M3 in TMEM.
template <typename T, int D, bool kCap, bool kAlibi, bool kFp8>
__global__ void __launch_bounds__(kThreadsTC, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = TcCfg<D, kFp8>;
  // shared-memory operand descriptor of a chunk: 128-byte swizzle (8-row
  // groups 1024 bytes apart), or 64-byte swizzle for E4M3 rows of head dim
  // 64 (8-row groups 512 bytes apart)
  constexpr bool kSw64 = C::ROWB == 64;
  auto sdesc = [](uint32_t a, uint32_t lbo) -> uint64_t {
    return kSw64 ? make_sdesc_sw64(a, lbo, 8 * 64) : make_sdesc_sw128(a, lbo, 8 * 128);
  };
  // TMEM: S_A, S_B [0, 256), O_B ends at 384 + D (P at D = 64 inside O's 128 columns)
  static_assert(384 + (kSepPLayout(D) ? 2 * D : D) <= 512, "tensor-memory columns");
  static_assert(C::SMEM <= 227 * 1024, "shared memory per CTA");
  // Head dim 64 leaves TMEM room for P beside O (P_t at [256+128t+64, +64)),
  // so S_t can be refilled while P_t still feeds the PV product.
  constexpr bool kSepP = (D == 64);
  // "Stage free" signals without commits of their own (one tcgen05 commit
  // fewer each per key tile): K from tile B's S commit, which follows both
  // QK^T of a tile; V (separate-P loop) from tile B's PV commit, which
  // follows both P.V.  A barrier whose phase is the tile cannot be two
  // phases past the tile the loader waits for when the stage count is odd:
  // the tile being loaded has not been issued, so its products cannot
  // complete.
  constexpr bool kKeFromS = (C::NSK % 2 == 1) && C::NSK >= 3;
  constexpr bool kVeFromPv = kSepP && (C::NSV % 2 == 1) && C::NSV >= 3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
  const uint32_t* tmem_slot = reinterpret_cast<const uint32_t*>(smem + C::OFF_TMEM);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_qp = (p.Sq + 2 * kRows - 1) / (2 * kRows);
  // with a right bound (causal) later query pairs see more keys: first
  int qp, hb;
  group_order((int)blockIdx.x, n_qp, p.Hq * p.B, p.wr >= 0, qp, hb);
  const int h = hb % p.Hq;
  const int b = hb / p.Hq;
  const int g = h / p.G;
  const int q0 = qp * 2 * kRows;
  // this sequence's lengths and rows (packed batches: its own lengths)
  const SeqView seq = seq_view(p, b);
  const int Sq = seq.sq, Sk = seq.sk;
  if (q0 >= Sq) return;  // a shorter sequence of a packed batch: no rows here
  // bounds-checked build: the CTA's head and batch coordinates (every
  // thread takes the same branch, before any barrier)
  if (!FA_IN_BOUNDS(h < p.Hq && g < p.Hkv && b < p.B, p.status)) return;
  const int off = Sk - Sq;
  const int qlast = min(q0 + 2 * kRows, Sq) - 1;
  int kmin = 0, kmax = Sk - 1;
  if (p.wl >= 0) kmin = max(kmin, q0 + off - p.wl);
  if (p.wr >= 0) kmax = min(kmax, qlast + off + p.wr);
  const int kt_begin = kmin / kRows;
  const int n_tiles = (kmax >= kmin) ? (kmax / kRows + 1 - kt_begin) : 0;
  // Head dim 128: Q tile A (the CTA's first 128 rows) skips the trailing key
  // tiles that a right bound (causal) masks for all of its rows; tile B
  // takes them alone.  (Not with ALiBi, whose tile order is rotated; not at
  // head dim 64, where the extra branches in the issue loop cost more than
  // the skipped products save.)
  int n_tiles_a = n_tiles;
  if (p.wr >= 0 && !kAlibi && !kSepP) {
    const int kmax_a = min(Sk - 1, min(q0 + kRows, Sq) - 1 + off + p.wr);
    n_tiles_a = (kmax_a >= kmin) ? min(n_tiles, kmax_a / kRows + 1 - kt_begin) : 0;
  }
  // Key-tile order.  Plain: ascending.  ALiBi: the tile at the diagonal of
  // the CTA's rows first, then the rest in ascending order from the far end,
  // so the running maximum is set at once and the (lower) bias of later
  // tiles rarely moves it: few rescales of O.  The result does not depend
  // on the order.
  const int rot = kAlibi ? min(max((q0 + off + kRows) / kRows - kt_begin, 0), max(n_tiles - 1, 0)) : 0;
  auto tile_k0 = [&](int j) {
    const int t = (j + rot < n_tiles) ? j + rot : j + rot - n_tiles;
    return (kt_begin + t) * kRows;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < C::NSK; ++s) {
      mbar_init(bar(C::B_KF + s), 1);
      mbar_init(bar(C::B_KE + s), 1);
    }
    for (int s = 0; s < C::NSV; ++s) {
      mbar_init(bar(C::B_VF + s), 1);
      mbar_init(bar(C::B_VE + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::B_S + t), 1);
      mbar_init(bar(C::B_P + t), 4 * 32);
      mbar_init(bar(C::B_O + t), 1);
      mbar_init(bar(C::B_SF + t), 4 * 32);
      mbar_init(bar(C::B_PV + t), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
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

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bar(C::B_Q), 2 * C::TILE);
      for (int t = 0; t < 2; ++t)
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d(sb + C::OFF_Q + t * C::TILE + c * C::CHUNK, &tmQ, c * C::CHUNK_ELEMS, h,
                      seq.qtma + q0 + t * kRows, seq.tb, bar(C::B_Q));
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int sk = j % C::NSK, uk = j / C::NSK;
        const int sv = j % C::NSV, uv = j / C::NSV;
        const int k0 = tile_k0(j);
        (void)FA_IN_BOUNDS(k0 >= 0 && k0 < Sk, p.status);  // TMA fills outside the tensor; report only
        // K stage free: both QK^T products of tile j - NSK done
        const bool free_k =
            j < C::NSK ||
            (!kKeFromS ? mbar_wait(bar(C::B_KE + sk), (uk - 1) & 1, abort_flag, kTcWaitNs)
                       : mbar_wait(bar(C::B_S + 1), (j - C::NSK) & 1, abort_flag, kTcWaitNs));
        if (!free_k) {
          fail();
          break;
        }
        mbar_expect_tx(bar(C::B_KF + sk), C::TILE);
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d(sb + C::OFF_K + sk * C::TILE + c * C::CHUNK, &tmK, c * C::CHUNK_ELEMS, g, seq.ktma + k0,
                      seq.tb, bar(C::B_KF + sk));
        const bool free_v =
            j < C::NSV ||
            (!kVeFromPv ? mbar_wait(bar(C::B_VE + sv), (uv - 1) & 1, abort_flag, kTcWaitNs)
                        : mbar_wait(bar(C::B_PV + 1), (j - C::NSV) & 1, abort_flag, kTcWaitNs));
        if (!free_v) {
          fail();
          issued = -(j + 1);  // K of tile j is in flight, V is not
          break;
        }
        mbar_expect_tx(bar(C::B_VF + sv), C::TILE);
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d(sb + C::OFF_V + sv * C::TILE + c * C::CHUNK, &tmV, c * C::CHUNK_ELEMS, g, seq.ktma + k0,
                      seq.tb, bar(C::B_VF + sv));
        issued = j + 1;
      }
      if (*abort_flag) {
        // let every load still in flight land before the CTA exits
        volatile int never = 0;
        const int nk = issued < 0 ? -issued : issued;   // tiles whose K was issued
        const int nv = issued < 0 ? nk - 1 : issued;    // tiles whose V was issued
        mbar_wait(bar(C::B_Q), 0, &never, kTcWaitNs);
        for (int j = max(0, nk - C::NSK); j < nk; ++j)
          mbar_wait(bar(C::B_KF + j % C::NSK), (j / C::NSK) & 1, &never, kTcWaitNs);
        for (int j = max(0, nv - C::NSV); j < nv; ++j)
          mbar_wait(bar(C::B_VF + j % C::NSV), (j / C::NSV) & 1, &never, kTcWaitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && n_tiles > 0) {
      // format fields: bf16 / f16 for kind::f16, E4M3 (0) for kind::f8f6f4
      constexpr bool kBf = !kFp8 && Elem<T>::kBf16;
      constexpr uint32_t idesc_qk = make_idesc(kBf, 128, 128, false);
      constexpr uint32_t idesc_pv = make_idesc(kBf, 128, D, true);
      constexpr int KS = kFp8 ? 32 : 16;  // elements per MMA k-step (32 bytes either way)
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 384};
      const uint32_t tP[2] = {kSepP ? tmem + 256 + D : tS[0], kSepP ? tmem + 384 + D : tS[1]};
      auto issue_qk = [&](int t, int st) {
        const uint64_t a0 = sdesc(sb + C::OFF_Q + t * C::TILE, 16);
        const uint64_t b0 = sdesc(sb + C::OFF_K + st * C::TILE, 16);
#pragma unroll
        for (int kk = 0; kk < D / KS; ++kk) {
          const uint32_t koff = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          const uint64_t ad = desc_advance(a0, koff);
          const uint64_t bd = desc_advance(b0, koff);
          if constexpr (kFp8)
            mma_ss_f8(tS[t], ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
          else
            mma_ss(tS[t], ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int st, bool acc) {
        const uint64_t b0 = sdesc(sb + C::OFF_V + st * C::TILE, C::CHUNK);
#pragma unroll
        for (int kk = 0; kk < kRows / KS; ++kk) {
          // KS keys of V (MN-major: rows of head-dim elements); P packs KS
          // keys into 8 TMEM columns
          const uint64_t bd = desc_advance(b0, kk * KS * C::ROWB);
          if constexpr (kFp8)
            mma_ts_f8(tO[t], tP[t] + kk * 8, bd, idesc_pv, (acc || kk > 0) ? 1u : 0u);
          else
            mma_ts(tO[t], tP[t] + kk * 8, bd, idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(bar(C::B_Q), 0, abort_flag, kTcWaitNs);
      ok = ok && mbar_wait(bar(C::B_KF + 0), 0, abort_flag, kTcWaitNs);
      if (ok) {
        tc_fence_after();
        if (n_tiles_a > 0) {
          issue_qk(0, 0);
          mma_commit(bar(C::B_S + 0));
        }
        issue_qk(1, 0);
        mma_commit(bar(C::B_S + 1));
        if (!kKeFromS) mma_commit(bar(C::B_KE + 0));
      }
      // Separate-P order: QK_t(j+1) as soon as the softmax has read S_t(j),
      // PV_t(j) once it has written P_t(j).
      for (int j = 0; kSepP && ok && j < n_tiles; ++j) {
        const int sv = j % C::NSV, uv = j / C::NSV;
        const int sk1 = (j + 1) % C::NSK, uk1 = (j + 1) / C::NSK;
        const bool more = j + 1 < n_tiles;
        if (more) {
          ok = mbar_wait(bar(C::B_KF + sk1), uk1 & 1, abort_flag, kTcWaitNs) &&
               mbar_wait(bar(C::B_SF + 0), j & 1, abort_flag, kTcWaitNs);
          if (!ok) break;
          tc_fence_after();
          issue_qk(0, sk1);
          mma_commit(bar(C::B_S + 0));
        }
        ok = mbar_wait(bar(C::B_VF + sv), uv & 1, abort_flag, kTcWaitNs) &&
             mbar_wait(bar(C::B_P + 0), j & 1, abort_flag, kTcWaitNs);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, sv, j > 0);
        mma_commit(bar(C::B_PV + 0));
        if (!more) mma_commit(bar(C::B_O + 0));
        if (more) {
          ok = mbar_wait(bar(C::B_SF + 1), j & 1, abort_flag, kTcWaitNs);
          if (!ok) break;
          tc_fence_after();
          issue_qk(1, sk1);
          mma_commit(bar(C::B_S + 1));
          if (!kKeFromS) mma_commit(bar(C::B_KE + sk1));
        }
        ok = mbar_wait(bar(C::B_P + 1), j & 1, abort_flag, kTcWaitNs);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, sv, j > 0);
        mma_commit(bar(C::B_PV + 1));
        if (!kVeFromPv) mma_commit(bar(C::B_VE + sv));
        if (!more) mma_commit(bar(C::B_O + 1));
      }
      for (int j = 0; !kSepP && ok && j < n_tiles; ++j) {
        const int sv = j % C::NSV, uv = j / C::NSV;
        const int sk1 = (j + 1) % C::NSK, uk1 = (j + 1) / C::NSK;
        const bool more = j + 1 < n_tiles;
        const bool a_now = j < n_tiles_a, a_more = j + 1 < n_tiles_a;
        ok = mbar_wait(bar(C::B_VF + sv), uv & 1, abort_flag, kTcWaitNs) &&
             (!a_now || mbar_wait(bar(C::B_P + 0), j & 1, abort_flag, kTcWaitNs));
        if (!ok) break;
        tc_fence_after();
        if (a_now) issue_pv(0, sv, j > 0);
        if (more) {
          ok = mbar_wait(bar(C::B_KF + sk1), uk1 & 1, abort_flag, kTcWaitNs);
          if (!ok) break;
          tc_fence_after();
        }
        if (a_more) {
          issue_qk(0, sk1);
          mma_commit(bar(C::B_S + 0));
        } else if (a_now) {
          mma_commit(bar(C::B_O + 0));
        }
        ok = mbar_wait(bar(C::B_P + 1), j & 1, abort_flag, kTcWaitNs);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, sv, j > 0);
        mma_commit(bar(C::B_VE + sv));
        if (more) {
          issue_qk(1, sk1);
          mma_commit(bar(C::B_S + 1));
          if (!kKeFromS) mma_commit(bar(C::B_KE + sk1));
        } else {
          mma_commit(bar(C::B_O + 1));
        }
      }
      if (!ok) fail();
      // drain: every MMA issued above has completed before TMEM is released
      mma_commit(bar(C::B_DRAIN));
      volatile int never = 0;
      mbar_wait(bar(C::B_DRAIN), 0, &never, kTcWaitNs);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;       // Q tile
    const int wq = warp & 3;       // lane quarter
    const int r = wq * 32 + lane;  // row in the tile = TMEM lane
    const uint32_t lanes = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lanes + t * 128;
    const uint32_t tO = tmem + lanes + 256 + t * 128;
    const uint32_t tP = kSepP ? tO + D : tS;
    const int qi = q0 + t * kRows + r;
    const int qpos = qi + off;
    const int qpos_first = q0 + off, qpos_last = qlast + off;
    float m_run = -INFINITY, l_run = 0.f, l_q = 0.f;
    // ALiBi slope of this (b, h), as a log2-domain factor of |qpos - key|
    const float mb = kAlibi ? -kLog2e * p.alibi[(long long)b * p.alibi_bstride + h] : 0.f;
    // 8-bit inputs: the q and k factors of (b, kv-head g) scale the raw scores
    const float qk_f = kFp8 ? descale_of(p.descale_q, b, g, p.Hkv) * descale_of(p.descale_k, b, g, p.Hkv) : 1.f;
    const float scale_log2 = p.scale_log2 * qk_f, cap_in = p.cap_in * qk_f;
    bool ok = true;
    const int n_mine = t == 0 ? n_tiles_a : n_tiles;
    for (int j = 0; j < n_mine; ++j) {
      // warp-uniform outcome: the TMEM accesses below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(bar(C::B_S + t), j & 1, abort_flag, kTcWaitNs))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[kRows];  // raw scores (fp32 bits), then log2-domain scores
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_wait_ld();
      reg_fence(s);
      if (kSepP) {
        // S_t may be overwritten by the next QK^T from here on
        tc_fence_before();
        mbar_arrive(bar(C::B_SF + t));
      }
      const int k0 = tile_k0(j);
      const bool full = (k0 + kRows <= Sk) && (p.wl < 0 || k0 >= qpos_last - p.wl) &&
                        (p.wr < 0 || k0 + kRows - 1 <= qpos_first + p.wr);
      // row maximum in the log2 domain (the scale is positive: max commutes)
      float mx = -INFINITY;
      if (kCap) {
#pragma unroll
        for (int i = 0; i < kRows; ++i) s[i] = __float_as_uint(p.cap_log2 * tanh_exp(f32(s[i]) * cap_in));
      }
      if (kAlibi) {
        // to the log2 domain, plus the distance bias mb |qpos - key| of key
        // k0 + i.  A tile on one side of every row of the warp has a bias
        // linear in i: t0 + step i, one fma per key (without the softcap:
        // beside the tanh the second copy of the loop costs spills).
        const float in = kCap ? 1.f : scale_log2;
        const bool left = !kCap && __all_sync(0xffffffffu, k0 + kRows - 1 <= qpos);
        const bool right = !kCap && __all_sync(0xffffffffu, k0 >= qpos);
        if (left || right) {
          const float t0 = mb * fabsf((float)(qpos - k0));
          const float step = left ? -mb : mb;
#pragma unroll
          for (int i = 0; i < kRows; ++i) s[i] = __float_as_uint(fmaf(f32(s[i]), in, fmaf(step, (float)i, t0)));
        } else {
          const float d0 = (float)(qpos - k0);
#pragma unroll
          for (int i = 0; i < kRows; ++i) s[i] = __float_as_uint(fmaf(f32(s[i]), in, mb * fabsf(d0 - (float)i)));
        }
      }
      if (!full) {
        // Visible keys of this row in this tile as one range [lo, hi]
        // relative to k0.  (A per-key test of the three bounds made these
        // tiles ~7x slower than unmasked ones: 15.5k against 2.1k cycles.)
        int lo = 0, hi = min(Sk - 1 - k0, kRows - 1);
        if (p.wl >= 0) lo = max(lo, qpos - p.wl - k0);
        if (p.wr >= 0) hi = min(hi, qpos + p.wr - k0);
        // one unsigned compare per score: i is visible iff i - lo <= hi - lo
        // (an empty range moves lo past the tile)
        if (hi < lo) lo = hi = kRows;
        const unsigned span = (unsigned)(hi - lo);
#pragma unroll
        for (int i = 0; i < kRows; ++i)
          if ((unsigned)(i - lo) > span) s[i] = __float_as_uint(-INFINITY);
      }
      {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < kRows; i += 8) {
          m4[0] = fmax3(m4[0], f32(s[i]), f32(s[i + 1]));
          m4[1] = fmax3(m4[1], f32(s[i + 2]), f32(s[i + 3]));
          m4[2] = fmax3(m4[2], f32(s[i + 4]), f32(s[i + 5]));
          m4[3] = fmax3(m4[3], f32(s[i + 6]), f32(s[i + 7]));
        }
        mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
      const float sl = (kCap || kAlibi) ? 1.f : scale_log2;  // multiplier into the log2 domain
      mx *= sl;
      // lazy rescale: move the running max only when it grows by > 2^8
      const bool move = (mx > m_run + kRescaleLog2) || (m_run == -INFINITY && mx != -INFINITY);
      const float alpha = move ? fast_exp2(m_run - mx) : 1.f;
      if (move) m_run = mx;
      const float mu = (m_run == -INFINITY) ? 0.f : m_run;
      // P = 2^(s*sl - mu), packed to 16 bits into P_t (over the first 64
      // columns of S_t at head dim 128).
      // Two row sums: of the exact fp32 values (for the LSE) and of the
      // 16-bit values the P.V product actually uses (for O = sum(P V) / l),
      // so that the rounding of a dominant probability cancels in O.
      // packed f32x2 arithmetic: one instruction per element pair for the
      // scale-and-shift and for each of the two row sums
      const unsigned long long sl2 = f2_pack(sl, sl), nmu2 = f2_pack(-mu, -mu);
      unsigned long long rs2 = f2_pack(0.f, 0.f), rq2 = f2_pack(0.f, 0.f);
      uint32_t pkall[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t (&pk)[16] = pkall[c];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(f32(s[c * 32 + 2 * i]), f32(s[c * 32 + 2 * i + 1])), sl2, nmu2), x0, x1);
          float p0, p1;
          if (full && poly_pair(i)) {
            exp2_poly2(x0, x1, p0, p1);
          } else {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          }
          rs2 = f2_add(rs2, f2_pack(p0, p1));
          float2 pr;
          if constexpr (kFp8) {
            // four E4M3 keys per TMEM column, lowest key in the low byte
            const uint32_t h8 = f32x2_to_e4m3x2(p0, p1);
            pk[i >> 1] = (i & 1) ? (pk[i >> 1] | (h8 << 16)) : h8;
            pr = e4m3x2_to_f32x2(h8);
          } else {
            pk[i] = Elem<T>::pack(p0, p1);
            pr = Elem<T>::unpack(pk[i]);
          }
          rq2 = f2_add(rq2, f2_pack(pr.x, pr.y));
        }
        if constexpr (kFp8) {
          if (!kSepP) tmem_st8(tP + c * 8, *reinterpret_cast<uint32_t(*)[8]>(&pk[0]));
        } else if (!kSepP) {
          tmem_st16(tP + c * 16, pk);
        }
      }
      if (kSepP) {
        // P_t and O_t are free once PV_t(j-1) has completed
        if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(C::B_PV + t), (j - 1) & 1, abort_flag, kTcWaitNs))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if constexpr (kFp8)
            tmem_st8(tP + c * 8, *reinterpret_cast<uint32_t(*)[8]>(&pkall[c][0]));
          else
            tmem_st16(tP + c * 16, pkall[c]);
        }
      }
      float rsa, rsb, rqa, rqb;
      f2_unpack(rs2, rsa, rsb);
      f2_unpack(rq2, rqa, rqb);
      l_run = l_run * alpha + (rsa + rsb);
      l_q = l_q * alpha + (rqa + rqb);
      if (__any_sync(0xffffffffu, move && j > 0 && alpha != 1.f)) {
        // O(j-1) is complete (head dim 128: S(j) was committed after
        // PV(j-1); head dim 64: waited for above); PV(j) waits for this
        // tile's arrive below.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld32(tO + c * 32, u);
          tmem_wait_ld();
          reg_fence(u);
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(f32(u[i]) * alpha);
          tmem_st32(tO + c * 32, u);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::B_P + t));
    }
    if (ok && n_mine > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_O + t), 0, abort_flag, kTcWaitNs));
    if (!ok) {
      fail();
    } else {
      // ---- epilogue: O / l in 16 bits, LSE
      tc_fence_after();
      // O / l (times the v factor of (b, g) for 8-bit inputs)
      const float ov = kFp8 ? descale_of(p.descale_v, b, g, p.Hkv) : 1.f;
      const float inv = l_q > 0.f ? ov / l_q : 0.f;
      const long long o_off =
          (long long)b * p.st_o[0] + (long long)(seq.qtma + qi) * p.st_o[1] + (long long)h * p.st_o[2];
      T* orow = reinterpret_cast<T*>(p.o) + o_off;
      const bool row_ok = qi < Sq && FA_IN_BOUNDS(o_off >= 0 && o_off + D <= p.ext_o, p.status);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        if (n_mine > 0) {
          tmem_ld32(tO + c * 32, u);
          tmem_wait_ld();
          reg_fence(u);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = 0u;
        }
        if (row_ok) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = Elem<T>::pack(f32(u[v4 * 8 + 0]) * inv, f32(u[v4 * 8 + 1]) * inv);
            w.y = Elem<T>::pack(f32(u[v4 * 8 + 2]) * inv, f32(u[v4 * 8 + 3]) * inv);
            w.z = Elem<T>::pack(f32(u[v4 * 8 + 4]) * inv, f32(u[v4 * 8 + 5]) * inv);
            w.w = Elem<T>::pack(f32(u[v4 * 8 + 6]) * inv, f32(u[v4 * 8 + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + v4 * 8) = w;
          }
        }
      }
      const long long li = stat_base(p, seq, b, h) + qi;
      if (qi < Sq && FA_IN_BOUNDS(li >= 0 && li < p.n_stat, p.status))
        p.lse[li] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <typename T, int D, bool kCap, bool kAlibi, bool kFp8 = false>
cudaError_t launch_t(const FwdParams& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     cudaStream_t s) {
  auto kern = fwd_tc_kernel<T, D, kCap, kAlibi, kFp8>;
  constexpr int smem = TcCfg<D, kFp8>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long ctas = (long long)((p.Sq + 255) / 256) * p.Hq * p.B;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;  // block index is an int
  dim3 grid((unsigned)ctas);
  trace_begin(s);
  kern<<<grid, kThreadsTC, smem, s>>>(mq, mk, mv, p);
  trace_end(s);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dt(const FwdParams& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      cudaStream_t s) {
  const bool cap = p.softcap > 0.f;
  if (p.alibi) {
    if (p.D == 64)
      return cap ? launch_t<T, 64, true, true>(p, mq, mk, mv, s) : launch_t<T, 64, false, true>(p, mq, mk, mv, s);
    return cap ? launch_t<T, 128, true, true>(p, mq, mk, mv, s) : launch_t<T, 128, false, true>(p, mq, mk, mv, s);
  }
  if (p.D == 64)
    return cap ? launch_t<T, 64, true, false>(p, mq, mk, mv, s) : launch_t<T, 64, false, false>(p, mq, mk, mv, s);
  return cap ? launch_t<T, 128, true, false>(p, mq, mk, mv, s) : launch_t<T, 128, false, false>(p, mq, mk, mv, s);
}

}  // namespace

bool fwd_tc_supported(const FwdParams& p) {
  return (p.D == 64 || p.D == 128) && p.Sk >= 1 && p.Sq >= 1 && tma_available();
}

cudaError_t launch_fwd_tc_fp8(const FwdParams& p, cudaStream_t s, int* launches) {
  if ((p.D != 128 && p.D != 64) || p.cu_q || p.alibi) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv;
  if (!make_bshd_map_u8(&mq, p.q, p.D, p.Hq, p.Sq, p.B, 128) || !make_bshd_map_u8(&mk, p.k, p.D, p.Hkv, p.Sk, p.B, 128) ||
      !make_bshd_map_u8(&mv, p.v, p.D, p.Hkv, p.Sk, p.B, 128))
    return cudaErrorNotSupported;
  const bool cap = p.softcap > 0.f;
  cudaError_t e;
  if (p.D == 64)
    e = cap ? launch_t<__nv_bfloat16, 64, true, false, true>(p, mq, mk, mv, s)
            : launch_t<__nv_bfloat16, 64, false, false, true>(p, mq, mk, mv, s);
  else
    e = cap ? launch_t<__nv_bfloat16, 128, true, false, true>(p, mq, mk, mv, s)
            : launch_t<__nv_bfloat16, 128, false, false, true>(p, mq, mk, mv, s);
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_fwd_tc(const FwdParams& p, fa_dtype dt, cudaStream_t s, int* launches) {
  CUtensorMap mq, mk, mv;
  const bool bf = dt == FA_BF16;
  // a packed batch is one batch of total_q / total_k token rows
  const int mq_s = p.cu_q ? p.total_q : p.Sq, mk_s = p.cu_q ? p.total_k : p.Sk, mb = p.cu_q ? 1 : p.B;
  if (!make_bshd_map_strided(&mq, p.q, bf, p.D, p.Hq, mq_s, mb, p.st_q, 128) ||
      !make_bshd_map_strided(&mk, p.k, bf, p.D, p.Hkv, mk_s, mb, p.st_k, 128) ||
      !make_bshd_map_strided(&mv, p.v, bf, p.D, p.Hkv, mk_s, mb, p.st_v, 128))
    return cudaErrorNotSupported;
  cudaError_t e = bf ? launch_dt<__nv_bfloat16>(p, mq, mk, mv, s) : launch_dt<__half>(p, mq, mk, mv, s);
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace fa
