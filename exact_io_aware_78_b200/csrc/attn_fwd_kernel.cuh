// attn_fwd_kernel.cuh -- exact attention forward for sm_100a.
//
// O = softmax(scale * Q K^T + mask) V and the per-row log-sum-exp, computed
// tile by tile in on-chip memory so that no N x N matrix reaches HBM
// ("Flash Attention" concept note (heepie.pages.dev), "Tiling" and the TO-BE
// diagram; FlashAttention quiz (aiunderstanding.org), questions 3-5).
//
// Design (B200-specific; the pages give no kernel design for this GPU):
//   * One persistent CTA per SM walks work items (batch b, query head h,
//     256-row query block) in a static heaviest-first order: parallelism over
//     sequence blocks of one head ("FlashAttention-2 (PL)", "Ulepszony
//     rownoleglosc").  With per-row key ranges, whose costs follow no order,
//     each CTA instead takes its next item from a global counter when it
//     starts one (a dynamic deal), and its load warp hands the item to the
//     other roles.
//   * A work item holds two 128-row query tiles of the same (b, h).  They
//     share every K/V tile the TMA warp streams through a shared-memory ring,
//     and ping-pong on the tensor core: while one tile's softmax runs on the
//     CUDA cores, the other tile's two products run on the tensor core
//     (asynchrony, quiz question 8 / FA-3 on the same page).
//   * tcgen05.mma computes S = Q K^T into tensor memory (fp32); the softmax
//     warpgroup owning the tile reads its rows (one thread per row, so row
//     max and row sum need no cross-thread exchange: "Zoptymalizowany podzial
//     pracy wewnatrz bloku"), applies the mask, runs exp2 with the scale
//     folded in, keeps a running max m and sum l, writes P (bf16 or e4m3)
//     back over S in tensor memory, and the MMA warp issues O += P V with P
//     read straight from tensor memory.
//   * The running max is used lazily: O and l are rescaled only when the
//     tile max exceeds the max in use by more than kTau (log2 units), so the
//     non-matmul work stays small ("Minimalizacja operacji nie-macierzowych").
//   * The epilogue divides by l, converts, stores O and LSE = ln2 (m + log2 l).
//   * Masks: causal and window masks become K/V tile ranges plus in-tile
//     masking; per-row key ranges (one contiguous range of visible keys per
//     query row, shared by all heads -- the mask decides which queries see
//     which keys: Hacker News discussion, item 40939398; richer masks as in
//     the FlashMask work listed by "FlashAttention-2 (PL)") are reduced
//     per 128-row tile to a K/V tile range by a small pre-pass kernel, and
//     each softmax thread masks its own row.  A tile no row of which sees a
//     key takes no part in the pipeline and stores O = 0, LSE = -inf.
//   * Every pipeline wait is bounded: past the time limit the thread records
//     a timeout in the device error word, raises a CTA-wide abort flag and
//     all roles unwind; tensor memory is released and no trap is issued.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace ea {

// Device error word layout: (kind << 16) | site.
enum : int { kErrTimeout = 1 };
enum : int {
  kSiteProdQEmpty = 1,
  kSiteProdKvEmpty = 2,
  kSiteMmaQFull = 3,
  kSiteMmaKvFull = 4,
  kSiteMmaPFull = 5,
  kSiteMmaOEmpty = 6,
  kSiteSoftSFull = 7,
  kSiteSoftOFull = 8,
  kSiteMmaDrain = 9,
  kSiteProdDrain = 10,
  kSiteItemFull = 11,   // row ranges: a consumer waiting for the next work item
  kSiteItemEmpty = 12   // row ranges: the load warp waiting for a free item slot
};

// Output modes of the epilogue.
enum : int {
  kOutBf16 = 0,      // O = acc / l (x v_scale for fp8), stored bf16
  kOutF32Split = 1,  // O = (acc[:, :dv/2] + acc[:, dv/2:]) / l, stored fp32
};

struct FwdParams {
  const float* q_scale;  // [Hq] (fp8 only)
  const float* k_scale;  // [Hkv]
  const float* v_scale;  // [Hkv]
  void* o;               // [B, N, Hq, d_out]
  float* lse;            // [B, Hq, N]
  int* err;              // device error word
  const int* key_lo;     // [B, N] per-row key ranges, or null: row i sees keys key_lo <= j < key_hi
  const int* key_hi;     // [B, N]
  const int2* tile_kv;   // [B, num_qtiles] K/V tile range [x, y) of each 128-row query tile (with ranges)
  const int* item_order; // [B * num_qblk] (batch, query block) pairs, most K/V tiles first (with ranges), or null
  int* item_counter;     // with ranges: the dynamic deal's counter of items taken after each CTA's first
                         // (zeroed before the launch), or null for the static deal
  int num_qtiles;        // ceil(N / 128)
  int B, Hq, Hkv, N, group;
  int causal, window;
  float scale_log2;      // scale * log2(e)
  int num_qblk;          // ceil(N / 256)
  int num_work;          // B * Hq * num_qblk
  int order;             // 0: heaviest query blocks first, 1: lightest first
  int skip_first_kv;     // test hook: never fill the first K/V stage
  unsigned long long timeout_ns;
};

template <int kEsize_, int kDqk_, int kDv_, int kOut_>
struct KernelCfg {
  static constexpr int kEsize = kEsize_;  // bytes per input element (2 = bf16, 1 = e4m3)
  static constexpr int kDqk = kDqk_;      // head dim of Q and K as stored
  static constexpr int kDv = kDv_;        // head dim of V as stored (accumulator width)
  static constexpr int kOut = kOut_;
  static constexpr int kDout = kOut == kOutF32Split ? kDv / 2 : kDv;
  static constexpr int BM = 128;          // query rows per tile
  static constexpr int BN = 128;          // keys per K/V tile
  static constexpr int kTiles = 2;        // query tiles per work item
  // Warpgroups 0, 1: softmax and epilogue of query tile 0, 1.  Warpgroup 2:
  // warp 8 issues the MMAs, warp 9 the TMA loads, warps 10-11 only hold the
  // warpgroup's register budget.  Launch budget
  // 384 x 168 registers; the split below gives the softmax threads 216 and
  // warpgroup 2 72: 256 * 216 + 128 * 72 = 64512 = 384 * 168.
  static constexpr int kThreads = 384;
  static constexpr int kLaunchRegs = 168;
  static constexpr int kSoftmaxRegs = 216;
  static constexpr int kControlRegs = 72;
  static constexpr int kChunkBytes = BM * 128;          // one 128-byte-wide column chunk of a tile
  static constexpr int kChunkElems = 128 / kEsize;      // elements per 128-byte row segment
  static constexpr int kQChunks = kDqk * kEsize / 128;
  static constexpr int kVChunks = kDv * kEsize / 128;
  static constexpr int kQBytes = kQChunks * kChunkBytes;
  static constexpr int kKBytes = kQChunks * kChunkBytes;
  static constexpr int kVBytes = kVChunks * kChunkBytes;
  static constexpr int kStageBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr int kKStep = 32 / kEsize;            // K extent of one MMA (32 bytes)
  static constexpr int kOutEsize = kOut == kOutF32Split ? 4 : 2;  // bytes per O element
  static constexpr int kSmemMax = 232448;               // per-CTA opt-in limit on sm_100
  static constexpr int kBarBytes = 1024;
  static constexpr int kStagesFit = (kSmemMax - 1024 - kBarBytes - kTiles * kQBytes) / kStageBytes;
  // 32 KB stages (bf16, d = 128): 4 of the 5 that fit -- a fifth measured
  // 0.3-0.9% slower (K/V already land two steps ahead; the 32 KB it would
  // take stay with the L1 cache).
  static constexpr int kStages = kStagesFit > 8 ? 8 : (kStageBytes == 32768 && kStagesFit > 4 ? 4 : kStagesFit);
  static constexpr int kQOffset = 0;
  static constexpr int kStageOffset = kTiles * kQBytes;
  static constexpr int kBarOffset = kStageOffset + kStages * kStageBytes;
  static constexpr int kSmemBytes = 1024 + kBarOffset + kBarBytes;  // + alignment slack
  // Tensor memory columns (fp32 accumulators; 128 lanes = 128 rows).
  static constexpr int kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t s_col(int t) { return static_cast<uint32_t>(t * 128); }
  __host__ __device__ static constexpr uint32_t o_col(int t) { return static_cast<uint32_t>(256 + t * kDv); }
  // Lazy-rescale threshold (log2 units): probabilities stay below 2^kTau.
  // bf16 P keeps its relative precision at any magnitude and the fp32 sums
  // have ample range, so 16 costs nothing and makes moves of the reference
  // (each one a rescale of O) rare; e4m3 P saturates at 448, so 8.
  static constexpr float kTau = kEsize == 2 ? 16.0f : 8.0f;
  static constexpr float kPShift = 0.0f;                    // P stored as 2^kPShift * p

  static_assert(kDqk * kEsize % 128 == 0 && kDv * kEsize % 128 == 0, "head dims must fill 128-byte rows");
  static_assert(kStages >= 2, "need at least two K/V stages");
  static_assert(kDv <= 128 && kDv % 16 == 0, "accumulator width");
  static_assert(kSmemBytes <= kSmemMax, "shared memory budget");
  static_assert(256 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs, "register split over budget");
  static_assert(kLaunchRegs * kThreads <= 65536, "launch register budget");
};

struct SharedCtl {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t s_full[2];
  uint64_t p_half[2];  // P of keys 0..63 stored
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  uint64_t item_full[2];   // row ranges: the load warp has published work item item[s]
  uint64_t item_empty[2];  // every consumer has read item[s]
  int4 item[2];            // (b, h, hkv, qblk); qblk < 0: no more items
};
static_assert(sizeof(SharedCtl) <= 1024, "control block");

struct WorkItem {
  int b, h, hkv, qblk;
};

struct TileRange {
  int active;    // tile has at least one valid query row
  int q0;        // first query row
  int last_row;  // last valid query row
  int lo, hi;    // K/V tile range [lo, hi) this tile visits (empty: no row sees a key)
};

// A tile that takes part in the pipeline: it has rows and visits K/V tiles
// (without row ranges every tile with rows does).
template <bool kRanges>
__device__ __forceinline__ bool live(const TileRange& r) {
  if constexpr (kRanges) return r.active && r.lo < r.hi;
  return r.active;
}

// The i-th work item of this CTA.  Items are ranked heaviest first (or
// lightest first); CTAs take them in a boustrophedon order over the ranking
// (CTA c gets ranks c, 2G-1-c, 2G+c, 4G-1-c, ... for G CTAs), which keeps
// the per-CTA sums of causal work within a few percent of each other.
__device__ __forceinline__ int work_rank(int i) {
  const int G = gridDim.x;
  const int c = blockIdx.x;
  return i * G + ((i & 1) ? (G - 1 - c) : c);
}

// Ring position cursor over the K/V stages: stage index and mbarrier phase.
template <int kStages>
struct RingCursor {
  uint32_t stage = 0, phase = 0;
  __device__ __forceinline__ void advance() {
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

template <bool kRanges>
__device__ __forceinline__ WorkItem decode_work(int w, const FwdParams& p) {
  if constexpr (kRanges) {
    // Ranked by cost: the Hq items of the pair order[w / Hq] are consecutive.
    if (p.item_order != nullptr) {
      WorkItem wk;
      const int pr = w / p.Hq;
      wk.h = w - pr * p.Hq;
      const int pair = __ldg(p.item_order + pr);
      wk.b = pair / p.num_qblk;
      wk.qblk = pair - wk.b * p.num_qblk;
      wk.hkv = wk.h / p.group;
      return wk;
    }
  }
  const int bh_count = p.B * p.Hq;
  const int r = w / bh_count;
  const int bh = w - r * bh_count;
  WorkItem wk;
  wk.qblk = p.order == 0 ? (p.num_qblk - 1 - r) : r;
  wk.b = bh / p.Hq;
  wk.h = bh - wk.b * p.Hq;
  wk.hkv = wk.h / p.group;
  return wk;
}

// K/V tiles a query tile must visit: up to its last row when causal, from
// the first key inside the first row's window when windowed; with per-row
// key ranges, the span of its rows' visible keys (computed by
// row_range_tiles_kernel before the launch).
template <bool kRanges>
__device__ __forceinline__ TileRange tile_range(const WorkItem& wk, int t, const FwdParams& p) {
  TileRange r;
  r.q0 = wk.qblk * 256 + t * 128;
  r.active = r.q0 < p.N;
  r.last_row = min(r.q0 + 127, p.N - 1);
  if (!r.active) {
    r.lo = r.hi = 0;
    return r;
  }
  if constexpr (kRanges) {
    const int2 e = __ldg(p.tile_kv + static_cast<size_t>(wk.b) * p.num_qtiles + (r.q0 >> 7));
    r.lo = e.x;
    r.hi = e.y;
    return r;
  }
  const int hi_key = p.causal ? r.last_row + 1 : p.N;
  r.hi = (hi_key + 127) / 128;
  const int lo_key = p.window > 0 ? max(0, r.q0 - p.window + 1) : 0;
  r.lo = lo_key / 128;
  return r;
}

// Bounded wait on an mbarrier phase.  Returns false when the CTA is
// aborting (another thread gave up) or when this wait ran past the time
// limit (it then records the failure and raises the abort flag).
__device__ __forceinline__ bool wait_phase_slow(uint32_t a, uint32_t parity, SharedCtl* ctl, const FwdParams& p,
                                             int site, bool honor_abort) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 31u) == 0) {
      if (honor_abort && *reinterpret_cast<volatile int*>(&ctl->abort)) return false;
      if (globaltimer_ns() - t0 > p.timeout_ns || it > (1u << 28)) {
        atomicCAS(p.err, 0, (kErrTimeout << 16) | site);
        *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, SharedCtl* ctl, const FwdParams& p,
                                           int site, bool honor_abort) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  return wait_phase_slow(a, parity, ctl, p, site, honor_abort);
}

// The same for a whole warp that must stay converged (the MMA issuer): every
// lane polls, and the warp proceeds only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait_phase(uint64_t* bar, uint32_t parity, SharedCtl* ctl, const FwdParams& p,
                                                int site, bool honor_abort) {
  return __all_sync(0xFFFFFFFFu, wait_phase(bar, parity, ctl, p, site, honor_abort));
}

// ------------------------------------------------- work items (row ranges)
// The kernel with per-row key ranges hands work items from the load warp to
// the MMA warp and the eight softmax warps through two shared-memory slots:
// the load warp ranks and decodes the CTA's i-th item and publishes it in
// slot i % 2.  With a counter the item is the CTA's own block index first,
// then gridDim.x plus the counter's next value (a dynamic deal: a CTA takes
// more work when it is free, so unequal item costs still fill every SM);
// without one, the static deal's rank.  A rank >= num_work publishes
// qblk = -1 and ends every role's walk.  (The causal / window kernel, whose
// static deal balances, computes its items in every role and has no slots.)
template <bool kRanges>
__device__ __forceinline__ bool publish_item(int i, WorkItem& wk, const FwdParams& p, SharedCtl* ctl) {
  const int w = p.item_counter == nullptr ? work_rank(i)
                : i == 0                  ? static_cast<int>(blockIdx.x)
                                          : static_cast<int>(gridDim.x) + atomicAdd(p.item_counter, 1);
  if (w < p.num_work) {
    wk = decode_work<kRanges>(w, p);
  } else {
    wk.b = wk.h = wk.hkv = 0;
    wk.qblk = -1;
  }
  const int s = i & 1;
  if (!wait_phase(&ctl->item_empty[s], ((static_cast<uint32_t>(i) >> 1) & 1u) ^ 1u, ctl, p, kSiteItemEmpty, true))
    return false;
  ctl->item[s] = make_int4(wk.b, wk.h, wk.hkv, wk.qblk);  // ordered before the arrive by its memory clobber
  mbar_arrive(&ctl->item_full[s]);
  return true;
}

// Every lane of a consumer warp calls this; lane 0 frees the slot once the
// whole warp has read it.
__device__ __forceinline__ bool take_item(int i, WorkItem& wk, const FwdParams& p, SharedCtl* ctl, int lane) {
  const int s = i & 1;
  const bool ok = __all_sync(0xFFFFFFFFu, wait_phase(&ctl->item_full[s], (static_cast<uint32_t>(i) >> 1) & 1u, ctl,
                                                     p, kSiteItemFull, true));
  if (!ok) return false;
  const int4 v = ctl->item[s];  // read after the wait (its asm has a memory clobber)
  wk.b = v.x;
  wk.h = v.y;
  wk.hkv = v.z;
  wk.qblk = v.w;
  __syncwarp();
  if (lane == 0) mbar_arrive(&ctl->item_empty[s]);
  return true;
}

// ------------------------------------------------------------- TMA producer
template <class C, bool kRanges>
__device__ void producer_role(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                              const FwdParams& p, SharedCtl* ctl, uint8_t* smem) {
  const uint64_t pol_kv = l2_policy_evict_last();
  const uint64_t pol_q = l2_policy_evict_first();
  RingCursor<C::kStages> cur;
  uint32_t issued = 0;  // K/V positions started
  uint32_t q_iter[2] = {0, 0};
  int skip = p.skip_first_kv;
  uint32_t skipped_pos = 0xFFFFFFFFu;
  bool ok = true;
  for (int i = 0; ok; ++i) {
    WorkItem wk;
    if constexpr (kRanges) {
      ok = publish_item<kRanges>(i, wk, p, ctl);
      if (!ok || wk.qblk < 0) break;
    } else {
      const int w = work_rank(i);
      if (w >= p.num_work) break;
      wk = decode_work<kRanges>(w, p);
    }
    const TileRange r0 = tile_range<kRanges>(wk, 0, p);
    const TileRange r1 = tile_range<kRanges>(wk, 1, p);
    int lo, hi;  // K/V tiles of the item: the span of both tiles' ranges
    if constexpr (kRanges) {
      if (!live<true>(r0) && !live<true>(r1)) continue;
      lo = !live<true>(r1) ? r0.lo : (!live<true>(r0) ? r1.lo : min(r0.lo, r1.lo));
      hi = !live<true>(r1) ? r0.hi : (!live<true>(r0) ? r1.hi : max(r0.hi, r1.hi));
    } else {  // causal / window ranges grow with the query tile
      lo = r0.lo;
      hi = r1.active ? r1.hi : r0.hi;
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const TileRange& rt = t == 0 ? r0 : r1;
      if (!ok || !live<kRanges>(rt)) continue;
      ok = wait_phase(&ctl->q_empty[t], (q_iter[t] & 1u) ^ 1u, ctl, p, kSiteProdQEmpty, true);
      if (!ok) break;
      ++q_iter[t];
      mbar_arrive_expect_tx(&ctl->q_full[t], C::kQBytes);
      uint8_t* dst = smem + C::kQOffset + t * C::kQBytes;
#pragma unroll
      for (int kc = 0; kc < C::kQChunks; ++kc)
        tma_load_4d(dst + kc * C::kChunkBytes, tm_q, &ctl->q_full[t], kc * C::kChunkElems, wk.h, rt.q0, wk.b,
                    pol_q);
    }
    for (int j = lo; j < hi && ok; ++j) {
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        if (!ok) break;
        ok = wait_phase(&ctl->empty[cur.stage], cur.phase ^ 1u, ctl, p, kSiteProdKvEmpty, true);
        if (!ok) break;
        uint64_t* full = &ctl->full[cur.stage];
        uint8_t* dst = smem + C::kStageOffset + cur.stage * C::kStageBytes;
        if (skip) {  // test hook: leave this stage unfilled
          skip = 0;
          skipped_pos = issued;
        } else if (which == 0) {
          mbar_arrive_expect_tx(full, C::kKBytes);
#pragma unroll
          for (int kc = 0; kc < C::kQChunks; ++kc)
            tma_load_4d(dst + kc * C::kChunkBytes, tm_k, full, kc * C::kChunkElems, wk.hkv, j * 128, wk.b, pol_kv);
        } else {
          mbar_arrive_expect_tx(full, C::kVBytes);
#pragma unroll
          for (int kc = 0; kc < C::kVChunks; ++kc)
            tma_load_4d(dst + kc * C::kChunkBytes, tm_v, full, kc * C::kChunkElems, wk.hkv, j * 128, wk.b, pol_kv);
        }
        ++issued;
        cur.advance();
      }
    }
  }
  if (!ok) {
    // Unwinding: wait (bounded, ignoring the abort flag) for every copy this
    // thread started, so none lands after the CTA has exited.  Only the last
    // kStages positions can still be in flight; position P sits in stage
    // P % kStages with phase (P / kStages) & 1.
    for (uint32_t P = issued > C::kStages ? issued - C::kStages : 0; P < issued; ++P) {
      if (P == skipped_pos) continue;
      wait_phase(&ctl->full[P % C::kStages], (P / C::kStages) & 1u, ctl, p, kSiteProdDrain, false);
    }
    for (int t = 0; t < 2; ++t)
      if (q_iter[t] > 0) wait_phase(&ctl->q_full[t], (q_iter[t] - 1) & 1u, ctl, p, kSiteProdDrain, false);
  }
}

// ------------------------------------------------------------ MMA issuer
// One converged warp runs this role: every lane follows the same control
// flow and waits, and elect.sync inside each MMA and commit picks lane 0
// to issue.
// O += P V over keys [K0 * kKStep, K1 * kKStep) of a tile: one MMA per
// kKStep keys, A = P from tensor memory (8 columns per step), B = V
// (MN-major, kKStep rows per step).
template <class C, int K, int K1>
__device__ __forceinline__ void mma_pv(uint32_t d_o, uint32_t a_p, uint32_t v_lo, uint32_t idesc, uint32_t acc0) {
  if constexpr (K < K1) {
    constexpr uint32_t kOff = K * (C::kKStep * 128 / 16);
    if constexpr (C::kEsize == 2)
      mma_f16_ts_lo<kOff>(d_o, a_p + K * 8, v_lo, idesc, K == 0 ? acc0 : 1u);
    else
      mma_f8_ts_lo<kOff>(d_o, a_p + K * 8, v_lo, idesc, K == 0 ? acc0 : 1u);
    mma_pv<C, K + 1, K1>(d_o, a_p, v_lo, idesc, acc0);
  }
}

// S = Q K^T over the head dimension: 4 MMAs (32 bytes of K each) per
// 128-byte chunk, both operands K-major.
template <class C, int I>
__device__ __forceinline__ void mma_qk(uint32_t d_s, uint32_t q_lo, uint32_t k_lo, uint32_t idesc) {
  if constexpr (I < C::kQChunks * 4) {
    constexpr uint32_t kOff = (I / 4) * (C::kChunkBytes >> 4) + (I % 4) * 2;
    if constexpr (C::kEsize == 2)
      mma_f16_ss_lo<kOff, kOff>(d_s, q_lo, k_lo, idesc, I == 0 ? 0u : 1u);
    else
      mma_f8_ss_lo<kOff, kOff>(d_s, q_lo, k_lo, idesc, I == 0 ? 0u : 1u);
    mma_qk<C, I + 1>(d_s, q_lo, k_lo, idesc);
  }
}

// The MMA issuer.  Per K/V step j of a work item it issues, in order:
//   O_0 += P_0(j-1) V(j-1)  in two halves (keys 0-63 once the softmax has
//                           published them, then keys 64-127),
//   S_0 = Q_0 K(j)^T,
//   O_1 += P_1(j-1) V(j-1)  in two halves,  then releases V(j-1),
//   S_1 = Q_1 K(j)^T,                         then releases K(j).
// S_T(j) overwrites the columns that held P_T(j-1), so it must follow
// O_T += P_T(j-1) V(j-1) (the tensor core runs one thread's MMAs in order).
// An mbarrier test costs the warp about 150 cycles even when the phase is
// complete, so none sits between a tile's P and its next S: both ring
// stages of the step (V(j-1), K(j)), which land well ahead, are checked at
// the start of the step, and each P is waited for right before its
// product.  Waits on P and on O being free (tensor memory written or read
// by other threads) are followed by tcgen05.fence::after_thread_sync; waits
// on copies into shared memory need none.
template <class C, bool kRanges>
__device__ void mma_role(const FwdParams& p, SharedCtl* ctl, uint8_t* smem, uint32_t tmem) {
  constexpr uint32_t kStageUnits = C::kStageBytes >> 4;
  constexpr uint32_t kFmt = C::kEsize == 2 ? 1u : 0u;  // bf16 : e4m3
  constexpr uint32_t kIdO = make_idesc(kFmt, 128, C::kDv, false, true);
  constexpr uint32_t kIdS = make_idesc(kFmt, 128, 128, false, false);
  constexpr int kHalf = C::BN / C::kKStep / 2;  // MMAs per half of a P V product
  const uint32_t q_lo[2] = {sw128_desc_lo(smem_u32(smem + C::kQOffset), 16),
                            sw128_desc_lo(smem_u32(smem + C::kQOffset + C::kQBytes), 16)};
  const uint32_t k_lo_base = sw128_desc_lo(smem_u32(smem + C::kStageOffset), 16);
  const uint32_t v_lo_base = sw128_desc_lo(smem_u32(smem + C::kStageOffset), C::kChunkBytes);
  RingCursor<C::kStages> cur;
  uint32_t q_phase[2] = {0, 0}, p_phase[2] = {0, 0}, o_iter[2] = {0, 0};
  bool ok = true;
  for (int i = 0; ok; ++i) {
    WorkItem wk;
    if constexpr (kRanges) {
      ok = take_item(i, wk, p, ctl, static_cast<int>(threadIdx.x & 31));
      if (!ok || wk.qblk < 0) break;
    } else {
      const int w = work_rank(i);
      if (w >= p.num_work) break;
      wk = decode_work<kRanges>(w, p);
    }
    const TileRange r[2] = {tile_range<kRanges>(wk, 0, p), tile_range<kRanges>(wk, 1, p)};
    const bool live0 = live<kRanges>(r[0]), live1 = live<kRanges>(r[1]);
    int lo, hi;
    if constexpr (kRanges) {
      if (!live0 && !live1) continue;
      lo = !live1 ? r[0].lo : (!live0 ? r[1].lo : min(r[0].lo, r[1].lo));
      hi = !live1 ? r[0].hi : (!live0 ? r[1].hi : max(r[0].hi, r[1].hi));
    } else {
      lo = r[0].lo;
      hi = r[1].active ? r[1].hi : r[0].hi;
    }
    if (live0) {
      ok = warp_wait_phase(&ctl->q_full[0], q_phase[0], ctl, p, kSiteMmaQFull, true);
      q_phase[0] ^= 1u;
    }
    if (ok && live1) {
      ok = warp_wait_phase(&ctl->q_full[1], q_phase[1], ctl, p, kSiteMmaQFull, true);
      q_phase[1] ^= 1u;
    }
    if (!ok) break;
    for (int j = lo; j <= hi; ++j) {
      // The step's ring stages: V(j-1), then K(j).
      uint32_t v_stage = 0, k_stage = 0;
      if (j > lo) {
        ok = warp_wait_phase(&ctl->full[cur.stage], cur.phase, ctl, p, kSiteMmaKvFull, true);
        if (!ok) break;
        v_stage = cur.stage;
        cur.advance();
      }
      if (j < hi) {
        ok = warp_wait_phase(&ctl->full[cur.stage], cur.phase, ctl, p, kSiteMmaKvFull, true);
        if (!ok) break;
        k_stage = cur.stage;
        cur.advance();
      }
      const uint32_t v_lo = v_lo_base + v_stage * kStageUnits;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const TileRange& rt = r[t];
        if (rt.active && j - 1 >= rt.lo && j - 1 < rt.hi) {  // O_t += P_t(j-1) V(j-1)
          const uint32_t d_o = tmem + C::o_col(t);
          const uint32_t a_p = tmem + C::s_col(t);
          ok = warp_wait_phase(&ctl->p_half[t], p_phase[t], ctl, p, kSiteMmaPFull, true);
          if (ok && j - 1 == rt.lo) {  // first product of this item: the previous epilogue must be done with O_t
            ok = warp_wait_phase(&ctl->o_empty[t], (o_iter[t] & 1u) ^ 1u, ctl, p, kSiteMmaOEmpty, true);
            ++o_iter[t];
          }
          if (!ok) break;
          tc_fence_after();
          mma_pv<C, 0, kHalf>(d_o, a_p, v_lo, kIdO, (j - 1 > rt.lo) ? 1u : 0u);
          ok = warp_wait_phase(&ctl->p_full[t], p_phase[t], ctl, p, kSiteMmaPFull, true);
          if (!ok) break;
          p_phase[t] ^= 1u;
          tc_fence_after();
          mma_pv<C, kHalf, 2 * kHalf>(d_o, a_p, v_lo, kIdO, 1u);
          if (j - 1 == rt.hi - 1) mma_commit_elect(&ctl->o_full[t]);
        }
        if (t == 1 && j > lo) mma_commit_elect(&ctl->empty[v_stage]);
        if (rt.active && j >= rt.lo && j < rt.hi) {  // S_t = Q_t K(j)^T
          mma_qk<C, 0>(tmem + C::s_col(t), q_lo[t], k_lo_base + k_stage * kStageUnits, kIdS);
          mma_commit_elect(&ctl->s_full[t]);
          if (j == rt.hi - 1) mma_commit_elect(&ctl->q_empty[t]);
        }
      }
      if (!ok) break;
      if (j < hi) mma_commit_elect(&ctl->empty[k_stage]);
    }
  }
  // Every product issued so far must finish before tensor memory is freed.
  mma_commit_elect(&ctl->drain);
  warp_wait_phase(&ctl->drain, 0, ctl, p, kSiteMmaDrain, false);
}

// ------------------------------------------------------------- softmax
// Packed P words per row: bf16 pairs or e4m3 quads of 128 probabilities.
template <class C>
struct PWords {
  static constexpr int kN = C::kEsize == 2 ? 64 : 32;
};

// Maximum of 128 values as a tree of three-input maxima (depth 5).
__device__ __forceinline__ float max128(const float (&x)[128]) {
  float a[43];
#pragma unroll
  for (int i = 0; i < 42; ++i) a[i] = fmax3(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
  a[42] = fmaxf(x[126], x[127]);
  float b[15];
#pragma unroll
  for (int i = 0; i < 14; ++i) b[i] = fmax3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
  b[14] = a[42];
  float c[5];
#pragma unroll
  for (int i = 0; i < 5; ++i) c[i] = fmax3(b[3 * i], b[3 * i + 1], b[3 * i + 2]);
  return fmaxf(fmax3(c[0], c[1], c[2]), fmaxf(c[3], c[4]));
}

// One pair of probabilities p = 2^(s cs - m) (the argument as one paired
// FMA), added to the paired row sums and packed into P words: bf16 pairs,
// or e4m3 quads (the first pair of a quad waits in e_prev).  I is the pair
// index in the row (a constant once the callers' loops are unrolled).
template <class C>
__device__ __forceinline__ void prob_pair(int I, const float (&x)[128], uint64_t cs2, uint64_t nr2,
                                          uint64_t (&acc)[2], uint32_t (&pk)[16], float (&e_prev)[2]) {
  const uint64_t y = f2_fma(f2_pack(x[2 * I], x[2 * I + 1]), cs2, nr2);
  float y0, y1;
  f2_unpack(y, y0, y1);
  const float e0 = ex2_approx(y0);
  const float e1 = ex2_approx(y1);
  const uint64_t e01 = f2_pack(e0, e1);
  acc[I & 1] = I < 2 ? e01 : f2_add(acc[I & 1], e01);
  if (C::kEsize == 2) {
    pk[I & 15] = pack_bf16x2(e0, e1);
  } else if (I & 1) {
    pk[(I & 15) >> 1] = pack_e4m3x4(e_prev[0], e_prev[1], e0, e1);
  } else {
    e_prev[0] = e0;
    e_prev[1] = e1;
  }
}

// Keys [32 Q, 32 Q + 32) of the row (16 pairs), their P words stored over
// the first columns of S (already read).  With kMax the same loop takes the
// row maximum of all 128 scores for the first two quarters (two chains of
// three-input maxima, interleaved with the exponentials and off their
// critical path).
template <class C, int Q, bool kMax>
__device__ __forceinline__ void prob_quarter(const float (&x)[128], uint64_t cs2, uint64_t nr2, uint64_t (&acc)[2],
                                             float (&e_prev)[2], float& mA, float& mB, uint32_t tS) {
  uint32_t pk[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int I = 16 * Q + k;
    if (kMax) {
      mA = fmax3(mA, x[2 * I], x[2 * I + 1]);
      mB = fmax3(mB, x[64 + 2 * I], x[65 + 2 * I]);
    }
    prob_pair<C>(I, x, cs2, nr2, acc, pk, e_prev);
  }
  if constexpr (C::kEsize == 2)
    tmem_st16(tS + 16 * Q, pk);
  else
    tmem_st8(tS + 8 * Q, pk);
}

template <class C, bool kRanges>
__device__ void softmax_role(int t, const FwdParams& p, SharedCtl* ctl, uint32_t tmem, int warp, int lane) {
  const int quad = warp & 3;
  const int row_in_tile = quad * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
  const uint32_t tS = tmem + lane_off + C::s_col(t);
  const uint32_t tO = tmem + lane_off + C::o_col(t);
  uint32_t s_phase = 0, o_phase = 0;

  for (int i = 0;; ++i) {
    WorkItem wk;
    if constexpr (kRanges) {
      if (!take_item(i, wk, p, ctl, lane)) return;
      if (wk.qblk < 0) break;
    } else {
      const int w = work_rank(i);
      if (w >= p.num_work) break;
      wk = decode_work<kRanges>(w, p);
    }
    const TileRange r = tile_range<kRanges>(wk, t, p);
    if (!r.active) continue;
    const int qrow = r.q0 + row_in_tile;
    if (kRanges && r.lo >= r.hi) {  // no row of this tile sees a key: O = 0, LSE = -inf
      if (qrow < p.N) {
        const size_t row_elem = ((static_cast<size_t>(wk.b) * p.N + qrow) * p.Hq + wk.h) * C::kDout;
        constexpr int kVec = C::kDout * C::kOutEsize / 16;
        uint4* dst = C::kOut == kOutBf16 ? reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) + row_elem)
                                         : reinterpret_cast<uint4*>(reinterpret_cast<float*>(p.o) + row_elem);
#pragma unroll 4
        for (int i = 0; i < kVec; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
        p.lse[(static_cast<size_t>(wk.b) * p.Hq + wk.h) * p.N + qrow] = -CUDART_INF_F;
      }
      continue;
    }
    float cs = p.scale_log2;
    float out_mult = 1.0f;
    if (C::kEsize == 1) {
      cs *= __ldg(p.q_scale + wk.h) * __ldg(p.k_scale + wk.hkv);
      out_mult = __ldg(p.v_scale + wk.hkv);
    }
    // Key columns this row may see: [key_lo, key_hi).
    int key_hi = p.causal ? min(p.N, qrow + 1) : p.N;
    int key_lo = p.window > 0 ? max(0, qrow - p.window + 1) : 0;
    if (kRanges && qrow < p.N) {
      const size_t ix = static_cast<size_t>(wk.b) * p.N + qrow;
      key_lo = max(key_lo, __ldg(p.key_lo + ix));
      key_hi = min(key_hi, __ldg(p.key_hi + ix));
    }
    const uint64_t cs2 = f2_pack(cs, cs);

    // m_used: the reference maximum of the row's probabilities (log2 units),
    // moved only when a tile's maximum exceeds it by more than kTau.
    float m_used = -CUDART_INF_F;
    float l = 0.0f;
    for (int j = r.lo; j < r.hi; ++j) {
      bool ok = wait_phase(&ctl->s_full[t], s_phase, ctl, p, kSiteSoftSFull, true);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) return;
      s_phase ^= 1u;
      tc_fence_after();

      // This thread's row of S: 128 fp32 scores, one tensor-memory read.
      float x[128];
      {
        uint32_t* raw = reinterpret_cast<uint32_t*>(x);
        tmem_ld32p(tS + 0, raw);
        tmem_ld32p(tS + 32, raw + 32);
        tmem_ld32p(tS + 64, raw + 64);
        tmem_ld32p(tS + 96, raw + 96);
        tmem_wait_ld();
      }
      const int kbase = j * 128;
      // Mask when some row sees only part of the tile (with row ranges: some
      // row of this warp).
      const bool need_mask = kRanges ? __any_sync(0xFFFFFFFFu, kbase < key_lo || kbase + 128 > key_hi)
                                     : (kbase + 128 > p.N) || (p.causal && kbase + 127 > r.q0) ||
                                           (p.window > 0 && kbase <= r.last_row - p.window);
      if (need_mask) {
        const int vlo = key_lo - kbase;  // visible columns [vlo, vhi) of this tile
        const int vhi = key_hi - kbase;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c < vlo || c >= vhi) x[c] = -CUDART_INF_F;
      }
      // The row's first visible keys set the reference before any
      // exponential.  Later tiles start their exponentials at once against
      // the reference in use while the tile's maximum is taken alongside;
      // only a maximum above the reference by more than kTau (rare once a
      // row's first tiles are done) moves it -- l and O are rescaled and the
      // first half is computed again, so the probabilities are exactly those
      // of moving the reference first.
      if (m_used == -CUDART_INF_F) m_used = max128(x) * cs;

      uint64_t acc[2];
      float e_prev[2];
#pragma unroll 1
      for (;;) {
        const float neg_ref = -((m_used == -CUDART_INF_F) ? 0.0f : m_used) + C::kPShift;
        const uint64_t nr2 = f2_pack(neg_ref, neg_ref);
        float mA = -CUDART_INF_F, mB = -CUDART_INF_F;
        prob_quarter<C, 0, true>(x, cs2, nr2, acc, e_prev, mA, mB, tS);
        prob_quarter<C, 1, true>(x, cs2, nr2, acc, e_prev, mA, mB, tS);
        const float m_tile = fmaxf(mA, mB) * cs;
        const bool up = m_tile > m_used + C::kTau;  // false while m_used is -inf: m_tile is then -inf too
        if (!__any_sync(0xFFFFFFFFu, up)) {
          // publish P of keys 0..63: the first half of P V can start
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->p_half[t]);
          // keys 64..127 against the same reference
          prob_quarter<C, 2, false>(x, cs2, nr2, acc, e_prev, mA, mB, tS);
          prob_quarter<C, 3, false>(x, cs2, nr2, acc, e_prev, mA, mB, tS);
          break;
        }
        float alpha = 1.0f;
        bool rescale_o = false;
        if (up) {
          alpha = ex2_approx(m_used - m_tile);
          rescale_o = j > r.lo;  // O holds products of earlier tiles (all finished: S(j) follows them)
          l *= alpha;
          m_used = m_tile;
        }
        if (__any_sync(0xFFFFFFFFu, rescale_o)) {
          const float f = rescale_o ? alpha : 1.0f;
#pragma unroll 1
          for (int cc = 0; cc < C::kDv; cc += 32) {
            uint32_t ov[32];
            tmem_ld32(tO + cc, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
            tmem_st32(tO + cc, ov);
          }
        }
      }
      {
        const uint64_t s2 = f2_add(acc[0], acc[1]);
        float s0, s1;
        f2_unpack(s2, s0, s1);
        l += s0 + s1;
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[t]);
    }

    // Epilogue: O = acc / l, LSE = ln 2 * (m + log2 l).  The row of O is read
    // from tensor memory at once and its columns are released before the
    // stores, so the next item's first P V can start meanwhile.
    {
      bool ok = wait_phase(&ctl->o_full[t], o_phase, ctl, p, kSiteSoftOFull, true);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) return;
      o_phase ^= 1u;
      tc_fence_after();
      uint32_t ov[C::kDv];
#pragma unroll
      for (int cc = 0; cc < C::kDv; cc += 32) tmem_ld32p(tO + cc, ov + cc);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->o_empty[t]);
      const float inv_l = l > 0.0f ? out_mult / l : 0.0f;
      if (qrow < p.N) {
        const size_t row_elem = ((static_cast<size_t>(wk.b) * p.N + qrow) * p.Hq + wk.h) * C::kDout;
        if constexpr (C::kOut == kOutBf16) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) + row_elem);
#pragma unroll
          for (int g = 0; g < C::kDv / 8; ++g) {  // 8 bf16 columns per 16-byte store
            const int c = g * 8;
            dst[g] = make_uint4(pack_bf16x2(__uint_as_float(ov[c + 0]) * inv_l, __uint_as_float(ov[c + 1]) * inv_l),
                                pack_bf16x2(__uint_as_float(ov[c + 2]) * inv_l, __uint_as_float(ov[c + 3]) * inv_l),
                                pack_bf16x2(__uint_as_float(ov[c + 4]) * inv_l, __uint_as_float(ov[c + 5]) * inv_l),
                                pack_bf16x2(__uint_as_float(ov[c + 6]) * inv_l, __uint_as_float(ov[c + 7]) * inv_l));
          }
        } else {  // fp32: the high and low halves of P V' summed, 4 columns per 16-byte store
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.o) + row_elem);
#pragma unroll
          for (int g = 0; g < C::kDout / 4; ++g) {
            const int c = g * 4;
            float4 v;
            v.x = (__uint_as_float(ov[c + 0]) + __uint_as_float(ov[C::kDout + c + 0])) * inv_l;
            v.y = (__uint_as_float(ov[c + 1]) + __uint_as_float(ov[C::kDout + c + 1])) * inv_l;
            v.z = (__uint_as_float(ov[c + 2]) + __uint_as_float(ov[C::kDout + c + 2])) * inv_l;
            v.w = (__uint_as_float(ov[c + 3]) + __uint_as_float(ov[C::kDout + c + 3])) * inv_l;
            dst[g] = v;
          }
        }
        const float lse = l > 0.0f ? (m_used + __log2f(l) - C::kPShift) * 0.69314718055994531f
                                   : -CUDART_INF_F;
        p.lse[(static_cast<size_t>(wk.b) * p.Hq + wk.h) * p.N + qrow] = lse;
      }
    }
  }
}

// --------------------------------------------- per-tile K/V ranges (masks)
// One block of 128 threads per (batch, 128-row query tile): thread r takes
// row q0 + r's visible keys [max(key_lo, 0, window start), min(key_hi, N,
// row + 1 when causal)) and the block reduces them to the span of K/V tiles
// [lo / 128, ceil(hi / 128)) that covers every non-empty row; (0, 0) when
// no row of the tile sees a key.  It also zeroes the attention kernel's
// item counter (dynamic deal), when there is one.
__global__ void __launch_bounds__(128) row_range_tiles_kernel(const int* __restrict__ key_lo,
                                                              const int* __restrict__ key_hi, int2* tile_kv,
                                                              int* item_counter, int N, int num_qtiles, int causal,
                                                              int window) {
  __shared__ int s_lo[4], s_hi[4];
  if (item_counter != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *item_counter = 0;
  const int b = blockIdx.x / num_qtiles;
  const int qt = blockIdx.x - b * num_qtiles;
  const int row = qt * 128 + static_cast<int>(threadIdx.x);
  int lo = INT_MAX, hi = INT_MIN;
  if (row < N) {
    const size_t ix = static_cast<size_t>(b) * N + row;
    int a = max(0, __ldg(key_lo + ix));
    int e = min(N, __ldg(key_hi + ix));
    if (window > 0) a = max(a, row - window + 1);
    if (causal) e = min(e, row + 1);
    if (a < e) {
      lo = a;
      hi = e;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
  }
  if ((threadIdx.x & 31) == 0) {
    s_lo[threadIdx.x >> 5] = lo;
    s_hi[threadIdx.x >> 5] = hi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    lo = min(min(s_lo[0], s_lo[1]), min(s_lo[2], s_lo[3]));
    hi = max(max(s_hi[0], s_hi[1]), max(s_hi[2], s_hi[3]));
    tile_kv[blockIdx.x] = lo < hi ? make_int2(lo / 128, (hi + 127) / 128) : make_int2(0, 0);
  }
}

// With per-row key ranges the cost of a work item depends on the data, so
// the (batch, query block) pairs are ranked by the number of K/V tiles their
// two query tiles visit, most first, before the launch: the kernel's
// boustrophedon deal over a descending ranking then gives every CTA about
// the same work.  One block, a bitonic sort of (cost, index) keys in shared
// memory (kOrderMaxPairs at most; beyond that the host passes no order and
// the default ranking is used).  Ties keep index order, so the ranking and
// the results do not vary from run to run.
constexpr int kOrderMaxPairs = 16384;

__global__ void __launch_bounds__(1024) order_items_kernel(const int2* __restrict__ tile_kv, int* order, int n,
                                                           int num_qblk, int num_qtiles, int pow2) {
  extern __shared__ unsigned long long keys[];
  for (int i = threadIdx.x; i < pow2; i += blockDim.x) {
    unsigned long long key = ~0ull;  // padding sorts last
    if (i < n) {
      const int b = i / num_qblk;
      const int qb = i - b * num_qblk;
      const int2 t0 = tile_kv[static_cast<size_t>(b) * num_qtiles + 2 * qb];
      int cost = max(0, t0.y - t0.x);
      if (2 * qb + 1 < num_qtiles) {
        const int2 t1 = tile_kv[static_cast<size_t>(b) * num_qtiles + 2 * qb + 1];
        cost += max(0, t1.y - t1.x);
      }
      key = (static_cast<unsigned long long>(0x7FFFFFFF - cost) << 32) | static_cast<unsigned>(i);
    }
    keys[i] = key;
  }
  __syncthreads();
  for (int k = 2; k <= pow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < pow2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = keys[i], c = keys[ixj];
          const bool ascending = (i & k) == 0;
          if (ascending ? (a > c) : (a < c)) {
            keys[i] = c;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) order[i] = static_cast<int>(keys[i] & 0xFFFFFFFFull);
}

// ------------------------------------------------------------- the kernel
template <class C, bool kRanges>
__global__ void __launch_bounds__(C::kThreads, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + C::kBarOffset);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl->q_full[t], 1);
      mbar_init(&ctl->q_empty[t], 1);
      mbar_init(&ctl->s_full[t], 1);
      mbar_init(&ctl->p_half[t], 4);
      mbar_init(&ctl->p_full[t], 4);
      mbar_init(&ctl->o_full[t], 1);
      mbar_init(&ctl->o_empty[t], 4);
    }
    mbar_init(&ctl->drain, 1);
    if constexpr (kRanges) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(&ctl->item_full[s], 1);
        mbar_init(&ctl->item_empty[s], 9);  // the MMA warp and the eight softmax warps
      }
    }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(&ctl->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp < 8) {
    regs_increase<C::kSoftmaxRegs>();
    softmax_role<C, kRanges>(warp >> 2, p, ctl, tmem, warp, lane);
  } else {
    regs_decrease<C::kControlRegs>();
    if (warp == 8) {
      mma_role<C, kRanges>(p, ctl, smem, tmem);
      __syncwarp();
    } else if (warp == 9) {
      if (lane == 0) producer_role<C, kRanges>(&tm_q, &tm_k, &tm_v, p, ctl, smem);
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace ea
