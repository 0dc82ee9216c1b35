// attn_bwd_kernel.cuh -- exact attention backward for sm_100a.
//
// Given the forward's inputs Q, K, V, its outputs O and LSE, and the
// upstream gradient dO, computes dQ, dK, dV without ever storing the N x N
// probabilities: S and P are recomputed tile by tile from Q, K and the saved
// LSE ("Flash Attention" concept note (heepie.pages.dev), "Tiling" -- more
// FLOPs through recomputation, far fewer HBM accesses -- and "FLOP != speed").
// The gradient formulas are the chain rule of the forward definition:
//     P = exp(S - LSE),  dV = P^T dO,  dP = dO V^T,  D = rowsum(dO o O),
//     dS = P o (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels:
//   * bwd_prep_kernel: per query row, (-LSE log2 e, D) -- HBM-bound, one pass
//     over O and dO.
//   * attn_bwd_dkdv_sm100: one persistent CTA per SM; a work item is (batch,
//     key/value head, 128-key tile).  K and V stay in shared memory while the
//     item walks every query tile of every query head of its group that sees
//     the key tile.  Per step the tensor core computes S^T = K Q^T and
//     dP^T = V dO^T into tensor memory; two compute warpgroups (one thread
//     per key row, half of the query columns each) form P^T and dS^T and
//     write them back over S^T and dP^T as bf16; the tensor core accumulates dV += P^T dO and dK += dS^T Q in
//     tensor memory (512 columns: S^T, dP^T, dV, dK).  The group's query
//     heads accumulate into the same dK, dV: no atomics.
//   * attn_bwd_dq_sm100: a work item is (batch, query head, 128-row query
//     tile); Q and dO stay in shared memory while the item walks the K/V
//     tiles it sees: S = Q K^T and dP = dO V^T into tensor memory, two
//     compute warpgroups (one thread per query row, half of the key columns
//     each) form dS over dP, the
//     tensor core accumulates dQ += dS K.  Recomputing S and dP here instead
//     of adding dQ from the first kernel with atomics keeps the results
//     deterministic.
// Each MMA pattern is one of the forward's: K-major products of two 128-row
// shared-memory tiles, and products whose A operand is a bf16 matrix in
// tensor memory and whose B operand is an MN-major 128-row tile.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "attn_fwd_kernel.cuh"
#include "sm100_ptx.cuh"

namespace ea {

struct BwdParams {
  const float2* stats;  // [B, Hq, N]: (-LSE * log2 e, or -inf for rows past N / with no key; D)
  void* dq;             // [B, N, Hq, d] bf16
  void* dk;             // [B, N, Hkv, d] bf16
  void* dv;             // [B, N, Hkv, d] bf16
  int* err;             // device error word
  const int* key_lo;    // [B, N] per-row key ranges (range variant only)
  const int* key_hi;
  const int2* tile_kv;  // [B, num_tiles]: K/V tiles [x, y) of each query tile (range variant)
  const int2* tile_q;   // [B, num_tiles]: query tiles [x, y) that see each key tile (range variant)
  int B, Hq, Hkv, N, group;
  int causal, window;
  float scale_log2;     // scale * log2(e)
  float scale;
  int num_tiles;        // ceil(N / 128)
  int num_work;
  int* item_counter;    // range variant: this launch's dynamic-deal counter (zeroed before the launch), or null
  unsigned long long timeout_ns;
};

enum : int {
  kSiteBwdProdKv = 20,
  kSiteBwdProdStage = 21,
  kSiteBwdMmaKv = 22,
  kSiteBwdMmaStage = 23,
  kSiteBwdMmaP = 24,
  kSiteBwdMmaDs = 25,
  kSiteBwdMmaAcc = 26,
  kSiteBwdMmaSFree = 27,
  kSiteBwdCompS = 28,
  kSiteBwdCompDp = 29,
  kSiteBwdCompAcc = 30,
  kSiteBwdDrain = 31,
  kSiteBwdCompStats = 32,
  kSiteBwdItemFull = 33,   // range variant: a consumer waiting for the next work item
  kSiteBwdItemEmpty = 34   // range variant: the load warp waiting for a free item slot
};

// ------------------------------------------------------------ preprocessing
// stats[b, h, i] = (-LSE[b, h, i] * log2 e, sum_c dO[b, i, h, c] O[b, i, h, c]);
// a row with LSE = -inf (no visible key) gets -inf, so its probabilities
// recompute to 0.  Sixteen threads per row, eight elements each.
template <int kD>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse, float2* stats, int B, int Hq,
                                                       int N) {
  constexpr int kLanesPerRow = kD / 8;
  const long long rows = static_cast<long long>(B) * N * Hq;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = t / kLanesPerRow;  // (b, i, h) in O's layout
  const int part = static_cast<int>(t % kLanesPerRow);
  float acc = 0.0f;
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * kD + part * 8);
    const uint4 g = *reinterpret_cast<const uint4*>(dout + row * kD + part * 8);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
    const uint32_t gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(av[i] << 16), __uint_as_float(gv[i] << 16), acc);
      acc = fmaf(__uint_as_float(av[i] & 0xFFFF0000u), __uint_as_float(gv[i] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (row < rows && part == 0) {
    const int h = static_cast<int>(row % Hq);
    const long long bi = row / Hq;
    const int i = static_cast<int>(bi % N);
    const int b = static_cast<int>(bi / N);
    const size_t s = (static_cast<size_t>(b) * Hq + h) * N + i;
    const float l = lse[s];
    stats[s] = make_float2(l == -CUDART_INF_F ? -CUDART_INF_F : -l * 1.4426950408889634f, acc);
  }
}

// ---------------------------------------------------------------- control
struct BwdCtl {
  uint64_t kv_full, kv_empty;          // dK/dV kernel: the item's K, V.  dQ kernel: the item's Q, dO
  uint64_t st_full[2], st_empty[2];    // per-step operand stages
  uint64_t s_full, dp_full;            // tensor core -> compute
  uint64_t s_free;                     // compute has read S (dQ kernel)
  uint64_t p_full, ds_full;            // compute -> tensor core
  uint64_t acc_full, acc_empty;        // accumulators ready / read
  uint64_t stats_ready[2];             // dK/dV kernel: a step's query-row stats are in shared memory
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  uint64_t item_full[2], item_empty[2];  // range variant: work-item slots (load warp -> other roles)
  int item[2];
};
static_assert(sizeof(BwdCtl) <= 1024, "control block");

__device__ __forceinline__ bool bwd_wait_slow(uint32_t a, uint32_t parity, BwdCtl* ctl, const BwdParams& p, int site,
                                           bool honor_abort) {
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

__device__ __forceinline__ bool bwd_wait(uint64_t* bar, uint32_t parity, BwdCtl* ctl, const BwdParams& p, int site,
                                         bool honor_abort = true) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  return bwd_wait_slow(a, parity, ctl, p, site, honor_abort);
}

// Range variant: the load warp takes the CTA's i-th work item and publishes
// its rank in slot i % 2 for the MMA warp and the eight compute warps (as
// the forward's range kernel does).  With a counter the rank is the CTA's
// own block index first, then gridDim.x plus the counter's next value (a
// dynamic deal: per-row key ranges give items unequal costs in no order);
// without one, the static deal's rank.  A rank >= num_work ends the walk.
__device__ __forceinline__ bool bwd_publish_rank(int i, int& w, const BwdParams& p, BwdCtl* ctl) {
  w = p.item_counter == nullptr ? work_rank(i)
      : i == 0                  ? static_cast<int>(blockIdx.x)
                                : static_cast<int>(gridDim.x) + atomicAdd(p.item_counter, 1);
  const int s = i & 1;
  if (!bwd_wait(&ctl->item_empty[s], ((static_cast<uint32_t>(i) >> 1) & 1u) ^ 1u, ctl, p, kSiteBwdItemEmpty))
    return false;
  ctl->item[s] = w;  // ordered before the arrive by its memory clobber
  mbar_arrive(&ctl->item_full[s]);
  return true;
}

// Every lane of a consumer warp calls this; lane 0 frees the slot once the
// whole warp has read it.
__device__ __forceinline__ bool bwd_take_rank(int i, int& w, const BwdParams& p, BwdCtl* ctl) {
  const int s = i & 1;
  if (!__all_sync(0xFFFFFFFFu, bwd_wait(&ctl->item_full[s], (static_cast<uint32_t>(i) >> 1) & 1u, ctl, p,
                                        kSiteBwdItemFull)))
    return false;
  w = ctl->item[s];  // read after the wait (its asm has a memory clobber)
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&ctl->item_empty[s]);
  return true;
}

// Both item slots' barriers (range variant): one producer arrival, nine
// consumer arrivals (the MMA warp and the eight compute warps).
__device__ __forceinline__ void bwd_init_item_slots(BwdCtl* ctl) {
  for (int s = 0; s < 2; ++s) {
    mbar_init(&ctl->item_full[s], 1);
    mbar_init(&ctl->item_empty[s], 9);
  }
}

__device__ __forceinline__ bool bwd_warp_wait(uint64_t* bar, uint32_t parity, BwdCtl* ctl, const BwdParams& p,
                                              int site) {
  return __all_sync(0xFFFFFFFFu, bwd_wait(bar, parity, ctl, p, site));
}

// Layout constants of one configuration (head dim kD, bf16).
template <int kD>
struct BwdCfg {
  using C = KernelCfg<2, kD, kD, kOutBf16>;  // the forward's tile layout and MMA helpers
  static constexpr int kTileBytes = 128 * kD * 2;
  // Warps 0-7 compute (two warpgroups), warp 8 issues MMAs, warp 9 TMA,
  // warps 10-11 only complete warpgroup 2.  setmaxnreg gives the compute
  // warpgroups 216 registers and warpgroup 2 72: 256 * 216 + 128 * 72 =
  // 64512 = 384 * 168, the launch budget.
  static constexpr int kThreads = 384;
  static constexpr int kLaunchRegs = 168;
  static constexpr int kComputeRegs = 216;
  static constexpr int kControlRegs = 72;
  static_assert(256 * kComputeRegs + 128 * kControlRegs <= kThreads * kLaunchRegs, "register split over budget");
  static_assert(kThreads * kLaunchRegs <= 65536, "launch register budget");
  static constexpr int kResOffset = 0;       // resident pair (K, V) or (Q, dO)
  static constexpr int kStageOffset = 2 * kTileBytes;
  static constexpr int kStatsOffset = kStageOffset + 4 * kTileBytes;  // two stages of two tiles
  static constexpr int kRangeOffset = kStatsOffset + 2 * 128 * 8;     // per-query key ranges (range variant)
  static constexpr int kCtlOffset = kRangeOffset + 2 * 128 * 8;
  static constexpr int kSmemBytes = 1024 + kCtlOffset + 1024;
  static constexpr uint32_t kColS = 0, kColDp = 128, kColA0 = 256, kColA1 = 256 + kD;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kD == 64 || kD == 128, "head dim");
};

// ------------------------------------------- per-key-tile query tiles (ranges)
// With per-row key ranges, tile_q[b, kt] = the span [x, y) of query tiles
// whose K/V tile range (tile_kv, from row_range_tiles_kernel) contains key
// tile kt; (0, 0) when none does.  One thread per (b, kt).  It also zeroes
// the dK/dV and dQ kernels' item counters (dynamic deal), when given.
__global__ void __launch_bounds__(128) key_tile_queries_kernel(const int2* __restrict__ tile_kv, int2* tile_q, int B,
                                                               int num_tiles, int* item_counters) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (item_counters != nullptr && t == 0) {
    item_counters[0] = 0;
    item_counters[1] = 0;
  }
  if (t >= static_cast<long long>(B) * num_tiles) return;
  const int b = static_cast<int>(t / num_tiles);
  const int kt = static_cast<int>(t - static_cast<long long>(b) * num_tiles);
  const int2* row = tile_kv + static_cast<size_t>(b) * num_tiles;
  int lo = INT_MAX, hi = INT_MIN;
  for (int qt = 0; qt < num_tiles; ++qt) {
    const int2 e = __ldg(row + qt);
    if (e.x <= kt && kt < e.y) {
      lo = min(lo, qt);
      hi = max(hi, qt + 1);
    }
  }
  tile_q[t] = lo < hi ? make_int2(lo, hi) : make_int2(0, 0);
}

// ------------------------------------------------------ dK, dV work items
struct KvItem {
  int b, hkv, kt;
  int qt_lo, qt_hi;  // query tiles that see key tile kt
  int steps;         // group * (qt_hi - qt_lo)
};

// Items ranked heaviest first: with causal masking the early key tiles are
// seen by the most query tiles.  With per-row key ranges the query tiles
// come from the table the pre-pass kernels built.
template <bool kRanges>
__device__ __forceinline__ KvItem kv_item(int w, const BwdParams& p) {
  KvItem it;
  const int bh_count = p.B * p.Hkv;
  it.kt = w / bh_count;
  const int bh = w - it.kt * bh_count;
  it.b = bh / p.Hkv;
  it.hkv = bh - it.b * p.Hkv;
  if constexpr (kRanges) {
    const int2 e = __ldg(p.tile_q + static_cast<size_t>(it.b) * p.num_tiles + it.kt);
    it.qt_lo = e.x;
    it.qt_hi = e.y;
    it.steps = it.qt_hi > it.qt_lo ? p.group * (it.qt_hi - it.qt_lo) : 0;
    return it;
  }
  it.qt_lo = p.causal ? it.kt : 0;
  it.qt_hi = p.num_tiles;
  if (p.window > 0) {
    // query i sees key j iff j > i - window: the last query row that sees the
    // tile's last key is kt*128 + 127 + window - 1
    const long long last = static_cast<long long>(it.kt) * 128 + 127 + p.window - 1;
    if (last / 128 + 1 < it.qt_hi) it.qt_hi = static_cast<int>(last / 128 + 1);
  }
  it.steps = it.qt_hi > it.qt_lo ? p.group * (it.qt_hi - it.qt_lo) : 0;
  return it;
}

template <int kD, bool kRanges>
__device__ void dkdv_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                              const CUtensorMap* tm_do, const BwdParams& p, BwdCtl* ctl, uint8_t* smem) {
  using G = BwdCfg<kD>;
  using C = typename G::C;
  const uint64_t pol_last = l2_policy_evict_last();
  uint32_t kv_armed = 0, st_armed[2] = {0, 0}, step = 0, items = 0;
  bool ok = true;
  for (int i = 0; ok; ++i) {
    int w;
    if constexpr (kRanges) {
      ok = bwd_publish_rank(i, w, p, ctl);
      if (!ok) break;
    } else {
      w = work_rank(i);
    }
    if (w >= p.num_work) break;
    const KvItem it = kv_item<kRanges>(w, p);
    if (it.steps == 0) continue;
    ok = bwd_wait(&ctl->kv_empty, (items & 1u) ^ 1u, ctl, p, kSiteBwdProdKv);
    if (!ok) break;
    ++items;
    mbar_arrive_expect_tx(&ctl->kv_full, 2 * G::kTileBytes);
    ++kv_armed;
#pragma unroll
    for (int c = 0; c < C::kQChunks; ++c) {
      tma_load_4d(smem + G::kResOffset + c * C::kChunkBytes, tm_k, &ctl->kv_full, c * 64, it.hkv, it.kt * 128, it.b,
                  pol_last);
      tma_load_4d(smem + G::kResOffset + G::kTileBytes + c * C::kChunkBytes, tm_v, &ctl->kv_full, c * 64, it.hkv,
                  it.kt * 128, it.b, pol_last);
    }
    for (int s = 0; s < it.steps && ok; ++s, ++step) {
      const int t = step & 1;
      ok = bwd_wait(&ctl->st_empty[t], ((step >> 1) & 1u) ^ 1u, ctl, p, kSiteBwdProdStage);
      if (!ok) break;
      const int qspan = it.qt_hi - it.qt_lo;
      const int h = it.hkv * p.group + s / qspan;
      const int qt = it.qt_lo + s % qspan;
      uint8_t* dst = smem + G::kStageOffset + t * 2 * G::kTileBytes;
      mbar_arrive_expect_tx(&ctl->st_full[t], 2 * G::kTileBytes);
      ++st_armed[t];
#pragma unroll
      for (int c = 0; c < C::kQChunks; ++c) {
        tma_load_4d(dst + c * C::kChunkBytes, tm_q, &ctl->st_full[t], c * 64, h, qt * 128, it.b, pol_last);
        tma_load_4d(dst + G::kTileBytes + c * C::kChunkBytes, tm_do, &ctl->st_full[t], c * 64, h, qt * 128, it.b,
                    pol_last);
      }
    }
  }
  if (!ok) {  // let every copy this thread started land before the CTA exits
    if (kv_armed) bwd_wait(&ctl->kv_full, (kv_armed - 1) & 1u, ctl, p, kSiteBwdDrain, false);
    for (int t = 0; t < 2; ++t)
      if (st_armed[t]) bwd_wait(&ctl->st_full[t], (st_armed[t] - 1) & 1u, ctl, p, kSiteBwdDrain, false);
  }
}

// One converged warp issues every MMA (elect.sync inside each).  Per step s:
//   dV += P^T(s) dO(s);  S^T(s+1) = K Q(s+1)^T;  dK += dS^T(s) Q(s);  dP^T(s+1) = V dO(s+1)^T
// S^T(s+1) overwrites the columns holding P^T(s), so it follows the dV
// product; dP^T(s+1) likewise follows the dK product.
template <int kD, bool kRanges>
__device__ void dkdv_mma(const BwdParams& p, BwdCtl* ctl, uint8_t* smem, uint32_t tmem) {
  using G = BwdCfg<kD>;
  using C = typename G::C;
  constexpr uint32_t kIdS = make_idesc(1, 128, 128, false, false);
  constexpr uint32_t kIdAcc = make_idesc(1, 128, kD, false, true);
  constexpr int kHalf = 4;  // 8 MMAs of 16 rows make one 128-row K extent
  const uint32_t k_lo = sw128_desc_lo(smem_u32(smem + G::kResOffset), 16);
  const uint32_t v_lo = sw128_desc_lo(smem_u32(smem + G::kResOffset + G::kTileBytes), 16);
  // Descriptors of stage 0; stage 1 sits 2 tiles further, i.e. its start
  // address field (address >> 4, 14 bits, no carry below 256 KB) is larger
  // by kStageStep.  Computed, not indexed, so they stay in registers.
  const uint32_t base0 = smem_u32(smem + G::kStageOffset);
  const uint32_t st_lo0 = sw128_desc_lo(base0, 16);                              // Q(s), K-major
  const uint32_t st_mn0 = sw128_desc_lo(base0, C::kChunkBytes);                  // Q(s), MN-major
  const uint32_t do_lo0 = sw128_desc_lo(base0 + G::kTileBytes, 16);              // dO(s), K-major
  const uint32_t do_mn0 = sw128_desc_lo(base0 + G::kTileBytes, C::kChunkBytes);  // dO(s), MN-major
  constexpr uint32_t kStageStep = (2 * G::kTileBytes) >> 4;
  const uint32_t tS = tmem + G::kColS, tDp = tmem + G::kColDp;
  const uint32_t tDv = tmem + G::kColA0, tDk = tmem + G::kColA1;
  uint32_t step = 0, items = 0, ph_p = 0, ph_ds = 0;
  bool ok = true;
  for (int i = 0; ok; ++i) {
    int w;
    if constexpr (kRanges) {
      ok = bwd_take_rank(i, w, p, ctl);
      if (!ok) break;
    } else {
      w = work_rank(i);
    }
    if (w >= p.num_work) break;
    const KvItem it = kv_item<kRanges>(w, p);
    if (it.steps == 0) continue;
    ok = bwd_warp_wait(&ctl->kv_full, items & 1u, ctl, p, kSiteBwdMmaKv);
    if (!ok) break;
    // prologue: S^T(0), dP^T(0)
    ok = bwd_warp_wait(&ctl->st_full[step & 1], (step >> 1) & 1u, ctl, p, kSiteBwdMmaStage);
    if (!ok) break;
    mma_qk<C, 0>(tS, k_lo, st_lo0 + (step & 1) * kStageStep, kIdS);
    mma_commit_elect(&ctl->s_full);
    mma_qk<C, 0>(tDp, v_lo, do_lo0 + (step & 1) * kStageStep, kIdS);
    mma_commit_elect(&ctl->dp_full);
    for (int s = 0; s < it.steps; ++s, ++step) {
      const int t = step & 1;
      ok = bwd_warp_wait(&ctl->p_full, ph_p, ctl, p, kSiteBwdMmaP);
      if (!ok) break;
      ph_p ^= 1u;
      if (s == 0) {  // the previous item's epilogue must be done with dV, dK
        ok = bwd_warp_wait(&ctl->acc_empty, (items & 1u) ^ 1u, ctl, p, kSiteBwdMmaAcc);
        if (!ok) break;
      }
      tc_fence_after();
      // A = P^T: query columns 0-63 from words [0, 32), 64-127 from [64, 96)
      mma_pv<C, 0, kHalf>(tDv, tS, do_mn0 + t * kStageStep, kIdAcc, s > 0 ? 1u : 0u);
      mma_pv<C, kHalf, 2 * kHalf>(tDv, tS + 32, do_mn0 + t * kStageStep, kIdAcc, 1u);
      const bool more = s + 1 < it.steps;
      if (more) {
        ok = bwd_warp_wait(&ctl->st_full[t ^ 1], ((step + 1) >> 1) & 1u, ctl, p, kSiteBwdMmaStage);
        if (!ok) break;
        mma_qk<C, 0>(tS, k_lo, st_lo0 + (t ^ 1) * kStageStep, kIdS);
        mma_commit_elect(&ctl->s_full);
      }
      ok = bwd_warp_wait(&ctl->ds_full, ph_ds, ctl, p, kSiteBwdMmaDs);
      if (!ok) break;
      ph_ds ^= 1u;
      tc_fence_after();
      mma_pv<C, 0, kHalf>(tDk, tDp, st_mn0 + t * kStageStep, kIdAcc, s > 0 ? 1u : 0u);
      mma_pv<C, kHalf, 2 * kHalf>(tDk, tDp + 32, st_mn0 + t * kStageStep, kIdAcc, 1u);
      mma_commit_elect(&ctl->st_empty[t]);
      if (more) {
        mma_qk<C, 0>(tDp, v_lo, do_lo0 + (t ^ 1) * kStageStep, kIdS);
        mma_commit_elect(&ctl->dp_full);
      }
    }
    if (!ok) break;
    mma_commit_elect(&ctl->acc_full);
    mma_commit_elect(&ctl->kv_empty);
    ++items;
  }
  mma_commit_elect(&ctl->drain);
  __all_sync(0xFFFFFFFFu, bwd_wait(&ctl->drain, 0, ctl, p, kSiteBwdDrain, false));
}

// Stats of one query row: (-lse2, D), or (-inf, 0) past N.
__device__ __forceinline__ float2 load_stats(const BwdParams& p, int b, int h, int q) {
  if (q >= p.N) return make_float2(-CUDART_INF_F, 0.0f);
  return __ldg(p.stats + (static_cast<size_t>(b) * p.Hq + h) * p.N + q);
}

// Per-row key range of one query row ((0, 0) past N: no key).
__device__ __forceinline__ int2 load_range(const BwdParams& p, int b, int q) {
  if (q >= p.N) return make_int2(0, 0);
  const size_t ix = static_cast<size_t>(b) * p.N + q;
  return make_int2(__ldg(p.key_lo + ix), __ldg(p.key_hi + ix));
}

// The query head and first query row of step s of a dK/dV item.
__device__ __forceinline__ void kv_step(const KvItem& it, const BwdParams& p, int s, int& h, int& q0) {
  const int qspan = it.qt_hi - it.qt_lo;
  h = it.hkv * p.group + s / qspan;
  q0 = (it.qt_lo + s % qspan) * 128;
}

// Two warpgroups; thread = key row j of the tile (warp % 4 picks the lane
// quadrant), warpgroup g takes the step's query columns [64 g, 64 g + 64).
// Nothing in the backward reduces over a row (P comes from the saved LSE),
// so the split needs no exchange; it puts two compute warps on every SMSP.
// Each warpgroup writes its packed P^T (dS^T) words into its own half of
// the S^T (dP^T) columns, which it has already read: g = 0 into columns
// [0, 32), g = 1 into [64, 96) (dP^T: +128).
template <int kD, bool kRanges>
__device__ void dkdv_compute(const BwdParams& p, BwdCtl* ctl, uint8_t* smem, uint32_t tmem, int warp, int lane) {
  using G = BwdCfg<kD>;
  const int g = warp >> 2;
  const int r = (warp & 3) * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tS = tmem + lane_off + G::kColS + 64 * g, tDp = tmem + lane_off + G::kColDp + 64 * g;
  const uint32_t tDv = tmem + lane_off + G::kColA0, tDk = tmem + lane_off + G::kColA1;
  float2* sbuf = reinterpret_cast<float2*>(smem + G::kStatsOffset);
  int2* rbuf = reinterpret_cast<int2*>(smem + G::kRangeOffset);
  const float cs = p.scale_log2;
  uint32_t step = 0, items = 0, ph_s = 0, ph_dp = 0;
  for (int i = 0;; ++i) {
    int w;
    if constexpr (kRanges) {
      if (!bwd_take_rank(i, w, p, ctl)) return;
    } else {
      w = work_rank(i);
    }
    if (w >= p.num_work) break;
    const KvItem it = kv_item<kRanges>(w, p);
    const int j = it.kt * 128 + r;  // this thread's key
    if (it.steps == 0) {            // no query sees this key tile: zero gradients
      if (j < p.N) {
        const size_t row = ((static_cast<size_t>(it.b) * p.N + j) * p.Hkv + it.hkv) * kD;
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(g == 0 ? p.dv : p.dk) + row);
        for (int x = 0; x < kD / 8; ++x) dst[x] = make_uint4(0, 0, 0, 0);
      }
      continue;
    }
    // warpgroup 0 fetches each step's stats (one row per thread) a step ahead;
    // with per-row key ranges also each query row's range
    float2 nxt = make_float2(0.0f, 0.0f);
    int2 nxt_rng = make_int2(0, 0);
    if (g == 0) {
      int h, q0;
      kv_step(it, p, 0, h, q0);
      nxt = load_stats(p, it.b, h, q0 + r);
      if constexpr (kRanges) nxt_rng = load_range(p, it.b, q0 + r);
    }
    for (int s = 0; s < it.steps; ++s, ++step) {
      int h, q0;
      kv_step(it, p, s, h, q0);
      // The step's (-lse2, D) pairs into the buffer of this step's parity;
      // all eight warps meet on an mbarrier (bounded wait).  A warp that
      // passed it knows every warp has finished the step before, so the
      // buffer written next is free.
      float2* st = sbuf + (step & 1) * 128;
      int2* rg = rbuf + (step & 1) * 128;
      if (g == 0) {
        st[r] = nxt;
        if constexpr (kRanges) rg[r] = nxt_rng;
        if (s + 1 < it.steps) {
          int h1, q1;
          kv_step(it, p, s + 1, h1, q1);
          nxt = load_stats(p, it.b, h1, q1 + r);
          if constexpr (kRanges) nxt_rng = load_range(p, it.b, q1 + r);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->stats_ready[step & 1]);
      if (!__all_sync(0xFFFFFFFFu, bwd_wait(&ctl->stats_ready[step & 1], (step >> 1) & 1u, ctl, p,
                                            kSiteBwdCompStats)))
        return;
      const float2* sg = st + 64 * g;
      const int2* rgg = rg + 64 * g;
      // visible columns of this warpgroup: c >= j - q0 - 64 g (causal), c < j - q0 - 64 g + window,
      // and with row ranges key_lo(row c) <= j < key_hi(row c)
      const int base = j - q0 - 64 * g;
      const int vlo = p.causal ? base : INT_MIN;
      const int vhi = p.window > 0 ? base + p.window : INT_MAX;
      const bool need_mask = kRanges || __any_sync(0xFFFFFFFFu, vlo > 0 || vhi < 64);

      bool ok = __all_sync(0xFFFFFFFFu, bwd_wait(&ctl->s_full, ph_s, ctl, p, kSiteBwdCompS));
      if (!ok) return;
      ph_s ^= 1u;
      tc_fence_after();
      float x[64];
      {
        uint32_t* raw = reinterpret_cast<uint32_t*>(x);
        tmem_ld32p(tS + 0, raw);
        tmem_ld32p(tS + 32, raw + 32);
        tmem_wait_ld();
      }
      // P^T: p = 2^(s cs - lse2), masked to 0; 32 packed bf16 words.
      const float4* sg4 = reinterpret_cast<const float4*>(sg);  // rows c, c + 1: (-lse2, D) each
      const uint64_t cs2 = f2_pack(cs, cs);
      uint32_t pk[32];
      if constexpr (kRanges) {
        // Row ranges mask every step: each column's test rides along with
        // its exponentials.
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) {
          const int c = 2 * ii;
          const float4 ab = sg4[ii];
          float y0, y1;
          f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), cs2, f2_pack(ab.x, ab.z)), y0, y1);
          float e0 = ex2_approx(y0), e1 = ex2_approx(y1);
          const int2 r0 = rgg[c], r1 = rgg[c + 1];
          if (c < vlo || c >= vhi || j < r0.x || j >= r0.y) e0 = 0.0f;
          if (c + 1 < vlo || c + 1 >= vhi || j < r1.x || j >= r1.y) e1 = 0.0f;
          x[c] = e0;
          x[c + 1] = e1;
          pk[ii] = pack_bf16x2(e0, e1);
        }
      } else {
        // Causal / window masks touch only tiles on the diagonal or the
        // window edge: masked scores become -inf first (exponential 0), so
        // the exponential loop has no branch and runs in batches of 8
        // column pairs -- loads, products, exponentials, packs -- whose
        // latencies overlap.
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < vlo || c >= vhi) x[c] = -CUDART_INF_F;
        }
#pragma unroll
        for (int b8 = 0; b8 < 4; ++b8) {
          float4 ab[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) ab[i] = sg4[8 * b8 + i];
          float e[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = 16 * b8 + 2 * i;
            f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), cs2, f2_pack(ab[i].x, ab[i].z)), e[2 * i], e[2 * i + 1]);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) e[i] = ex2_approx(e[i]);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = 16 * b8 + 2 * i;
            x[c] = e[2 * i];
            x[c + 1] = e[2 * i + 1];
            pk[8 * b8 + i] = pack_bf16x2(e[2 * i], e[2 * i + 1]);
          }
        }
      }
      tmem_st32(tS, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full);

      ok = __all_sync(0xFFFFFFFFu, bwd_wait(&ctl->dp_full, ph_dp, ctl, p, kSiteBwdCompDp));
      if (!ok) return;
      ph_dp ^= 1u;
      tc_fence_after();
      // dS^T: p (dp - D), packed bf16, 32 columns at a time (chunk k's 16
      // words land in columns this warpgroup has already read).
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint32_t dp[32];
        tmem_ld32(tDp + 32 * k, dp);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int c = 32 * k + 2 * ii;
          const float4 ab = sg4[16 * k + ii];
          const float d0 = x[c] * (__uint_as_float(dp[2 * ii]) - ab.y);
          const float d1 = x[c + 1] * (__uint_as_float(dp[2 * ii + 1]) - ab.w);
          pk[ii] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tDp + 16 * k, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->ds_full);
    }
    // Epilogue: warpgroup 0 stores dV, warpgroup 1 scale * dK, bf16.
    bool ok = __all_sync(0xFFFFFFFFu, bwd_wait(&ctl->acc_full, items & 1u, ctl, p, kSiteBwdCompAcc));
    if (!ok) return;
    tc_fence_after();
    {
      const bool store = j < p.N;
      const size_t row = ((static_cast<size_t>(it.b) * p.N + j) * p.Hkv + it.hkv) * kD;
      const uint32_t src = g == 0 ? tDv : tDk;
      const float f = g == 0 ? 1.0f : p.scale;
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(g == 0 ? p.dv : p.dk) + row);
#pragma unroll 1
      for (int cc = 0; cc < kD; cc += 32) {
        uint32_t v[32];
        tmem_ld32(src + cc, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          pk[q] = pack_bf16x2(__uint_as_float(v[2 * q]) * f, __uint_as_float(v[2 * q + 1]) * f);
        if (store) {
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[cc / 8 + q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->acc_empty);
    ++items;
  }
}

template <int kD, bool kRanges>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dkdv_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const BwdParams p) {
  using G = BwdCfg<kD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdCtl* ctl = reinterpret_cast<BwdCtl*>(smem + G::kCtlOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&ctl->kv_full, 1);
    mbar_init(&ctl->kv_empty, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl->st_full[t], 1);
      mbar_init(&ctl->st_empty[t], 1);
    }
    mbar_init(&ctl->s_full, 1);
    mbar_init(&ctl->dp_full, 1);
    mbar_init(&ctl->s_free, 8);
    mbar_init(&ctl->p_full, 8);
    mbar_init(&ctl->ds_full, 8);
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->acc_empty, 8);
    mbar_init(&ctl->stats_ready[0], 8);
    mbar_init(&ctl->stats_ready[1], 8);
    mbar_init(&ctl->drain, 1);
    if constexpr (kRanges) bwd_init_item_slots(ctl);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  if (warp < 8) {
    regs_increase<G::kComputeRegs>();
    dkdv_compute<kD, kRanges>(p, ctl, smem, tmem, warp, lane);
  } else {
    regs_decrease<G::kControlRegs>();
    if (warp == 8) {
      dkdv_mma<kD, kRanges>(p, ctl, smem, tmem);
      __syncwarp();
    } else if (warp == 9) {
      if (lane == 0) dkdv_producer<kD, kRanges>(&tm_q, &tm_k, &tm_v, &tm_do, p, ctl, smem);
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ dQ work items
struct QItem {
  int b, h, qt;
  int kt_lo, kt_hi;  // K/V tiles query tile qt sees
};

// Heaviest first: with causal masking the late query tiles see the most keys.
// With per-row key ranges the K/V tiles come from the forward's tile table.
template <bool kRanges>
__device__ __forceinline__ QItem q_item(int w, const BwdParams& p) {
  QItem it;
  const int bh_count = p.B * p.Hq;
  const int rnk = w / bh_count;
  const int bh = w - rnk * bh_count;
  it.qt = p.causal ? p.num_tiles - 1 - rnk : rnk;
  it.b = bh / p.Hq;
  it.h = bh - it.b * p.Hq;
  if constexpr (kRanges) {
    const int2 e = __ldg(p.tile_kv + static_cast<size_t>(it.b) * p.num_tiles + it.qt);
    it.kt_lo = e.x;
    it.kt_hi = e.y;
    return it;
  }
  const int last_row = min(it.qt * 128 + 127, p.N - 1);
  it.kt_hi = p.causal ? last_row / 128 + 1 : p.num_tiles;
  it.kt_lo = p.window > 0 ? max(0, it.qt * 128 - p.window + 1) / 128 : 0;
  return it;
}

template <int kD, bool kRanges>
__device__ void dq_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                            const CUtensorMap* tm_do, const BwdParams& p, BwdCtl* ctl, uint8_t* smem) {
  using G = BwdCfg<kD>;
  using C = typename G::C;
  const uint64_t pol_last = l2_policy_evict_last();
  const uint64_t pol_first = l2_policy_evict_first();
  uint32_t res_armed = 0, st_armed[2] = {0, 0}, step = 0, items = 0;
  bool ok = true;
  for (int i = 0; ok; ++i) {
    int w;
    if constexpr (kRanges) {
      ok = bwd_publish_rank(i, w, p, ctl);
      if (!ok) break;
    } else {
      w = work_rank(i);
    }
    if (w >= p.num_work) break;
    const QItem it = q_item<kRanges>(w, p);
    if (kRanges && it.kt_hi <= it.kt_lo) continue;  // no key visible to this tile: dQ = 0
    ok = bwd_wait(&ctl->kv_empty, (items & 1u) ^ 1u, ctl, p, kSiteBwdProdKv);
    if (!ok) break;
    ++items;
    mbar_arrive_expect_tx(&ctl->kv_full, 2 * G::kTileBytes);
    ++res_armed;
#pragma unroll
    for (int c = 0; c < C::kQChunks; ++c) {
      tma_load_4d(smem + G::kResOffset + c * C::kChunkBytes, tm_q, &ctl->kv_full, c * 64, it.h, it.qt * 128, it.b,
                  pol_first);
      tma_load_4d(smem + G::kResOffset + G::kTileBytes + c * C::kChunkBytes, tm_do, &ctl->kv_full, c * 64, it.h,
                  it.qt * 128, it.b, pol_first);
    }
    const int hkv = it.h / p.group;
    for (int kt = it.kt_lo; kt < it.kt_hi && ok; ++kt, ++step) {
      const int t = step & 1;
      ok = bwd_wait(&ctl->st_empty[t], ((step >> 1) & 1u) ^ 1u, ctl, p, kSiteBwdProdStage);
      if (!ok) break;
      uint8_t* dst = smem + G::kStageOffset + t * 2 * G::kTileBytes;
      mbar_arrive_expect_tx(&ctl->st_full[t], 2 * G::kTileBytes);
      ++st_armed[t];
#pragma unroll
      for (int c = 0; c < C::kQChunks; ++c) {
        tma_load_4d(dst + c * C::kChunkBytes, tm_k, &ctl->st_full[t], c * 64, hkv, kt * 128, it.b, pol_last);
        tma_load_4d(dst + G::kTileBytes + c * C::kChunkBytes, tm_v, &ctl->st_full[t], c * 64, hkv, kt * 128, it.b,
                    pol_last);
      }
    }
  }
  if (!ok) {
    if (res_armed) bwd_wait(&ctl->kv_full, (res_armed - 1) & 1u, ctl, p, kSiteBwdDrain, false);
    for (int t = 0; t < 2; ++t)
      if (st_armed[t]) bwd_wait(&ctl->st_full[t], (st_armed[t] - 1) & 1u, ctl, p, kSiteBwdDrain, false);
  }
}

// Per step s (K/V tile kt_lo + s):
//   S(s+1) = Q K(s+1)^T as soon as the compute warps have read S(s);
//   dQ += dS(s) K(s) once dS(s) is in tensor memory (over dP(s));
//   dP(s+1) = dO V(s+1)^T after it (it overwrites dS(s)).
template <int kD, bool kRanges>
__device__ void dq_mma(const BwdParams& p, BwdCtl* ctl, uint8_t* smem, uint32_t tmem) {
  using G = BwdCfg<kD>;
  using C = typename G::C;
  constexpr uint32_t kIdS = make_idesc(1, 128, 128, false, false);
  constexpr uint32_t kIdAcc = make_idesc(1, 128, kD, false, true);
  const uint32_t q_lo = sw128_desc_lo(smem_u32(smem + G::kResOffset), 16);
  const uint32_t do_lo = sw128_desc_lo(smem_u32(smem + G::kResOffset + G::kTileBytes), 16);
  // Stage-0 descriptors; stage 1's start address field is kStageStep larger
  // (computed, not indexed, so they stay in registers).
  const uint32_t base0 = smem_u32(smem + G::kStageOffset);
  const uint32_t k_lo0 = sw128_desc_lo(base0, 16);
  const uint32_t k_mn0 = sw128_desc_lo(base0, C::kChunkBytes);
  const uint32_t v_lo0 = sw128_desc_lo(base0 + G::kTileBytes, 16);
  constexpr uint32_t kStageStep = (2 * G::kTileBytes) >> 4;
  const uint32_t tS = tmem + G::kColS, tDp = tmem + G::kColDp, tDq = tmem + G::kColA0;
  uint32_t step = 0, items = 0, ph_free = 0, ph_ds = 0;
  bool ok = true;
  for (int i = 0; ok; ++i) {
    int w;
    if constexpr (kRanges) {
      ok = bwd_take_rank(i, w, p, ctl);
      if (!ok) break;
    } else {
      w = work_rank(i);
    }
    if (w >= p.num_work) break;
    const QItem it = q_item<kRanges>(w, p);
    const int n = it.kt_hi - it.kt_lo;
    if (kRanges && n <= 0) continue;
    ok = bwd_warp_wait(&ctl->kv_full, items & 1u, ctl, p, kSiteBwdMmaKv);
    if (!ok) break;
    ok = bwd_warp_wait(&ctl->st_full[step & 1], (step >> 1) & 1u, ctl, p, kSiteBwdMmaStage);
    if (!ok) break;
    mma_qk<C, 0>(tS, q_lo, k_lo0 + (step & 1) * kStageStep, kIdS);
    mma_commit_elect(&ctl->s_full);
    mma_qk<C, 0>(tDp, do_lo, v_lo0 + (step & 1) * kStageStep, kIdS);
    mma_commit_elect(&ctl->dp_full);
    for (int s = 0; s < n; ++s, ++step) {
      const int t = step & 1;
      const bool more = s + 1 < n;
      ok = bwd_warp_wait(&ctl->s_free, ph_free, ctl, p, kSiteBwdMmaSFree);
      if (!ok) break;
      ph_free ^= 1u;
      if (more) {
        ok = bwd_warp_wait(&ctl->st_full[t ^ 1], ((step + 1) >> 1) & 1u, ctl, p, kSiteBwdMmaStage);
        if (!ok) break;
        tc_fence_after();
        mma_qk<C, 0>(tS, q_lo, k_lo0 + (t ^ 1) * kStageStep, kIdS);
        mma_commit_elect(&ctl->s_full);
      }
      ok = bwd_warp_wait(&ctl->ds_full, ph_ds, ctl, p, kSiteBwdMmaDs);
      if (!ok) break;
      ph_ds ^= 1u;
      if (s == 0) {
        ok = bwd_warp_wait(&ctl->acc_empty, (items & 1u) ^ 1u, ctl, p, kSiteBwdMmaAcc);
        if (!ok) break;
      }
      tc_fence_after();
      // A = dS: key columns 0-63 from words [128, 160), 64-127 from [192, 224)
      mma_pv<C, 0, 4>(tDq, tDp, k_mn0 + t * kStageStep, kIdAcc, s > 0 ? 1u : 0u);
      mma_pv<C, 4, 8>(tDq, tDp + 32, k_mn0 + t * kStageStep, kIdAcc, 1u);
      mma_commit_elect(&ctl->st_empty[t]);
      if (more) {
        mma_qk<C, 0>(tDp, do_lo, v_lo0 + (t ^ 1) * kStageStep, kIdS);
        mma_commit_elect(&ctl->dp_full);
      }
    }
    if (!ok) break;
    mma_commit_elect(&ctl->acc_full);
    mma_commit_elect(&ctl->kv_empty);
    ++items;
  }
  mma_commit_elect(&ctl->drain);
  __all_sync(0xFFFFFFFFu, bwd_wait(&ctl->drain, 0, ctl, p, kSiteBwdDrain, false));
}

// Two warpgroups; thread = query row i of the tile, warpgroup g takes the
// step's key columns [64 g, 64 g + 64) and writes its packed dS words into
// its own half of the dP columns ([128, 160) or [192, 224)).
template <int kD, bool kRanges>
__device__ void dq_compute(const BwdParams& p, BwdCtl* ctl, uint32_t tmem, int warp, int lane) {
  using G = BwdCfg<kD>;
  const int g = warp >> 2;
  const int r = (warp & 3) * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tS = tmem + lane_off + G::kColS + 64 * g, tDp = tmem + lane_off + G::kColDp + 64 * g;
  const uint32_t tDq = tmem + lane_off + G::kColA0;
  const float cs = p.scale_log2;
  uint32_t items = 0, ph_s = 0, ph_dp = 0;
  for (int i = 0;; ++i) {
    int w;
    if constexpr (kRanges) {
      if (!bwd_take_rank(i, w, p, ctl)) return;
    } else {
      w = work_rank(i);
    }
    if (w >= p.num_work) break;
    const QItem it = q_item<kRanges>(w, p);
    const int qrow = it.qt * 128 + r;
    if (kRanges && it.kt_hi <= it.kt_lo) {  // no row of the tile sees a key: dQ = 0
      if (qrow < p.N) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.dq) +
                                              ((static_cast<size_t>(it.b) * p.N + qrow) * p.Hq + it.h) * kD);
        for (int x = g * (kD / 16); x < (g + 1) * (kD / 16); ++x) dst[x] = make_uint4(0, 0, 0, 0);
      }
      continue;
    }
    const float2 st = load_stats(p, it.b, it.h, qrow);
    int key_hi = p.causal ? min(p.N, qrow + 1) : p.N;  // visible keys [key_lo, key_hi)
    int key_lo = p.window > 0 ? max(0, qrow - p.window + 1) : 0;
    if (kRanges && qrow < p.N) {
      const size_t ix = static_cast<size_t>(it.b) * p.N + qrow;
      key_lo = max(key_lo, __ldg(p.key_lo + ix));
      key_hi = min(key_hi, __ldg(p.key_hi + ix));
    }
    for (int kt = it.kt_lo; kt < it.kt_hi; ++kt) {
      const int kbase = kt * 128 + 64 * g;
      const bool need_mask = __any_sync(0xFFFFFFFFu, kbase < key_lo || kbase + 64 > key_hi);
      bool ok = __all_sync(0xFFFFFFFFu, bwd_wait(&ctl->s_full, ph_s, ctl, p, kSiteBwdCompS));
      if (!ok) return;
      ph_s ^= 1u;
      tc_fence_after();
      float x[64];
      {
        uint32_t* raw = reinterpret_cast<uint32_t*>(x);
        tmem_ld32p(tS + 0, raw);
        tmem_ld32p(tS + 32, raw + 32);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_free);
      {
        // masked scores to -inf first (exponential 0): the loop below has
        // no branch, so the exponentials of consecutive columns overlap
        if (need_mask) {
          const int vlo = key_lo - kbase, vhi = key_hi - kbase;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < vlo || c >= vhi) x[c] = -CUDART_INF_F;
        }
        const uint64_t cs2 = f2_pack(cs, cs);
        const uint64_t nl2 = f2_pack(st.x, st.x);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float y0, y1;
          f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), cs2, nl2), y0, y1);
          x[c] = ex2_approx(y0);
          x[c + 1] = ex2_approx(y1);
        }
      }
      ok = __all_sync(0xFFFFFFFFu, bwd_wait(&ctl->dp_full, ph_dp, ctl, p, kSiteBwdCompDp));
      if (!ok) return;
      ph_dp ^= 1u;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint32_t dp[32];
        tmem_ld32(tDp + 32 * k, dp);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int c = 32 * k + 2 * ii;
          const float d0 = x[c] * (__uint_as_float(dp[2 * ii]) - st.y);
          const float d1 = x[c + 1] * (__uint_as_float(dp[2 * ii + 1]) - st.y);
          pk[ii] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tDp + 16 * k, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->ds_full);
    }
    // Epilogue: warpgroup g stores dQ columns [g kD/2, (g + 1) kD/2), scaled.
    bool ok = __all_sync(0xFFFFFFFFu, bwd_wait(&ctl->acc_full, items & 1u, ctl, p, kSiteBwdCompAcc));
    if (!ok) return;
    tc_fence_after();
    const bool store = qrow < p.N;
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.dq) +
                                          ((static_cast<size_t>(it.b) * p.N + qrow) * p.Hq + it.h) * kD);
#pragma unroll 1
    for (int cc = g * (kD / 2); cc < (g + 1) * (kD / 2); cc += 32) {
      uint32_t v[32];
      tmem_ld32(tDq + cc, v);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        pk[q] = pack_bf16x2(__uint_as_float(v[2 * q]) * p.scale, __uint_as_float(v[2 * q + 1]) * p.scale);
      if (store) {
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[cc / 8 + q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->acc_empty);
    ++items;
  }
}

template <int kD, bool kRanges>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dq_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const BwdParams p) {
  using G = BwdCfg<kD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdCtl* ctl = reinterpret_cast<BwdCtl*>(smem + G::kCtlOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&ctl->kv_full, 1);
    mbar_init(&ctl->kv_empty, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl->st_full[t], 1);
      mbar_init(&ctl->st_empty[t], 1);
    }
    mbar_init(&ctl->s_full, 1);
    mbar_init(&ctl->dp_full, 1);
    mbar_init(&ctl->s_free, 8);
    mbar_init(&ctl->p_full, 8);
    mbar_init(&ctl->ds_full, 8);
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->acc_empty, 8);
    mbar_init(&ctl->stats_ready[0], 8);
    mbar_init(&ctl->stats_ready[1], 8);
    mbar_init(&ctl->drain, 1);
    if constexpr (kRanges) bwd_init_item_slots(ctl);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  if (warp < 8) {
    regs_increase<G::kComputeRegs>();
    dq_compute<kD, kRanges>(p, ctl, tmem, warp, lane);
  } else {
    regs_decrease<G::kControlRegs>();
    if (warp == 8) {
      dq_mma<kD, kRanges>(p, ctl, smem, tmem);
      __syncwarp();
    } else if (warp == 9) {
      if (lane == 0) dq_producer<kD, kRanges>(&tm_q, &tm_k, &tm_v, &tm_do, p, ctl, smem);
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, 512);
}

}  // namespace ea
