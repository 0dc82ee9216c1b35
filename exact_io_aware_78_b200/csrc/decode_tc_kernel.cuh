// decode_tc_kernel.cuh -- decode / split-KV forward on the tensor cores
// (sm_100a): Nq new query rows of the g query heads of one key/value head,
// g * Nq <= 32 rows, against a long key/value cache.
//
// The same exact attention as the prefill kernel (softmax(scale Q K^T +
// mask) V with a running row maximum and sum: "Flash Attention" concept
// note (heepie.pages.dev), TO-BE diagram and "Tiling"), with the keys split
// across CTAs and the parts merged through their log-sum-exps by
// decode_combine_kernel (the decoding work the pages list by title,
// FlashDecoding++).
//
// Design.  A decode step is bound by reading K and V once; the arithmetic is
// ~4 FLOP per byte.  The g * Nq query rows of a key/value head fill the first
// rows of one 128-row tcgen05 tile (the rest stay zero), so S = Q K^T and
// O += P V each cost 8 MMAs per 128-key tile -- a third of the tile's HBM
// time.  The rows are written into all four 32-lane quadrants of the tile,
// so that four softmax warps (one per SMSP) can each own a quarter of a
// tile's keys.
//   * 148 persistent CTAs split the whole stream of K/V tiles (all (batch,
//     key/value head) pairs, each pair's visible tiles in order) into equal
//     contiguous ranges ("stream-K").  Per pair its range touches, a CTA
//     emits four partial results (m, l, unnormalised O), one per softmax
//     warp, into that pair's slots 4 k .. 4 k + 3, k = the CTA's rank among
//     the pair's contributors; the pair's last contributor marks the
//     remaining slots empty.  The combine kernel merges them all by their
//     log-sum-exps, exactly.
//   * Warp 5 issues TMA copies: the pair's query rows as one box of g heads
//     x Nq rows into each lane quadrant of the query tile, then K(j), V(j)
//     into a shared-memory ring.  Warp 4 issues the MMAs: S(j) into one of
//     two tensor-memory buffers, so S(j + 1) runs while the softmax works on
//     S(j); O += P(j) V(j) with P read from tensor memory.  Warps 0-3 are
//     the softmax: warp w, one thread per query row in quadrant w, keeps its
//     own running maximum and sum over key columns [32 w, 32 w + 32) of
//     every tile (an independent split of the keys, as the combine expects),
//     writes P for its columns and zeros elsewhere over its rows' S buffer,
//     and rescales its own copy of O lazily (only when its maximum moves by
//     more than 8 in log2 units).
//   * Every wait is bounded; on expiry the kernel records the site in the
//     error word, all roles unwind, tensor memory is freed.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda.h>
#include <math_constants.h>

#include "attn_fwd_kernel.cuh"
#include "sm100_ptx.cuh"

namespace ea {

constexpr int kDecodeTcMaxRows = 32;

struct DecodeTcParams {
  float* part_ml;              // [pairs, kmax, R, 2]: m (log2 units), l
  float* part_acc;             // [pairs, kmax, R, d]: unnormalised O
  int* err;
  int B, Hq, Hkv, Nq, Nk, group, rows;  // rows R = group * Nq
  int causal, window;
  float scale_log2;
  int key_tile_lo;             // first K/V tile any row sees
  int tiles_per_pair;          // visible tiles of one (b, kv head)
  long long total_tiles;       // pairs * tiles_per_pair
  int kmax;                    // partial slots per pair
  unsigned long long timeout_ns;
};

enum : int {
  kSiteDtProdQ = 40,
  kSiteDtProdKv = 41,
  kSiteDtMmaQ = 42,
  kSiteDtMmaKv = 43,
  kSiteDtMmaP = 44,
  kSiteDtMmaO = 45,
  kSiteDtSoftS = 46,
  kSiteDtSoftPv = 47,
  kSiteDtSoftO = 48,
  kSiteDtDrain = 49
};

template <int kD>
struct DecodeTcCfg {
  using C = KernelCfg<2, kD, kD, kOutBf16>;  // the forward's tile layout and MMA helpers
  static constexpr int kTileBytes = 128 * kD * 2;
  static constexpr int kStages = kD == 128 ? 6 : 8;
  static constexpr int kQOffset = 0;
  static constexpr int kRingOffset = kTileBytes;
  static constexpr int kCtlOffset = kRingOffset + kStages * kTileBytes;
  static constexpr int kSmemBytes = 1024 + kCtlOffset + 1024;
  static constexpr int kThreads = 192;  // warps 0-3 softmax, 4 MMA, 5 TMA
  static constexpr uint32_t kColS = 0, kColO = 256;  // S buffers at 0 and 128
  static constexpr float kTau = 8.0f;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct DecodeTcCtl {
  uint64_t full[8], empty[8];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_full, o_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(DecodeTcCtl) <= 1024, "control block");

__device__ __forceinline__ bool dt_wait(uint64_t* bar, uint32_t parity, DecodeTcCtl* ctl, const DecodeTcParams& p,
                                        int site, bool honor_abort = true) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
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

__device__ __forceinline__ bool dt_warp_wait(uint64_t* bar, uint32_t parity, DecodeTcCtl* ctl,
                                             const DecodeTcParams& p, int site) {
  return __all_sync(0xFFFFFFFFu, dt_wait(bar, parity, ctl, p, site));
}

// The CTA's range of the global tile stream, [start(c), start(c + 1)).
__device__ __forceinline__ long long dt_start(long long c, const DecodeTcParams& p) {
  return c * p.total_tiles / gridDim.x;
}

// The first CTA whose range holds global tile x.
__device__ __forceinline__ long long dt_owner(long long x, const DecodeTcParams& p) {
  return ((x + 1) * gridDim.x - 1) / p.total_tiles;
}

// One segment of this CTA's range: pair `pair`, local tiles [j0, j1).
struct DtSeg {
  int pair, j0, j1;
};

__device__ __forceinline__ DtSeg dt_seg(long long t, long long end, const DecodeTcParams& p) {
  DtSeg s;
  s.pair = static_cast<int>(t / p.tiles_per_pair);
  s.j0 = static_cast<int>(t - static_cast<long long>(s.pair) * p.tiles_per_pair);
  const long long pair_end = static_cast<long long>(s.pair + 1) * p.tiles_per_pair;
  s.j1 = static_cast<int>((end < pair_end ? end : pair_end) - static_cast<long long>(s.pair) * p.tiles_per_pair);
  return s;
}

template <int kD>
__device__ void dt_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                            const DecodeTcParams& p, DecodeTcCtl* ctl, uint8_t* smem) {
  using G = DecodeTcCfg<kD>;
  using C = typename G::C;
  const uint64_t pol = l2_policy_evict_first();
  const long long end = dt_start(blockIdx.x + 1, p);
  uint32_t ld = 0, q_n = 0;
  bool ok = true;
  for (long long t = dt_start(blockIdx.x, p); t < end && ok;) {
    const DtSeg sg = dt_seg(t, end, p);
    t += sg.j1 - sg.j0;
    const int b = sg.pair / p.Hkv, hkv = sg.pair - b * p.Hkv;
    ok = dt_wait(&ctl->q_empty, (q_n & 1u) ^ 1u, ctl, p, kSiteDtProdQ);
    if (!ok) break;
    ++q_n;
    mbar_arrive_expect_tx(&ctl->q_full, static_cast<uint32_t>(4 * C::kQChunks * p.rows * 128));
#pragma unroll
    for (int c = 0; c < C::kQChunks; ++c)
#pragma unroll
      for (int quad = 0; quad < 4; ++quad)  // rows 32 quad .. 32 quad + R - 1
        tma_load_4d(smem + G::kQOffset + c * C::kChunkBytes + quad * 32 * 128, tm_q, &ctl->q_full, c * 64,
                    hkv * p.group, 0, b, pol);
    for (int j = sg.j0; j < sg.j1 && ok; ++j) {
      const int kt = p.key_tile_lo + j;
#pragma unroll
      for (int which = 0; which < 2; ++which, ++ld) {
        const uint32_t st = ld % G::kStages, ph = (ld / G::kStages) & 1u;
        ok = dt_wait(&ctl->empty[st], ph ^ 1u, ctl, p, kSiteDtProdKv);
        if (!ok) break;
        uint8_t* dst = smem + G::kRingOffset + st * G::kTileBytes;
        mbar_arrive_expect_tx(&ctl->full[st], G::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kQChunks; ++c)
          tma_load_4d(dst + c * C::kChunkBytes, which == 0 ? tm_k : tm_v, &ctl->full[st], c * 64, hkv, kt * 128, b,
                      pol);
      }
    }
  }
  if (!ok) {  // let every copy this thread started land before the CTA exits
    for (uint32_t P = ld > G::kStages ? ld - G::kStages : 0; P < ld; ++P)
      dt_wait(&ctl->full[P % G::kStages], (P / G::kStages) & 1u, ctl, p, kSiteDtDrain, false);
    if (q_n) dt_wait(&ctl->q_full, (q_n - 1) & 1u, ctl, p, kSiteDtDrain, false);
  }
}

// Per segment of n tiles (load index of K(j) = base + 2j, of V(j) = base + 2j + 1):
//   S(0), S(1); then per j: O (+)= P(j) V(j); S(j + 2) into the buffer P(j) used.
template <int kD>
__device__ void dt_mma(const DecodeTcParams& p, DecodeTcCtl* ctl, uint8_t* smem, uint32_t tmem) {
  using G = DecodeTcCfg<kD>;
  using C = typename G::C;
  constexpr uint32_t kIdS = make_idesc(1, 128, 128, false, false);
  constexpr uint32_t kIdO = make_idesc(1, 128, kD, false, true);
  const uint32_t q_lo = sw128_desc_lo(smem_u32(smem + G::kQOffset), 16);
  const uint32_t ring_k = sw128_desc_lo(smem_u32(smem + G::kRingOffset), 16);
  const uint32_t ring_v = sw128_desc_lo(smem_u32(smem + G::kRingOffset), C::kChunkBytes);
  constexpr uint32_t kUnits = G::kTileBytes >> 4;
  const long long end = dt_start(blockIdx.x + 1, p);
  uint32_t base = 0, q_n = 0, segs = 0, p_use[2] = {0, 0};
  bool ok = true;
  auto issue_s = [&](uint32_t j) -> bool {  // S(j) = Q K(j)^T into buffer j & 1
    const uint32_t ld = base + 2 * j, st = ld % G::kStages;
    if (!dt_warp_wait(&ctl->full[st], (ld / G::kStages) & 1u, ctl, p, kSiteDtMmaKv)) return false;
    mma_qk<C, 0>(tmem + G::kColS + 128 * (j & 1), q_lo, ring_k + st * kUnits, kIdS);
    mma_commit_elect(&ctl->empty[st]);
    mma_commit_elect(&ctl->s_full[j & 1]);
    return true;
  };
  for (long long t = dt_start(blockIdx.x, p); t < end && ok;) {
    const DtSeg sg = dt_seg(t, end, p);
    t += sg.j1 - sg.j0;
    const uint32_t n = static_cast<uint32_t>(sg.j1 - sg.j0);
    ok = dt_warp_wait(&ctl->q_full, q_n & 1u, ctl, p, kSiteDtMmaQ);
    if (!ok) break;
    ++q_n;
    ok = issue_s(0) && (n < 2 || issue_s(1));
    for (uint32_t j = 0; j < n && ok; ++j) {
      const uint32_t bsel = j & 1;
      ok = dt_warp_wait(&ctl->p_full[bsel], p_use[bsel] & 1u, ctl, p, kSiteDtMmaP);
      if (!ok) break;
      ++p_use[bsel];
      if (j == 0) {  // the previous segment's epilogue must be done with O
        ok = dt_warp_wait(&ctl->o_empty, (segs & 1u) ^ 1u, ctl, p, kSiteDtMmaO);
        if (!ok) break;
      }
      tc_fence_after();
      const uint32_t ld = base + 2 * j + 1, st = ld % G::kStages;
      ok = dt_warp_wait(&ctl->full[st], (ld / G::kStages) & 1u, ctl, p, kSiteDtMmaKv);
      if (!ok) break;
      mma_pv<C, 0, 8>(tmem + G::kColO, tmem + G::kColS + 128 * bsel, ring_v + st * kUnits, kIdO, j > 0 ? 1u : 0u);
      mma_commit_elect(&ctl->empty[st]);
      mma_commit_elect(&ctl->pv_done);
      if (j + 1 == n) mma_commit_elect(&ctl->q_empty);
      if (j + 2 < n) ok = issue_s(j + 2);
    }
    if (!ok) break;
    mma_commit_elect(&ctl->o_full);
    base += 2 * n;
    ++segs;
  }
  mma_commit_elect(&ctl->drain);
  __all_sync(0xFFFFFFFFu, dt_wait(&ctl->drain, 0, ctl, p, kSiteDtDrain, false));
}

// Warp w (0-3): thread = tile row 32 w + t, query row t (< R valid), key
// columns [32 w, 32 w + 32) of every tile.  Row t is query head hkv * g +
// t % g at new-token index t / g (the query box is heads-fastest); its
// partial row is r = (t % g) * Nq + t / g, the combine kernel's order.
template <int kD>
__device__ void dt_softmax(const DecodeTcParams& p, DecodeTcCtl* ctl, uint32_t tmem, int warp, int lane) {
  using G = DecodeTcCfg<kD>;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem + lane_off + G::kColS, tO = tmem + lane_off + G::kColO;
  const long long end = dt_start(blockIdx.x + 1, p);
  const bool valid = lane < p.rows;
  const int hg = lane % p.group, qi = lane / p.group;
  const int r = hg * p.Nq + qi;
  const int pos = p.Nk - p.Nq + qi;  // this row's token position
  const int key_hi = valid ? (p.causal ? pos + 1 : p.Nk) : 0;
  const int key_lo = p.window > 0 ? max(0, pos - p.window + 1) : 0;
  const float cs = p.scale_log2;
  uint32_t s_use[2] = {0, 0}, pv_n = 0, segs = 0;
  for (long long t = dt_start(blockIdx.x, p); t < end;) {
    const DtSeg sg = dt_seg(t, end, p);
    t += sg.j1 - sg.j0;
    const int n = sg.j1 - sg.j0;
    float m_used = -CUDART_INF_F, l = 0.0f;
    for (int j = 0; j < n; ++j) {
      const int bsel = j & 1;
      if (!__all_sync(0xFFFFFFFFu, dt_wait(&ctl->s_full[bsel], s_use[bsel] & 1u, ctl, p, kSiteDtSoftS))) return;
      ++s_use[bsel];
      tc_fence_after();
      float x[32];
      tmem_ld32(tS + 128 * bsel + 32 * warp, *reinterpret_cast<uint32_t(*)[32]>(x));
      tmem_wait_ld();
      const int kbase = (p.key_tile_lo + sg.j0 + j) * 128 + 32 * warp;
      const int vlo = key_lo - kbase, vhi = key_hi - kbase;
      if (__any_sync(0xFFFFFFFFu, vlo > 0 || vhi < 32)) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c < vlo || c >= vhi) x[c] = -CUDART_INF_F;
      }
      float mx = fmax3(x[0], x[1], x[2]);
#pragma unroll
      for (int c = 3; c < 31; c += 2) mx = fmax3(mx, x[c], x[c + 1]);
      const float m_tile = fmaxf(mx, x[31]) * cs;
      // The previous product O += P(j - 1) V(j - 1) must be complete before O
      // is rescaled; waiting for each product once keeps the phases in step.
      if (j > 0) {
        if (!__all_sync(0xFFFFFFFFu, dt_wait(&ctl->pv_done, pv_n & 1u, ctl, p, kSiteDtSoftPv))) return;
        ++pv_n;
      }
      float alpha = 1.0f;
      bool rescale = false;
      if (m_tile > m_used + G::kTau) {
        alpha = ex2_approx(m_used - m_tile);  // 0 when m_used is -inf
        rescale = j > 0 && m_used != -CUDART_INF_F;
        l *= alpha;
        m_used = m_tile;
      }
      if (__any_sync(0xFFFFFFFFu, rescale)) {
        tc_fence_after();
        const float f = rescale ? alpha : 1.0f;
#pragma unroll 1
        for (int cc = 0; cc < kD; cc += 32) {
          uint32_t ov[32];
          tmem_ld32(tO + cc, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
          tmem_st32(tO + cc, ov);
        }
      }
      // P over the S buffer: this warp's 16 packed words, zeros elsewhere.
      const float neg_ref = -((m_used == -CUDART_INF_F) ? 0.0f : m_used);
      float sum = 0.0f;
      uint32_t own[16];
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const float e0 = ex2_approx(fmaf(x[2 * ii], cs, neg_ref));
        const float e1 = ex2_approx(fmaf(x[2 * ii + 1], cs, neg_ref));
        sum += e0 + e1;
        own[ii] = pack_bf16x2(e0, e1);
      }
      l += sum;
      uint32_t pk[32];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) {
          const int word = 32 * h2 + ii;  // columns 2 word, 2 word + 1
          pk[ii] = (word >> 4) == warp ? own[word & 15] : 0u;
        }
        tmem_st32(tS + 128 * bsel + 32 * h2, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[bsel]);
    }
    // Epilogue of the segment: this warp's partial in slot 4 k + w.
    if (!__all_sync(0xFFFFFFFFu, dt_wait(&ctl->o_full, segs & 1u, ctl, p, kSiteDtSoftO))) return;
    if (!__all_sync(0xFFFFFFFFu, dt_wait(&ctl->pv_done, pv_n & 1u, ctl, p, kSiteDtSoftPv))) return;
    ++pv_n;
    tc_fence_after();
    const long long pair_first = static_cast<long long>(sg.pair) * p.tiles_per_pair;
    const int k = static_cast<int>(blockIdx.x - dt_owner(pair_first, p));
    const size_t slot0 = static_cast<size_t>(sg.pair) * p.kmax;  // kmax counts the four slots per CTA
    const size_t prow = (slot0 + 4 * k + warp) * p.rows + r;
#pragma unroll 1
    for (int cc = 0; cc < kD; cc += 32) {
      uint32_t ov[32];
      tmem_ld32(tO + cc, ov);
      tmem_wait_ld();
      if (valid) {
        float4* dst = reinterpret_cast<float4*>(p.part_acc + prow * kD + cc);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(ov[4 * i]), __uint_as_float(ov[4 * i + 1]),
                               __uint_as_float(ov[4 * i + 2]), __uint_as_float(ov[4 * i + 3]));
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->o_empty);
    if (valid) {
      p.part_ml[2 * prow] = m_used;
      p.part_ml[2 * prow + 1] = l;
    }
    // The pair's last contributor marks the slots after its own empty.
    if (sg.j1 == p.tiles_per_pair && valid) {
      for (int k2 = 4 * (k + 1) + warp; k2 < p.kmax; k2 += 4) {
        const size_t e = (slot0 + k2) * p.rows + r;
        p.part_ml[2 * e] = -CUDART_INF_F;
        p.part_ml[2 * e + 1] = 0.0f;
        float4* dst = reinterpret_cast<float4*>(p.part_acc + e * kD);
        for (int i = 0; i < kD / 4; ++i) dst[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
    }
    ++segs;
  }
}

template <int kD>
__global__ void __launch_bounds__(192, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeTcParams p) {
  using G = DecodeTcCfg<kD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DecodeTcCtl* ctl = reinterpret_cast<DecodeTcCtl*>(smem + G::kCtlOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  launch_dependents();  // the combine kernel may be scheduled; it waits for this grid
  // Rows R..127 of the query tile stay zero (the box fills rows 0..R-1).
  for (int i = threadIdx.x; i < G::kTileBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + G::kQOffset)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->s_full[b], 1);
      mbar_init(&ctl->p_full[b], 4);
    }
    mbar_init(&ctl->pv_done, 1);
    mbar_init(&ctl->o_full, 1);
    mbar_init(&ctl->o_empty, 4);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (warp == 4) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 5 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  if (warp < 4) {
    dt_softmax<kD>(p, ctl, tmem, warp, lane);
  } else if (warp == 4) {
    dt_mma<kD>(p, ctl, smem, tmem);
    __syncwarp();
  } else {
    if (lane == 0) dt_producer<kD>(&tm_q, &tm_k, &tm_v, p, ctl, smem);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, 512);
}

}  // namespace ea
