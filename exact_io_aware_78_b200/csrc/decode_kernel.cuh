// Decode / split-KV attention forward: a few query rows (Nq, at the end of
// the sequence) against a long key/value cache (Nk keys), bf16 in, bf16 out.
//
// What it computes (same exact attention as the prefill kernel): for query
// row i at position p = Nk - Nq + i (bottom-right alignment: the new tokens
// are the last ones of the sequence) and key/value head h / (Hq / Hkv),
//   O = softmax(scale * q K^T + mask) V,  LSE = natural-log log-sum-exp,
// with mask allowing keys j <= p (causal) and j > p - window (window > 0).
// Sources: the pages' softmax(Q K^T) V with a mask (Hacker News discussion,
// item 40939398; "Flash Attention" concept note, AS-IS diagram); the key
// range is split across workers whose partial results are combined with
// their normalisation factors, the method's blockwise combination ("Flash
// Attention" note, TO-BE diagram and "Tiling" section; FlashAttention quiz,
// question 4), as in the decoding work the pages list by title
// (FlashDecoding++).
//
// Design for B200: one query row per (b, head) and a long cache make this
// HBM-bound (about 4 FLOP per byte of K/V for a GQA group of 4), so the
// kernel streams each K/V row of a (batch, key/value head) exactly once, for
// all g * Nq query rows of its GQA group together, on the CUDA cores; no
// tensor-core tiles padded from a handful of rows to 128.
//   * split kernel: one warp per (b, kv head, key range).  Per batch of 32
//     keys each lane owns one key: it loads that K row with 16-byte loads
//     (a row is d contiguous bf16) and computes its dot products with the R
//     query rows (staged in shared memory, pre-scaled by scale * log2 e, read
//     by broadcast); the warp takes the batch maximum per row by shuffles,
//     rescales its running sums, and forms p = 2^(s - m).  For P V each lane
//     owns d / 32 output columns: it reads its slice of every V row of the
//     batch (the warp reads each row as one coalesced 2*d-byte segment) and
//     takes each key's p by shuffle.  At the end of its key range the warp
//     writes (m, l) and the unnormalised accumulator per row.
//   * combine kernel: one warp per output row merges the key ranges'
//     partial results: M = max m, L = sum l 2^(m - M),
//     O = sum acc 2^(m - M) / L, LSE = ln 2 * (M + log2 L).
#pragma once

#include <cstdint>
#include <type_traits>

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"
#include "decode_tc_kernel.cuh"  // the tensor-core key-range kernel (decode_tc_kernel)

namespace ea {

constexpr int kDecodeMaxRows = 8;     // g * Nq query rows per (b, kv head) of the CUDA-core kernel
constexpr int kDecodeWarps = 4;       // warps per block
constexpr int kCombineFast = 16;      // ranges the combine kernel loads all at once

struct DecodeParams {
  const __nv_bfloat16* q;  // [B, Nq, Hq, d]
  const __nv_bfloat16* k;  // [B, Nk, Hkv, d]
  const __nv_bfloat16* v;  // [B, Nk, Hkv, d]
  __nv_bfloat16* o;        // [B, Nq, Hq, d]
  float* lse;              // [B, Hq, Nq]
  float* part_ml;          // [tasks, R, 2]: m (log2 units), l
  float* part_acc;         // [tasks, R, d]: unnormalised accumulator
  int B, Hq, Hkv, Nq, Nk, group, rows;  // rows = group * Nq
  int causal, window;
  int splits;       // key ranges per (b, kv head)
  int chunk;        // keys per range (a multiple of 32)
  int key_lo;       // first key any row can see
  float scale_log2; // scale * log2(e)
};

// 16-byte asynchronous global->shared copy; src_bytes 0 writes zeros.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory"); }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int kD, int kRows>  // kRows: row capacity, p.rows <= kRows <= kDecodeMaxRows
__global__ void __launch_bounds__(32 * kDecodeWarps)
    decode_split_kernel(const DecodeParams p) {
  constexpr int kPerLane = kD / 32;  // output columns per lane (2 or 4: one or two f32 pairs)
  // shared memory: per warp the staged query rows [kRows][kD] (fp32, scaled)
  // and the batch's probabilities [32 keys][kRows]
  extern __shared__ float dec_smem[];
  launch_dependents();  // the combine kernel may be scheduled; it waits for this grid
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long task = static_cast<long long>(blockIdx.x) * kDecodeWarps + warp;
  const long long tasks = static_cast<long long>(p.B) * p.Hkv * p.splits;
  if (task >= tasks) return;  // whole warp
  // Consecutive warps take consecutive kv heads of the same batch and key
  // range, so a block reads neighbouring 2*d-byte pieces of the same key
  // rows (a key row of all heads is contiguous) at about the same time.
  const int hkv = static_cast<int>(task % p.Hkv);
  const int split = static_cast<int>((task / p.Hkv) % p.splits);
  const int b = static_cast<int>(task / (static_cast<long long>(p.Hkv) * p.splits));
  const int bk = b * p.Hkv + hkv;
  const long long part = static_cast<long long>(bk) * p.splits + split;  // partial-result slot
  const int R = p.rows;
  constexpr int kRowBytes = kD * 2 + 16;  // a staged K row, padded so lanes reading rows hit distinct banks
  constexpr int kWarpFloats = kRows * kD + 32 * kRows + 2 * 32 * kRowBytes / 4;
  float* qs = dec_smem + warp * kWarpFloats;
  float* ps = qs + kRows * kD;
  uint8_t* kbuf = reinterpret_cast<uint8_t*>(ps + 32 * kRows);  // two batches of 32 K rows

  // Stage this group's query rows (row r = head-in-group * Nq + i), scaled;
  // rows past R are zero.
  for (int e = lane; e < kRows * kD; e += 32) {
    const int r = e / kD, c = e - r * kD;
    float val = 0.0f;
    if (r < R) {
      const int hg = r / p.Nq, i = r - hg * p.Nq;
      const size_t src = ((static_cast<size_t>(b) * p.Nq + i) * p.Hq + hkv * p.group + hg) * kD + c;
      val = __bfloat162float(p.q[src]) * p.scale_log2;
    }
    qs[e] = val;
  }
  __syncwarp();

  const int k_begin = p.key_lo + split * p.chunk;
  const int k_end = min(p.Nk, k_begin + p.chunk);
  const size_t row_stride = static_cast<size_t>(p.Hkv) * kD;  // elements between consecutive keys
  const __nv_bfloat16* kbase = p.k + (static_cast<size_t>(b) * p.Nk * p.Hkv + hkv) * kD;
  const __nv_bfloat16* vbase = p.v + (static_cast<size_t>(b) * p.Nk * p.Hkv + hkv) * kD;

  float m[kRows], l[kRows];
  uint64_t acc[kRows][kPerLane / 2];  // f32 pairs
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    m[r] = -CUDART_INF_F;
    l[r] = 0.0f;
#pragma unroll
    for (int c = 0; c < kPerLane / 2; ++c) acc[r][c] = 0ull;
  }

  // Loads are software-pipelined: a batch's V slices are requested before
  // its scores are computed, and the next batch's K rows before its P V, so
  // each load's latency overlaps compute.
  using VSlice = typename std::conditional<kPerLane == 4, uint2, uint32_t>::type;
  // K rows of a batch are copied to shared memory by the whole warp, each
  // instruction covering two whole rows (coalesced), one batch ahead.
  constexpr int kChunks = kD * 2 / 16;  // 16-byte chunks per row
  auto load_k = [&](int kb, int buf) {
    uint8_t* dst = kbuf + buf * 32 * kRowBytes;
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = i * 32 + lane;
      const int row = c / kChunks, col = c - row * kChunks;
      const int jj = kb + row;
      const int js = jj < k_end ? jj : k_end - 1;  // a valid address; no bytes read past the range
      cp_async16(dst + row * kRowBytes + col * 16, kbase + static_cast<size_t>(js) * row_stride + col * 8,
                 jj < k_end ? 16u : 0u);
    }
    cp_async_commit();
  };
  if (k_begin < k_end) load_k(k_begin, 0);

  int buf = 0;
  for (int kb = k_begin; kb < k_end; kb += 32, buf ^= 1) {
    const int j = kb + lane;  // this lane's key
    const bool have = j < k_end;
    const int nk = min(32, k_end - kb);
    VSlice vw[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      if (t < nk)
        vw[t] = __ldg(reinterpret_cast<const VSlice*>(vbase + static_cast<size_t>(kb + t) * row_stride +
                                                      lane * kPerLane));
      else
        vw[t] = VSlice{};
    }
    if (kb + 32 < k_end) {
      load_k(kb + 32, buf ^ 1);
      cp_async_wait<1>();  // this batch's rows have landed; the next batch's may still be in flight
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint4* krow = reinterpret_cast<const uint4*>(kbuf + buf * 32 * kRowBytes + lane * kRowBytes);
    // ---- scores s_r = q_r . k_j (log2 units): this lane's K row, paired FMAs
    uint64_t s2[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) s2[r] = 0ull;
    {
#pragma unroll
      for (int c = 0; c < kD / 8; ++c) {
        const uint4 kw = krow[c];
        const uint64_t k0 = f2_pack(bf16_lo(kw.x), bf16_hi(kw.x));
        const uint64_t k1 = f2_pack(bf16_lo(kw.y), bf16_hi(kw.y));
        const uint64_t k2 = f2_pack(bf16_lo(kw.z), bf16_hi(kw.z));
        const uint64_t k3 = f2_pack(bf16_lo(kw.w), bf16_hi(kw.w));
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          const ulonglong2 qa = *reinterpret_cast<const ulonglong2*>(qs + r * kD + 8 * c);
          const ulonglong2 qb = *reinterpret_cast<const ulonglong2*>(qs + r * kD + 8 * c + 4);
          s2[r] = f2_fma(qa.x, k0, s2[r]);
          s2[r] = f2_fma(qa.y, k1, s2[r]);
          s2[r] = f2_fma(qb.x, k2, s2[r]);
          s2[r] = f2_fma(qb.y, k3, s2[r]);
        }
      }
    }
    // ---- mask, batch maximum, running rescale, p = 2^(s - m); p goes to
    // shared memory as [key][row] so P V reads one key's row set at once
    float pr[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      float s0, s1;
      f2_unpack(s2[r], s0, s1);
      float sr = s0 + s1;
      pr[r] = 0.0f;
      if (r >= R) continue;
      const int pos = p.Nk - p.Nq + (r % p.Nq);  // this row's query position
      const bool visible = (!p.causal || j <= pos) && (p.window <= 0 || j > pos - p.window);
      if (!have || !visible) sr = -CUDART_INF_F;
      float mb = sr;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, off));
      const float m_new = fmaxf(m[r], mb);
      const float ref = m_new == -CUDART_INF_F ? 0.0f : m_new;  // no visible key yet: nothing to scale
      const float alpha = exp2f(m[r] - ref);
      pr[r] = exp2f(sr - ref);
      l[r] = l[r] * alpha + pr[r];  // this lane's part of the row sum
      const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
      for (int c = 0; c < kPerLane / 2; ++c) acc[r][c] = f2_fma(acc[r][c], a2, 0ull);
      m[r] = m_new;
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) ps[lane * kRows + r] = pr[r];
    __syncwarp();
    // ---- O += P V over the batch: this lane's column slice of each V row
    // (the warp reads each row as one coalesced segment); keys past the
    // range have p = 0 and were not loaded
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      uint64_t v2[kPerLane / 2];
      if constexpr (kPerLane == 4) {
        v2[0] = f2_pack(bf16_lo(vw[t].x), bf16_hi(vw[t].x));
        v2[1] = f2_pack(bf16_lo(vw[t].y), bf16_hi(vw[t].y));
      } else {
        v2[0] = f2_pack(bf16_lo(vw[t]), bf16_hi(vw[t]));
      }
      float pt[kRows];
      if constexpr (kRows % 4 == 0) {
#pragma unroll
        for (int r = 0; r < kRows; r += 4) {
          const float4 q4 = *reinterpret_cast<const float4*>(ps + t * kRows + r);
          pt[r] = q4.x; pt[r + 1] = q4.y; pt[r + 2] = q4.z; pt[r + 3] = q4.w;
        }
      } else {
#pragma unroll
        for (int r = 0; r < kRows; ++r) pt[r] = ps[t * kRows + r];
      }
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const uint64_t p2 = f2_pack(pt[r], pt[r]);
#pragma unroll
        for (int c = 0; c < kPerLane / 2; ++c) acc[r][c] = f2_fma(p2, v2[c], acc[r][c]);
      }
    }
    __syncwarp();  // ps is rewritten by the next batch
  }

  // ---- this key range's partial result
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    if (r >= R) continue;
    float lr = l[r];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lr += __shfl_xor_sync(0xFFFFFFFFu, lr, off);
    const size_t pr_idx = static_cast<size_t>(part) * R + r;
    if (lane == 0) {
      p.part_ml[2 * pr_idx] = m[r];
      p.part_ml[2 * pr_idx + 1] = lr;
    }
    float* dst = p.part_acc + pr_idx * kD + lane * kPerLane;
#pragma unroll
    for (int c = 0; c < kPerLane / 2; ++c) {
      float x0, x1;
      f2_unpack(acc[r][c], x0, x1);
      dst[2 * c] = x0;
      dst[2 * c + 1] = x1;
    }
  }
}

template <int kD>
__global__ void __launch_bounds__(32 * kDecodeWarps) decode_combine_kernel(const DecodeParams p) {
  constexpr int kPerLane = kD / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kDecodeWarps + warp;  // (b, kv head, r)
  const long long rows = static_cast<long long>(p.B) * p.Hkv * p.rows;
  if (row >= rows) return;
  const int r = static_cast<int>(row % p.rows);
  const int bk = static_cast<int>(row / p.rows);
  const int b = bk / p.Hkv, hkv = bk - b * p.Hkv;
  const int hg = r / p.Nq, i = r - hg * p.Nq;
  const int h = hkv * p.group + hg;
  // The partials come from the key-range kernel queued just before this one
  // (a programmatic dependent launch: this grid may start early).
  grid_dependency_wait();

  // Ranges' weights computed across lanes (lane t handles ranges t, t + 32,
  // ...): M = max m over ranges with l > 0, then w = 2^(m - M) (0 for an
  // empty range) and L = sum l w; the accumulators are then summed with
  // loads that do not wait on any test.
  const size_t base = static_cast<size_t>(bk) * p.splits * p.rows + r;  // range s at base + s * rows
  float M = -CUDART_INF_F;
  float L = 0.0f, o[kPerLane];
#pragma unroll
  for (int c = 0; c < kPerLane; ++c) o[c] = 0.0f;
  if (p.splits <= kCombineFast) {
    // Up to 16 ranges: every range's accumulator slice is requested at once,
    // together with the (m, l) pairs, so the row costs about one memory
    // latency instead of three.
    float mv = -CUDART_INF_F, lv = 0.0f;
    if (lane < p.splits) {
      const size_t idx = base + static_cast<size_t>(lane) * p.rows;
      const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + 2 * idx);
      mv = ml.x;
      lv = ml.y;
    }
    float a[kCombineFast][kPerLane];
#pragma unroll
    for (int t = 0; t < kCombineFast; ++t) {
      if (t < p.splits) {
        const float* src = p.part_acc + (base + static_cast<size_t>(t) * p.rows) * kD + lane * kPerLane;
        if constexpr (kPerLane == 4) {
          const float4 v = *reinterpret_cast<const float4*>(src);
          a[t][0] = v.x, a[t][1] = v.y, a[t][2] = v.z, a[t][3] = v.w;
        } else {
#pragma unroll
          for (int c = 0; c < kPerLane; ++c) a[t][c] = src[c];
        }
      }
    }
    M = lv > 0.0f ? mv : -CUDART_INF_F;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, off));
    const float w = (lv > 0.0f && M != -CUDART_INF_F) ? exp2f(mv - M) : 0.0f;
    L = lv > 0.0f ? lv * w : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, off);
#pragma unroll
    for (int t = 0; t < kCombineFast; ++t) {
      const float wt = __shfl_sync(0xFFFFFFFFu, w, t);
      if (t < p.splits) {
#pragma unroll
        for (int c = 0; c < kPerLane; ++c) o[c] += wt * a[t][c];
      }
    }
  } else {  // more ranges: weights first, then the accumulators 32 ranges at a time
    for (int s = lane; s < p.splits; s += 32) {
      const size_t idx = base + static_cast<size_t>(s) * p.rows;
      if (p.part_ml[2 * idx + 1] > 0.0f) M = fmaxf(M, p.part_ml[2 * idx]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, off));
    if (M != -CUDART_INF_F) {
      for (int s0 = 0; s0 < p.splits; s0 += 32) {
        float w = 0.0f;
        const int s = s0 + lane;
        if (s < p.splits) {
          const size_t idx = base + static_cast<size_t>(s) * p.rows;
          const float ls = p.part_ml[2 * idx + 1];
          w = ls > 0.0f ? exp2f(p.part_ml[2 * idx] - M) : 0.0f;
          L += ls > 0.0f ? ls * w : 0.0f;
        }
        const int n = min(32, p.splits - s0);
#pragma unroll 8
        for (int t = 0; t < n; ++t) {
          const float wt = __shfl_sync(0xFFFFFFFFu, w, t);
          const float* src = p.part_acc + (base + static_cast<size_t>(s0 + t) * p.rows) * kD + lane * kPerLane;
#pragma unroll
          for (int c = 0; c < kPerLane; ++c) o[c] += wt * src[c];
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, off);
    }
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
  __nv_bfloat16* dst = p.o + ((static_cast<size_t>(b) * p.Nq + i) * p.Hq + h) * kD + lane * kPerLane;
#pragma unroll
  for (int c = 0; c < kPerLane; ++c) dst[c] = __float2bfloat16_rn(o[c] * inv);
  if (lane == 0)
    p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.Nq + i] =
        L > 0.0f ? (M + log2f(L)) * 0.69314718055994531f : -CUDART_INF_F;
}

}  // namespace ea
