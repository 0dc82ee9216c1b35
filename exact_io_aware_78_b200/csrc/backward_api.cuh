// attn_bwd, attn_bwd_masked: the C entry points of the attention backward
// (declared in include/exactattn.h), included at the end of exactattn.cu,
// whose helpers (device_state, check_range, aligned, make_map and the
// process-wide options) they use.  They validate the arguments, take the
// per-row statistics' space (and with per-row key ranges the two tile
// tables) from the library's pool, and launch the kernels of
// attn_bwd_kernel.cuh on the caller's stream: with ranges the tile-range
// pre-pass of the forward and the key-tile table first, then the
// (-lse2, D) pass, the dK/dV kernel and the dQ kernel.

namespace {

template <int kD, bool kRanges>
int launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                    const ea::BwdParams& base, const DeviceState& ds, cudaStream_t stream) {
  using G = ea::BwdCfg<kD>;
  static std::atomic<bool> attr_done[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  const int rc = once_per_device(attr_done, dev, [] {
    if (cudaFuncSetAttribute(ea::attn_bwd_dkdv_sm100<kD, kRanges>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             G::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(ea::attn_bwd_dq_sm100<kD, kRanges>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             G::kSmemBytes) != cudaSuccess)
      return static_cast<int>(EA_ELAUNCH);
    // The warpgroups re-split the registers the block is launched with
    // (setmaxnreg); a block launched with fewer would wait there forever.
    cudaFuncAttributes a1, a2;
    if (cudaFuncGetAttributes(&a1, ea::attn_bwd_dkdv_sm100<kD, kRanges>) != cudaSuccess ||
        cudaFuncGetAttributes(&a2, ea::attn_bwd_dq_sm100<kD, kRanges>) != cudaSuccess ||
        a1.numRegs < G::kLaunchRegs || a2.numRegs < G::kLaunchRegs)
      return static_cast<int>(EA_ELAUNCH);
    return static_cast<int>(EA_OK);
  });
  if (rc != EA_OK) return rc;
  ea::BwdParams p = base;
  p.item_counter = base.item_counter;  // counters[0]: dK/dV items, counters[1]: dQ items (dynamic deal)
  p.num_work = p.B * p.Hkv * p.num_tiles;  // (batch, kv head, key tile)
  int grid = p.num_work < ds.num_sms ? p.num_work : ds.num_sms;
  if (g_max_ctas > 0 && grid > g_max_ctas) grid = g_max_ctas;
  ea::attn_bwd_dkdv_sm100<kD, kRanges><<<grid, G::kThreads, G::kSmemBytes, stream>>>(tq, tk, tv, tdo, p);
  if (cudaGetLastError() != cudaSuccess) return EA_ELAUNCH;
  p.item_counter = base.item_counter != nullptr ? base.item_counter + 1 : nullptr;
  p.num_work = p.B * p.Hq * p.num_tiles;  // (batch, query head, query tile)
  grid = p.num_work < ds.num_sms ? p.num_work : ds.num_sms;
  if (g_max_ctas > 0 && grid > g_max_ctas) grid = g_max_ctas;
  ea::attn_bwd_dq_sm100<kD, kRanges><<<grid, G::kThreads, G::kSmemBytes, stream>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ELAUNCH;
}

int backward_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                  void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int causal, int window,
                  const int* key_lo, const int* key_hi, float scale, int dtype, void* stream_ptr) {
  // ---- arguments that need no device
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return EA_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d < 1) return EA_EINVAL;
  if (Hq % Hkv != 0) return EA_EINVAL;
  if (causal != 0 && causal != 1) return EA_EINVAL;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return EA_EINVAL;
  if (dtype != EA_BF16 && dtype != EA_FP8_E4M3 && dtype != EA_FP32) return EA_EINVAL;
  if (dtype != EA_BF16) return EA_EUNSUPPORTED;
  if (d != 64 && d != 128) return EA_EUNSUPPORTED;
  if (static_cast<long long>(Hq) * N >= (1LL << 31) || static_cast<long long>(Hkv) * N >= (1LL << 31))
    return EA_EINVAL;
  const long long num_tiles = (N + 127) / 128;
  if (static_cast<long long>(B) * Hq * num_tiles > INT_MAX) return EA_EINVAL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return EA_EALIGN;

  // ---- device checks
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != EA_OK) return rc;
  const size_t q_bytes = static_cast<size_t>(B) * N * Hq * d * 2;
  const size_t kv_bytes = static_cast<size_t>(B) * N * Hkv * d * 2;
  if (check_range(q, q_bytes) || check_range(k, kv_bytes) || check_range(v, kv_bytes) || check_range(o, q_bytes) ||
      check_range(dout, q_bytes) || check_range(dq, q_bytes) || check_range(dk, kv_bytes) ||
      check_range(dv, kv_bytes) || check_range(lse, static_cast<size_t>(B) * Hq * N * 4))
    return EA_EINVAL;
  const bool ranges = key_lo != nullptr;
  if (ranges && (check_range(key_lo, static_cast<size_t>(B) * N * 4) ||
                 check_range(key_hi, static_cast<size_t>(B) * N * 4)))
    return EA_EINVAL;
  CUtensorMap tq, tk, tv, tdo;
  if (make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hq, N, B) ||
      make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, N, B) ||
      make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, N, B) ||
      make_map(&tdo, dout, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hq, N, B))
    return EA_EINVAL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_ptr);

  // ---- per-row statistics (-LSE log2 e, D), and with row ranges the two
  // tile tables and the two kernels' item counters (dynamic deal), in
  // stream-ordered pool scratch
  const long long rows = static_cast<long long>(B) * N * Hq;
  const size_t stats_bytes = static_cast<size_t>(rows) * sizeof(float2);
  const size_t table_bytes = static_cast<size_t>(B) * num_tiles * sizeof(int2);
  void* scratch = nullptr;
  if (cudaMallocFromPoolAsync(&scratch, stats_bytes + (ranges ? 2 * table_bytes + 2 * sizeof(int) : 0), ds->pool,
                              stream) != cudaSuccess)
    return EA_ENOMEM;
  float2* stats = static_cast<float2*>(scratch);
  int2* tile_kv = ranges ? reinterpret_cast<int2*>(static_cast<char*>(scratch) + stats_bytes) : nullptr;
  int2* tile_q = ranges ? tile_kv + static_cast<size_t>(B) * num_tiles : nullptr;
  int* counters = nullptr;
  // The dynamic deal numbers items past the CTA count; that stays in int.
  if (ranges && g_item_deal == 0 && static_cast<long long>(B) * Hq * num_tiles + ds->num_sms < INT_MAX)
    counters = reinterpret_cast<int*>(tile_q + static_cast<size_t>(B) * num_tiles);
  if (ranges) {
    ea::row_range_tiles_kernel<<<static_cast<unsigned>(B * num_tiles), 128, 0, stream>>>(
        key_lo, key_hi, tile_kv, nullptr, N, static_cast<int>(num_tiles), causal, window > 0 ? window : 0);
    const long long tt = static_cast<long long>(B) * num_tiles;
    ea::key_tile_queries_kernel<<<static_cast<unsigned>((tt + 127) / 128), 128, 0, stream>>>(
        tile_kv, tile_q, B, static_cast<int>(num_tiles), counters);
    if (cudaGetLastError() != cudaSuccess) {
      cudaFreeAsync(scratch, stream);
      return EA_ELAUNCH;
    }
  }
  const long long threads = rows * (d / 8);
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  if (d == 128)
    ea::bwd_prep_kernel<128><<<blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(o),
                                                        static_cast<const uint16_t*>(dout), lse, stats, B, Hq, N);
  else
    ea::bwd_prep_kernel<64><<<blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(o),
                                                       static_cast<const uint16_t*>(dout), lse, stats, B, Hq, N);
  rc = cudaGetLastError() == cudaSuccess ? EA_OK : EA_ELAUNCH;
  if (rc == EA_OK) {
    ea::BwdParams p{};
    p.stats = stats;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.err = ds->err;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.N = N;
    p.group = Hq / Hkv;
    p.causal = causal;
    p.window = window > 0 ? window : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.scale = scale;
    p.num_tiles = static_cast<int>(num_tiles);
    p.item_counter = counters;
    p.timeout_ns = g_timeout_ns;
    p.key_lo = key_lo;
    p.key_hi = key_hi;
    p.tile_kv = tile_kv;
    p.tile_q = tile_q;
    if (ranges)
      rc = d == 128 ? launch_backward<128, true>(tq, tk, tv, tdo, p, *ds, stream)
                    : launch_backward<64, true>(tq, tk, tv, tdo, p, *ds, stream);
    else
      rc = d == 128 ? launch_backward<128, false>(tq, tk, tv, tdo, p, *ds, stream)
                    : launch_backward<64, false>(tq, tk, tv, tdo, p, *ds, stream);
  }
  cudaFreeAsync(scratch, stream);
  return rc;
}

}  // namespace

extern "C" int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                        int causal, int window, float scale, int dtype, void* stream) {
  return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, causal, window, nullptr, nullptr, scale,
                       dtype, stream);
}

extern "C" int attn_bwd_masked(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                               int causal, int window, const int32_t* key_lo, const int32_t* key_hi, float scale,
                               int dtype, void* stream) {
  if (!key_lo || !key_hi) return EA_EINVAL;
  if (!aligned(key_lo, 4) || !aligned(key_hi, 4)) return EA_EALIGN;
  return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, causal, window, key_lo, key_hi, scale,
                       dtype, stream);
}
