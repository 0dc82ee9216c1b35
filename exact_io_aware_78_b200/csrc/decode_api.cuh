// attn_fwd_decode: the C entry point of the decode / split-KV forward
// (declared in include/exactattn.h), included inside the extern "C" block of
// exactattn.cu, whose helpers (device_state, check_range, aligned, g_encode)
// it uses.  Validates the arguments, splits the visible keys into ranges,
// takes the partial results' space from the library's pool and launches a
// key-range kernel and the combine kernel on the caller's stream: by default
// (num_splits == 0, g * Nq <= 32 rows) the tensor-core kernel of
// decode_tc_kernel.cuh over a stream-K split of all K/V tiles; with an
// explicit split count the CUDA-core kernel of decode_kernel.cuh.

// The combine kernel, launched as a programmatic dependent of the key-range
// kernel queued just before it: its blocks may be scheduled while that
// kernel finishes, and wait in-kernel for its completion before reading the
// partials, so the launch gap between the two disappears.
static int launch_combine(int d, unsigned blocks, const ea::DecodeParams& cp, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(32 * ea::kDecodeWarps);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = d == 128 ? cudaLaunchKernelEx(&cfg, ea::decode_combine_kernel<128>, cp)
                                 : cudaLaunchKernelEx(&cfg, ea::decode_combine_kernel<64>, cp);
  return e == cudaSuccess ? EA_OK : EA_ELAUNCH;
}

// Tensor map over q [B, Nq, Hq, d] with boxes of 128 bytes x `group` heads x
// Nq rows: one box is the query rows of one key/value head's group.
static int make_group_q_map(CUtensorMap* m, const void* base, int d, int Hq, int Nq, int B, int group) {
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(Nq),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(Hq) * d * 2,
                           static_cast<cuuint64_t>(Nq) * Hq * d * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(Nq), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? EA_OK : EA_EINVAL;
}

// The tensor-core path: stream-K over all (b, kv head) pairs' visible K/V
// tiles, one partial per pair a CTA touches, then the combine kernel.
static int decode_tc_launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                            int Nq, int Nk, int d, int causal, int window, float scale, DeviceState* ds,
                            cudaStream_t stream) {
  const int group = Hq / Hkv;
  const int rows = group * Nq;
  const int key_lo = window > 0 ? std::max(0, Nk - Nq - window + 1) : 0;  // no row sees a key before it
  const int key_tile_lo = key_lo / 128;
  const int tpp = (Nk + 127) / 128 - key_tile_lo;
  const long long pairs = static_cast<long long>(B) * Hkv;
  const long long total = pairs * tpp;
  const long long G = std::min<long long>(ds->num_sms, total);
  // slots per pair: four (one per softmax warp) for each of the most CTAs
  // whose ranges touch one pair
  auto owner = [&](long long x) { return ((x + 1) * G - 1) / total; };
  long long kmax = 1;
  for (long long pr = 0; pr < pairs; ++pr)
    kmax = std::max(kmax, owner((pr + 1) * tpp - 1) - owner(pr * tpp) + 1);
  kmax *= 4;
  if (pairs * kmax * rows >= (1LL << 31)) return EA_EINVAL;

  CUtensorMap tq, tk, tv;
  if (make_group_q_map(&tq, q, d, Hq, Nq, B, group) ||
      make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, Nk, B) ||
      make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, Nk, B))
    return EA_EINVAL;
  // the accumulators start on a 256-byte boundary (the kernel stores them as float4)
  const size_t ml_bytes = (static_cast<size_t>(pairs * kmax) * rows * 2 * sizeof(float) + 255) & ~size_t(255);
  const size_t acc_bytes = static_cast<size_t>(pairs * kmax) * rows * d * sizeof(float);
  void* scratch = nullptr;
  if (cudaMallocFromPoolAsync(&scratch, ml_bytes + acc_bytes, ds->pool, stream) != cudaSuccess) return EA_ENOMEM;

  ea::DecodeTcParams tp{};
  tp.part_ml = static_cast<float*>(scratch);
  tp.part_acc = reinterpret_cast<float*>(static_cast<char*>(scratch) + ml_bytes);
  tp.err = ds->err;
  tp.B = B;
  tp.Hq = Hq;
  tp.Hkv = Hkv;
  tp.Nq = Nq;
  tp.Nk = Nk;
  tp.group = group;
  tp.rows = rows;
  tp.causal = causal;
  tp.window = window > 0 ? window : 0;
  tp.scale_log2 = scale * 1.4426950408889634f;
  tp.key_tile_lo = key_tile_lo;
  tp.tiles_per_pair = tpp;
  tp.total_tiles = total;
  tp.kmax = static_cast<int>(kmax);
  tp.timeout_ns = g_timeout_ns;

  ea::DecodeParams cp{};
  cp.o = static_cast<__nv_bfloat16*>(o);
  cp.lse = lse;
  cp.part_ml = tp.part_ml;
  cp.part_acc = tp.part_acc;
  cp.B = B;
  cp.Hq = Hq;
  cp.Hkv = Hkv;
  cp.Nq = Nq;
  cp.Nk = Nk;
  cp.group = group;
  cp.rows = rows;
  cp.splits = static_cast<int>(kmax);

  auto kern = d == 128 ? ea::decode_tc_kernel<128> : ea::decode_tc_kernel<64>;
  const int smem = d == 128 ? ea::DecodeTcCfg<128>::kSmemBytes : ea::DecodeTcCfg<64>::kSmemBytes;
  int rc = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess ? EA_OK
                                                                                                   : EA_ELAUNCH;
  if (rc == EA_OK) {
    kern<<<static_cast<unsigned>(G), 192, smem, stream>>>(tq, tk, tv, tp);
    const unsigned comb_blocks = static_cast<unsigned>((pairs * rows + ea::kDecodeWarps - 1) / ea::kDecodeWarps);
    rc = cudaGetLastError() == cudaSuccess ? launch_combine(d, comb_blocks, cp, stream) : EA_ELAUNCH;
  }
  cudaFreeAsync(scratch, stream);
  return rc;
}

int attn_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                    int Nk, int d, int causal, int window, float scale, int dtype, int num_splits,
                    void* stream_ptr) {
  // ---- arguments that need no device
  if (!q || !k || !v || !o || !lse) return EA_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || d < 1 || num_splits < 0) return EA_EINVAL;
  if (Hq % Hkv != 0 || Nq > Nk) return EA_EINVAL;
  if (causal != 0 && causal != 1) return EA_EINVAL;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return EA_EINVAL;
  if (dtype != EA_BF16 && dtype != EA_FP8_E4M3 && dtype != EA_FP32) return EA_EINVAL;
  if (dtype != EA_BF16) return EA_EUNSUPPORTED;
  if (d != 64 && d != 128) return EA_EUNSUPPORTED;
  const int group = Hq / Hkv;
  // tensor-core path: up to 32 query rows per kv head; CUDA-core path (an
  // explicit split count): up to 8
  const long long nrows = static_cast<long long>(group) * Nq;
  if (nrows > ea::kDecodeTcMaxRows || (num_splits > 0 && nrows > ea::kDecodeMaxRows)) return EA_EUNSUPPORTED;
  if (static_cast<long long>(B) * Nk * Hkv >= (1LL << 40) || static_cast<long long>(B) * Hq * Nq >= (1LL << 31))
    return EA_EINVAL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return EA_EALIGN;

  // ---- device checks
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != EA_OK) return rc;
  if (check_range(q, static_cast<size_t>(B) * Nq * Hq * d * 2) ||
      check_range(k, static_cast<size_t>(B) * Nk * Hkv * d * 2) ||
      check_range(v, static_cast<size_t>(B) * Nk * Hkv * d * 2) ||
      check_range(o, static_cast<size_t>(B) * Nq * Hq * d * 2) || check_range(lse, static_cast<size_t>(B) * Hq * Nq * 4))
    return EA_EINVAL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_ptr);
  if (num_splits == 0)
    return decode_tc_launch(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, window, scale, ds, stream);

  // ---- the CUDA-core kernel for this head dim and row count (row capacity 1, 2, 4, 8)
  const int rows = group * Nq;
  const int cap = rows <= 1 ? 1 : rows <= 2 ? 2 : rows <= 4 ? 4 : 8;
  const size_t smem = static_cast<size_t>(ea::kDecodeWarps) * (cap * (d + 32) * sizeof(float) + 2 * 32 * (d * 2 + 16));
  auto split = d == 128 ? (cap == 1 ? ea::decode_split_kernel<128, 1> : cap == 2 ? ea::decode_split_kernel<128, 2>
                           : cap == 4 ? ea::decode_split_kernel<128, 4> : ea::decode_split_kernel<128, 8>)
                        : (cap == 1 ? ea::decode_split_kernel<64, 1> : cap == 2 ? ea::decode_split_kernel<64, 2>
                           : cap == 4 ? ea::decode_split_kernel<64, 4> : ea::decode_split_kernel<64, 8>);

  // ---- key ranges: the keys some row can see, [key_lo, Nk), in `num_splits`
  // ranges of whole 32-key batches (at most one per batch).
  const int key_lo = window > 0 ? std::max(0, Nk - Nq - window + 1) : 0;
  const long long len = Nk - key_lo;
  const long long batches = (len + 31) / 32;
  if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return EA_ELAUNCH;
  long long splits = num_splits;
  splits = std::max(1LL, std::min(splits, batches));
  const long long chunk = ((batches + splits - 1) / splits) * 32;
  splits = (len + chunk - 1) / chunk;  // <= the splits asked for
  const long long tasks = static_cast<long long>(B) * Hkv * splits;
  if (tasks * rows >= (1LL << 31)) return EA_EINVAL;

  ea::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.group = group;
  p.rows = rows;
  p.causal = causal;
  p.window = window > 0 ? window : 0;
  p.splits = static_cast<int>(splits);
  p.chunk = static_cast<int>(chunk);
  p.key_lo = key_lo;
  p.scale_log2 = scale * 1.4426950408889634f;

  // Partial results, stream-ordered from the library's pool.
  const size_t ml_bytes = (static_cast<size_t>(tasks) * rows * 2 * sizeof(float) + 255) & ~size_t(255);
  const size_t acc_bytes = static_cast<size_t>(tasks) * rows * d * sizeof(float);
  void* scratch = nullptr;
  if (cudaMallocFromPoolAsync(&scratch, ml_bytes + acc_bytes, ds->pool, stream) != cudaSuccess) return EA_ENOMEM;
  p.part_ml = static_cast<float*>(scratch);
  p.part_acc = reinterpret_cast<float*>(static_cast<char*>(scratch) + ml_bytes);

  const unsigned split_blocks = static_cast<unsigned>((tasks + ea::kDecodeWarps - 1) / ea::kDecodeWarps);
  const unsigned comb_blocks =
      static_cast<unsigned>((static_cast<long long>(B) * Hkv * rows + ea::kDecodeWarps - 1) / ea::kDecodeWarps);
  split<<<split_blocks, 32 * ea::kDecodeWarps, smem, stream>>>(p);
  rc = cudaGetLastError() == cudaSuccess ? launch_combine(d, comb_blocks, p, stream) : EA_ELAUNCH;
  cudaFreeAsync(scratch, stream);
  return rc;
}
