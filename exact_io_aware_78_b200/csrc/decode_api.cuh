// attn_fwd_decode: the C entry point of the decode / split-KV forward
// (declared in include/exactattn.h), included inside the extern "C" block of
// exactattn.cu, whose helpers (device_state, check_range, aligned) it uses.
// Validates the arguments, picks the key-range kernel for the head dim and
// row count, splits the visible keys into ranges, takes the partial results'
// space from the library's pool and launches the key-range and combine
// kernels of decode_kernel.cuh on the caller's stream.

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
  if (static_cast<long long>(group) * Nq > ea::kDecodeMaxRows) return EA_EUNSUPPORTED;
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

  // ---- the kernel for this head dim and row count (row capacity 1, 2, 4, 8)
  const int rows = group * Nq;
  const int cap = rows <= 1 ? 1 : rows <= 2 ? 2 : rows <= 4 ? 4 : 8;
  const size_t smem = static_cast<size_t>(ea::kDecodeWarps) * (cap * (d + 32) * sizeof(float) + 2 * 32 * (d * 2 + 16));
  auto split = d == 128 ? (cap == 1 ? ea::decode_split_kernel<128, 1> : cap == 2 ? ea::decode_split_kernel<128, 2>
                           : cap == 4 ? ea::decode_split_kernel<128, 4> : ea::decode_split_kernel<128, 8>)
                        : (cap == 1 ? ea::decode_split_kernel<64, 1> : cap == 2 ? ea::decode_split_kernel<64, 2>
                           : cap == 4 ? ea::decode_split_kernel<64, 4> : ea::decode_split_kernel<64, 8>);

  // ---- key ranges: the keys some row can see, [key_lo, Nk), in `splits`
  // ranges of whole 32-key batches; by default as many ranges as fit the
  // GPU's resident warps in one wave (rounded down, so no task waits for a
  // second wave), none shorter than four batches.
  const int key_lo = window > 0 ? std::max(0, Nk - Nq - window + 1) : 0;
  const long long len = Nk - key_lo;
  const long long batches = (len + 31) / 32;
  if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return EA_ELAUNCH;
  long long splits = num_splits;
  if (splits == 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, split, 32 * ea::kDecodeWarps, smem) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    const long long warps = static_cast<long long>(per_sm) * ea::kDecodeWarps * ds->num_sms;
    const long long pairs = static_cast<long long>(B) * Hkv;
    splits = std::max(1LL, std::min(warps / pairs, batches / 4));
  }
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
  const size_t ml_bytes = static_cast<size_t>(tasks) * rows * 2 * sizeof(float);
  const size_t acc_bytes = static_cast<size_t>(tasks) * rows * d * sizeof(float);
  void* scratch = nullptr;
  if (cudaMallocFromPoolAsync(&scratch, ml_bytes + acc_bytes, ds->pool, stream) != cudaSuccess) return EA_ENOMEM;
  p.part_ml = static_cast<float*>(scratch);
  p.part_acc = reinterpret_cast<float*>(static_cast<char*>(scratch) + ml_bytes);

  const unsigned split_blocks = static_cast<unsigned>((tasks + ea::kDecodeWarps - 1) / ea::kDecodeWarps);
  const unsigned comb_blocks =
      static_cast<unsigned>((static_cast<long long>(B) * Hkv * rows + ea::kDecodeWarps - 1) / ea::kDecodeWarps);
  split<<<split_blocks, 32 * ea::kDecodeWarps, smem, stream>>>(p);
  if (cudaGetLastError() == cudaSuccess) {
    if (d == 128)
      ea::decode_combine_kernel<128><<<comb_blocks, 32 * ea::kDecodeWarps, 0, stream>>>(p);
    else
      ea::decode_combine_kernel<64><<<comb_blocks, 32 * ea::kDecodeWarps, 0, stream>>>(p);
  }
  rc = cudaGetLastError() == cudaSuccess ? EA_OK : EA_ELAUNCH;
  cudaFreeAsync(scratch, stream);
  return rc;
}
