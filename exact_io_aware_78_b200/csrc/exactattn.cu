// exactattn.cu -- host side of the C ABI declared in include/exactattn.h:
// argument validation, per-device state, TMA tensor-map encoding, the fp32
// split pre-pass, and the launch of the sm_100a attention kernel.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_fwd_kernel.cuh"
#include "attn_bwd_kernel.cuh"
#include "decode_kernel.cuh"
#include "exactattn.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kAbiVersion = 10000;  // 1.0.0

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int* err = nullptr;             // device error word
  cudaMemPool_t pool = nullptr;   // stream-ordered scratch for the fp32 split operands
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
PFN_cuMemGetAddressRange_v3020 g_addr_range = nullptr;

// attn_fwd_fp32_noalloc's per-device set-up: the device address of its
// static scratch array (looked up by the first call on each device and
// forgotten by attn_shutdown, which also ends that set-up) and the SM count.
std::mutex g_noalloc_mutex;
uint8_t* g_noalloc_ptr[kMaxDevices] = {};
int g_noalloc_sms[kMaxDevices] = {};

// Options (attn_set_option).
unsigned long long g_timeout_ns = 2000000000ull;
int g_max_ctas = 0;
int g_order = 0;
int g_item_deal = 0;
int g_skip_arrive_once = 0;


// The two driver entry points, looked up once per process (every path that
// needs them goes through here, so they are published exactly once and read
// without a lock afterwards).
std::once_flag g_entry_once;
int g_entry_rc = EA_ECUDA;

int load_driver_entry_points() {
  std::call_once(g_entry_once, [] {
    cudaDriverEntryPointQueryResult q1, q2;
    void* f1 = nullptr;
    void* f2 = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || f1 == nullptr)
      return;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || f2 == nullptr)
      return;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f1);
    g_addr_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(f2);
    g_entry_rc = EA_OK;
  });
  return g_entry_rc;
}

// One-time, per-device set-up of a kernel's launch attributes.  The flag is
// read without the lock once it is set; the set-up itself runs under a lock,
// so concurrent first calls on one device perform it once and none launches
// before it has finished.
std::mutex g_attr_mutex;

template <class F>
int once_per_device(std::atomic<bool>* done, int dev, F&& setup) {
  if (done[dev].load(std::memory_order_acquire)) return EA_OK;
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  if (done[dev].load(std::memory_order_relaxed)) return EA_OK;
  const int rc = setup();
  if (rc == EA_OK) done[dev].store(true, std::memory_order_release);
  return rc;
}

// Per-device state, created on first use with the device current.
int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EA_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return EA_EUNSUPPORTED;
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!s.ready) {
      int rc = load_driver_entry_points();
      if (rc != EA_OK) return rc;
      int major = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return EA_ECUDA;
      if (major != 10) return EA_EUNSUPPORTED;  // built for sm_100a only
      if (cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return EA_ECUDA;
      if (cudaMalloc(&s.err, sizeof(int)) != cudaSuccess) return EA_ENOMEM;
      if (cudaMemset(s.err, 0, sizeof(int)) != cudaSuccess) return EA_ECUDA;
      // A library-owned pool that keeps its memory between calls, so the
      // per-call scratch of the fp32 path is a stream-ordered sub-allocation
      // rather than a fresh mapping.
      cudaMemPoolProps props{};
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      if (cudaMemPoolCreate(&s.pool, &props) != cudaSuccess) return EA_ENOMEM;
      uint64_t keep = UINT64_MAX;
      if (cudaMemPoolSetAttribute(s.pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) return EA_ECUDA;
      s.ready = true;
    }
  }
  *out = &s;
  return EA_OK;
}

// The buffer [p, p + bytes) must lie inside one device allocation of the
// current context (this rejects host pointers and most size mistakes before
// any device access is queued).
int check_range(const void* p, size_t bytes) {
  if (p == nullptr) return EA_EINVAL;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (g_addr_range(&base, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS) return EA_EINVAL;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  if (a + bytes > static_cast<uintptr_t>(base) + size) return EA_EINVAL;
  return EA_OK;
}

// Tensor map over a [B, N, H, d] tensor, 128-byte-wide boxes of 128 rows of
// one head, 128-byte swizzle (the layout the tcgen05 descriptors expect).
int make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int d, int H, int N, int B) {
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * esize, static_cast<cuuint64_t>(H) * d * esize,
                           static_cast<cuuint64_t>(N) * H * d * esize};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / esize), 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? EA_OK : EA_EINVAL;
}

template <class C, bool kRanges>
int launch_variant(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const ea::FwdParams& p,
                   const DeviceState& ds, cudaStream_t stream) {
  static std::atomic<bool> attr_done[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  const int rc = once_per_device(attr_done, dev, [] {
    if (cudaFuncSetAttribute(ea::attn_fwd_sm100<C, kRanges>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess)
      return static_cast<int>(EA_ELAUNCH);
    // The warpgroups re-split the registers the block is launched with
    // (setmaxnreg); a block launched with fewer than the split assumes would
    // wait in setmaxnreg forever, so refuse to launch it.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, ea::attn_fwd_sm100<C, kRanges>) != cudaSuccess || fa.numRegs < C::kLaunchRegs)
      return static_cast<int>(EA_ELAUNCH);
    return static_cast<int>(EA_OK);
  });
  if (rc != EA_OK) return rc;
  int grid = p.num_work < ds.num_sms ? p.num_work : ds.num_sms;
  if (g_max_ctas > 0 && grid > g_max_ctas) grid = g_max_ctas;
  ea::attn_fwd_sm100<C, kRanges><<<grid, C::kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ELAUNCH;
}

// The kernel variant with per-row key ranges is a separate instantiation,
// so the plain causal / window kernel carries none of its code.
template <class C>
int launch_attention(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const ea::FwdParams& p,
                     const DeviceState& ds, cudaStream_t stream) {
  return p.tile_kv != nullptr ? launch_variant<C, true>(tq, tk, tv, p, ds, stream)
                              : launch_variant<C, false>(tq, tk, tv, p, ds, stream);
}

// fp32 -> (hi, lo) bf16 split.  x = hi + lo + O(2^-17 |x|); the attention
// kernel then sees Q' = [hi, hi, lo], K' = [hi, lo, hi] (so that
// Q' K'^T = Qh Kh^T + Qh Kl^T + Ql Kh^T) and V' = [hi, lo] (so that
// P V' = [P Vh, P Vl], summed in the epilogue).
struct SplitJob {
  const float* x;
  uint16_t* y;
  long long rows;
};

// One launch splits Q, K and V: a grid-stride loop over groups of 8
// consecutive elements of 64-wide rows, Q's groups first, then K's, then V's.
__global__ void split_fp32_kernel(SplitJob q, SplitJob k, SplitJob v) {
  const long long gq = q.rows * 8, gk = k.rows * 8;
  const long long groups = gq + gk + v.rows * 8;
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < groups;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int pattern = g < gq ? 0 : (g < gq + gk ? 1 : 2);  // 0: Q, 1: K, 2: V
    const float* x = pattern == 0 ? q.x : (pattern == 1 ? k.x : v.x);
    uint16_t* y = pattern == 0 ? q.y : (pattern == 1 ? k.y : v.y);
    const long long gl = g - (pattern == 0 ? 0 : (pattern == 1 ? gq : gq + gk));
    const long long row = gl >> 3;
    const int col = static_cast<int>(gl & 7) * 8;
    const float4* src = reinterpret_cast<const float4*>(x + row * 64 + col);
    const float4 a = src[0], b = src[1];
    const float vals[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint16_t hi[8], lo[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat16 h = __float2bfloat16_rn(vals[i]);
      const __nv_bfloat16 l = __float2bfloat16_rn(vals[i] - __bfloat162float(h));
      hi[i] = *reinterpret_cast<const uint16_t*>(&h);
      lo[i] = *reinterpret_cast<const uint16_t*>(&l);
    }
    const uint4 H = make_uint4(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16), hi[4] | (hi[5] << 16),
                               hi[6] | (hi[7] << 16));
    const uint4 L = make_uint4(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16), lo[4] | (lo[5] << 16),
                               lo[6] | (lo[7] << 16));
    if (pattern == 2) {
      uint16_t* dst = y + row * 128 + col;
      *reinterpret_cast<uint4*>(dst) = H;
      *reinterpret_cast<uint4*>(dst + 64) = L;
    } else {
      uint16_t* dst = y + row * 192 + col;
      *reinterpret_cast<uint4*>(dst) = H;
      *reinterpret_cast<uint4*>(dst + 64) = pattern == 0 ? H : L;
      *reinterpret_cast<uint4*>(dst + 128) = pattern == 0 ? L : H;
    }
  }
}

int launch_split(SplitJob q, SplitJob k, SplitJob v, int num_sms, cudaStream_t stream) {
  const long long groups = (q.rows + k.rows + v.rows) * 8;
  long long blocks = (groups + 255) / 256;
  if (blocks > 8LL * num_sms) blocks = 8LL * num_sms;
  if (blocks < 1) blocks = 1;
  split_fp32_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(q, k, v);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ELAUNCH;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int forward_launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, int causal, int window, const int* key_lo, const int* key_hi, const int2* tile_kv,
                   const int* item_order, int* item_counter, int num_qtiles, float scale, int dtype,
                   const float* q_scale, const float* k_scale, const float* v_scale, DeviceState* ds,
                   cudaStream_t stream);

// The forward behind attn_fwd (key_lo == key_hi == null) and attn_fwd_masked:
// argument checks, the per-tile range pre-pass when row ranges are given,
// then forward_launch.
int forward_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                 int d, int causal, int window, const int* key_lo, const int* key_hi, float scale, int dtype,
                 const float* q_scale, const float* k_scale, const float* v_scale, void* stream_ptr) {
  // ---- arguments that need no device
  if (!q || !k || !v || !o || !lse) return EA_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d < 1) return EA_EINVAL;
  if (Hq % Hkv != 0) return EA_EINVAL;
  if (causal != 0 && causal != 1) return EA_EINVAL;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return EA_EINVAL;
  if (dtype != EA_BF16 && dtype != EA_FP8_E4M3 && dtype != EA_FP32) return EA_EINVAL;
  const bool fp8 = dtype == EA_FP8_E4M3;
  if (fp8 != (q_scale != nullptr) || fp8 != (k_scale != nullptr) || fp8 != (v_scale != nullptr))
    return EA_EINVAL;
  if (static_cast<long long>(Hq) * N >= (1LL << 31) || static_cast<long long>(Hkv) * N >= (1LL << 31))
    return EA_EINVAL;
  const long long num_qblk = (N + 255) / 256;
  if (static_cast<long long>(B) * Hq * num_qblk > INT_MAX) return EA_EINVAL;
  if (dtype == EA_FP32) {
    if (d != 64) return EA_EUNSUPPORTED;
  } else if (d != 64 && d != 128) {
    return EA_EUNSUPPORTED;
  }
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return EA_EALIGN;
  if (fp8 && (!aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4))) return EA_EALIGN;

  // ---- device checks
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != EA_OK) return rc;
  const size_t esize = dtype == EA_FP32 ? 4 : (fp8 ? 1 : 2);
  const size_t q_bytes = static_cast<size_t>(B) * N * Hq * d * esize;
  const size_t kv_bytes = static_cast<size_t>(B) * N * Hkv * d * esize;
  const size_t o_bytes = static_cast<size_t>(B) * N * Hq * d * (dtype == EA_FP32 ? 4 : 2);
  const size_t lse_bytes = static_cast<size_t>(B) * Hq * N * 4;
  if (check_range(q, q_bytes) || check_range(k, kv_bytes) || check_range(v, kv_bytes) ||
      check_range(o, o_bytes) || check_range(lse, lse_bytes))
    return EA_EINVAL;
  if (fp8 && (check_range(q_scale, Hq * 4) || check_range(k_scale, Hkv * 4) || check_range(v_scale, Hkv * 4)))
    return EA_EINVAL;
  const bool ranges = key_lo != nullptr;
  const long long num_qtiles = (N + 127) / 128;
  if (ranges && (check_range(key_lo, static_cast<size_t>(B) * N * 4) ||
                 check_range(key_hi, static_cast<size_t>(B) * N * 4)))
    return EA_EINVAL;

  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_ptr);
  // Per-row key ranges: reduce them to a K/V tile range per 128-row query
  // tile (the same pre-pass zeroes the item counter of the dynamic deal),
  // or rank the (batch, query block) pairs by cost (stream-ordered scratch
  // from the pool, freed after the launch).
  int2* tile_kv = nullptr;
  int* order = nullptr;
  int* counter = nullptr;
  if (ranges) {
    const long long pairs = static_cast<long long>(B) * num_qblk;
    const size_t tb = static_cast<size_t>(B) * num_qtiles * sizeof(int2);
    const size_t ob = static_cast<size_t>(pairs) * sizeof(int);
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, tb + ob + sizeof(int), ds->pool, stream) != cudaSuccess) return EA_ENOMEM;
    tile_kv = static_cast<int2*>(scratch);
    // The dynamic deal numbers items past the CTA count; that stays in int.
    if (g_order == 0 && g_item_deal == 0 && B * Hq * num_qblk + ds->num_sms < INT_MAX)
      counter = reinterpret_cast<int*>(static_cast<char*>(scratch) + tb + ob);
    ea::row_range_tiles_kernel<<<static_cast<unsigned>(B * num_qtiles), 128, 0, stream>>>(
        key_lo, key_hi, tile_kv, counter, N, static_cast<int>(num_qtiles), causal, window > 0 ? window : 0);
    rc = cudaGetLastError() == cudaSuccess ? EA_OK : EA_ELAUNCH;
    if (rc == EA_OK && pairs <= ea::kOrderMaxPairs && g_order == 2) {
      int pow2 = 1;
      while (pow2 < pairs) pow2 <<= 1;
      const size_t smem = static_cast<size_t>(pow2) * sizeof(unsigned long long);
      static std::atomic<bool> attr_done[kMaxDevices];
      int dev = 0;
      cudaGetDevice(&dev);
      rc = once_per_device(attr_done, dev, [] {
        return cudaFuncSetAttribute(ea::order_items_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    ea::kOrderMaxPairs * static_cast<int>(sizeof(unsigned long long))) == cudaSuccess
                   ? static_cast<int>(EA_OK)
                   : static_cast<int>(EA_ELAUNCH);
      });
      if (rc == EA_OK) {
        order = reinterpret_cast<int*>(static_cast<char*>(scratch) + tb);
        ea::order_items_kernel<<<1, 1024, smem, stream>>>(tile_kv, order, static_cast<int>(pairs),
                                                          static_cast<int>(num_qblk), static_cast<int>(num_qtiles),
                                                          pow2);
        if (cudaGetLastError() != cudaSuccess) rc = EA_ELAUNCH;
      }
    }
    if (rc != EA_OK) {
      cudaFreeAsync(scratch, stream);
      return rc;
    }
  }
  rc = forward_launch(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, window, key_lo, key_hi, tile_kv, order, counter,
                      static_cast<int>(num_qtiles), scale, dtype, q_scale, k_scale, v_scale, ds, stream);
  if (tile_kv) cudaFreeAsync(tile_kv, stream);
  return rc;
}

int forward_launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, int causal, int window, const int* key_lo, const int* key_hi, const int2* tile_kv,
                   const int* item_order, int* item_counter, int num_qtiles, float scale, int dtype,
                   const float* q_scale, const float* k_scale, const float* v_scale, DeviceState* ds,
                   cudaStream_t stream) {
  const bool fp8 = dtype == EA_FP8_E4M3;
  const long long num_qblk = (N + 255) / 256;
  int rc = EA_OK;
  ea::FwdParams p{};
  p.key_lo = key_lo;
  p.key_hi = key_hi;
  p.tile_kv = tile_kv;
  p.item_order = item_order;
  p.item_counter = item_counter;
  p.num_qtiles = num_qtiles;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.o = o;
  p.lse = lse;
  p.err = ds->err;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.causal = causal;
  p.window = window > 0 ? window : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_qblk = static_cast<int>(num_qblk);
  p.num_work = static_cast<int>(B * Hq * num_qblk);
  p.order = g_order == 1 ? 1 : 0;
  p.skip_first_kv = g_skip_arrive_once;
  p.timeout_ns = g_timeout_ns;
  g_skip_arrive_once = 0;

  CUtensorMap tq, tk, tv;
  if (dtype == EA_BF16) {
    if (make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hq, N, B) ||
        make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, N, B) ||
        make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, N, B))
      return EA_EINVAL;
    if (d == 128)
      return launch_attention<ea::KernelCfg<2, 128, 128, ea::kOutBf16>>(tq, tk, tv, p, *ds, stream);
    return launch_attention<ea::KernelCfg<2, 64, 64, ea::kOutBf16>>(tq, tk, tv, p, *ds, stream);
  }
  if (fp8) {
    if (make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, Hq, N, B) ||
        make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, Hkv, N, B) ||
        make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, Hkv, N, B))
      return EA_EINVAL;
    if (d == 128)
      return launch_attention<ea::KernelCfg<1, 128, 128, ea::kOutBf16>>(tq, tk, tv, p, *ds, stream);
    return EA_EUNSUPPORTED;  // e4m3 rows must be 128 bytes (d = 128)
  }
  // EA_FP32, d == 64: split into bf16 parts in stream-ordered scratch.
  const long long q_rows = static_cast<long long>(B) * N * Hq;
  const long long kv_rows = static_cast<long long>(B) * N * Hkv;
  const size_t sq = static_cast<size_t>(q_rows) * 192 * 2;
  const size_t sk = static_cast<size_t>(kv_rows) * 192 * 2;
  const size_t sv = static_cast<size_t>(kv_rows) * 128 * 2;
  void* scratch = nullptr;
  if (cudaMallocFromPoolAsync(&scratch, sq + sk + sv, ds->pool, stream) != cudaSuccess) return EA_ENOMEM;
  uint16_t* qs = static_cast<uint16_t*>(scratch);
  uint16_t* ks = reinterpret_cast<uint16_t*>(static_cast<char*>(scratch) + sq);
  uint16_t* vs = reinterpret_cast<uint16_t*>(static_cast<char*>(scratch) + sq + sk);
  rc = launch_split({static_cast<const float*>(q), qs, q_rows}, {static_cast<const float*>(k), ks, kv_rows},
                    {static_cast<const float*>(v), vs, kv_rows}, ds->num_sms, stream);
  if (rc == EA_OK) {
    if (make_map(&tq, qs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 192, Hq, N, B) ||
        make_map(&tk, ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 192, Hkv, N, B) ||
        make_map(&tv, vs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, Hkv, N, B))
      rc = EA_EINVAL;
  }
  if (rc == EA_OK) rc = launch_attention<ea::KernelCfg<2, 192, 128, ea::kOutF32Split>>(tq, tk, tv, p, *ds, stream);
  cudaFreeAsync(scratch, stream);
  return rc;
}

}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N, int d,
             int causal, int window, float scale, int dtype, const float* q_scale, const float* k_scale,
             const float* v_scale, void* stream) {
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, window, nullptr, nullptr, scale, dtype, q_scale,
                      k_scale, v_scale, stream);
}

int attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                    int d, int causal, int window, const int32_t* key_lo, const int32_t* key_hi, float scale,
                    int dtype, const float* q_scale, const float* k_scale, const float* v_scale, void* stream) {
  if (!key_lo || !key_hi) return EA_EINVAL;
  if (!aligned(key_lo, 4) || !aligned(key_hi, 4)) return EA_EALIGN;
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, window, key_lo, key_hi, scale, dtype, q_scale,
                      k_scale, v_scale, stream);
}

int attn_get_last_error(void* stream_ptr, int* device_code, int* site) {
  if (device_code) *device_code = 0;
  if (site) *site = 0;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != EA_OK) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream_ptr)) != cudaSuccess) return EA_ECUDA;
  int word = 0;
  if (cudaMemcpy(&word, ds->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return EA_ECUDA;
  if (word == 0) return EA_OK;
  if (cudaMemset(ds->err, 0, sizeof(int)) != cudaSuccess) return EA_ECUDA;
  if (device_code) *device_code = word >> 16;
  if (site) *site = word & 0xFFFF;
  return EA_EDEVICE_TIMEOUT;
}

const char* attn_status_string(int status) {
  switch (status) {
    case EA_OK: return "EA_OK";
    case EA_EINVAL: return "EA_EINVAL: invalid argument";
    case EA_EUNSUPPORTED: return "EA_EUNSUPPORTED: no kernel for this request";
    case EA_EALIGN: return "EA_EALIGN: pointer not 16-byte aligned";
    case EA_ELAUNCH: return "EA_ELAUNCH: kernel launch failed";
    case EA_EDEVICE_TIMEOUT: return "EA_EDEVICE_TIMEOUT: a device pipeline wait ran past its limit";
    case EA_ECUDA: return "EA_ECUDA: CUDA error";
    case EA_ENOMEM: return "EA_ENOMEM: out of device memory";
    default: return "unknown status";
  }
}

int attn_set_option(int option, long long value) {
  switch (option) {
    case EA_OPT_WAIT_TIMEOUT_NS:
      if (value < 1000) return EA_EINVAL;
      g_timeout_ns = static_cast<unsigned long long>(value);
      return EA_OK;
    case EA_OPT_MAX_CTAS:
      if (value < 0 || value > INT_MAX) return EA_EINVAL;
      g_max_ctas = static_cast<int>(value);
      return EA_OK;
    case EA_OPT_SCHEDULE_ORDER:
      if (value < 0 || value > 2) return EA_EINVAL;
      g_order = static_cast<int>(value);
      return EA_OK;
    case EA_OPT_SKIP_ARRIVE_ONCE:
      if (value != 0 && value != 1) return EA_EINVAL;
      g_skip_arrive_once = static_cast<int>(value);
      return EA_OK;
    case EA_OPT_ITEM_DEAL:
      if (value != 0 && value != 1) return EA_EINVAL;
      g_item_deal = static_cast<int>(value);
      return EA_OK;

    default:
      return EA_EINVAL;
  }
}

int attn_shutdown(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  {
    // attn_fwd_fp32_noalloc looks its array's address up again on its next
    // call (the address does not outlive a context the caller may reset).
    std::lock_guard<std::mutex> nlock(g_noalloc_mutex);
    for (int dev = 0; dev < kMaxDevices; ++dev) {
      g_noalloc_ptr[dev] = nullptr;
      g_noalloc_sms[dev] = 0;
    }
  }
  int rc = EA_OK;
  int prev = 0;
  cudaGetDevice(&prev);
  for (int dev = 0; dev < kMaxDevices; ++dev) {
    DeviceState& s = g_dev[dev];
    if (!s.ready) continue;
    cudaSetDevice(dev);
    if (cudaDeviceSynchronize() != cudaSuccess) rc = EA_ECUDA;
    if (cudaFree(s.err) != cudaSuccess) rc = EA_ECUDA;
    if (s.pool && cudaMemPoolDestroy(s.pool) != cudaSuccess) rc = EA_ECUDA;
    s = DeviceState{};
  }
  cudaSetDevice(prev);
  return rc;
}

int attn_version(void) { return kAbiVersion; }

#include "decode_api.cuh"  // attn_fwd_decode

}  // extern "C"

// ---------------------------------------------------------------------------
// attn_fwd_fp32_noalloc: the fp32 forward with its split operands in a
// statically allocated device array instead of pool scratch.
namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[EA_NOALLOC_SCRATCH_BYTES];

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Once per device, with that device current: the array's device address
// (host code must not use the symbol itself as a device pointer).
int noalloc_setup(int dev, uint8_t** base, int* num_sms) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] != nullptr) {
    *base = g_noalloc_ptr[dev];
    *num_sms = g_noalloc_sms[dev];
    return EA_OK;
  }
  int rc = load_driver_entry_points();
  if (rc != EA_OK) return rc;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return EA_ECUDA;
  if (major != 10) return EA_EUNSUPPORTED;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return EA_ECUDA;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return EA_ECUDA;
  // The array's last 256 bytes hold the timeout record of calls without a
  // status word; start it at zero.
  if (cudaMemset(static_cast<uint8_t*>(ptr) + EA_NOALLOC_SCRATCH_BYTES - 256, 0, 256) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess)
    return EA_ECUDA;
  g_noalloc_sms[dev] = sms;
  g_noalloc_ptr[dev] = static_cast<uint8_t*>(ptr);
  *base = g_noalloc_ptr[dev];
  *num_sms = sms;
  return EA_OK;
}

}  // namespace

extern "C" int attn_fwd_fp32_noalloc(const float* q, const float* k, const float* v, float* o, float* lse, int B,
                                     int Hq, int Hkv, int N, int d, int causal, int window, float scale,
                                     int* status, void* stream_ptr) {
  if (!q || !k || !v || !o || !lse) return EA_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d < 1) return EA_EINVAL;
  if (Hq % Hkv != 0) return EA_EINVAL;
  if (causal != 0 && causal != 1) return EA_EINVAL;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return EA_EINVAL;
  if (d != 64) return EA_EUNSUPPORTED;
  if (static_cast<long long>(Hq) * N >= (1LL << 31) || static_cast<long long>(Hkv) * N >= (1LL << 31))
    return EA_EINVAL;
  const long long num_qblk = (N + 255) / 256;
  if (static_cast<long long>(B) * Hq * num_qblk > INT_MAX) return EA_EINVAL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(status, 4))
    return EA_EALIGN;
  const long long q_rows = static_cast<long long>(B) * N * Hq;
  const long long kv_rows = static_cast<long long>(B) * N * Hkv;
  const size_t sq = round256(static_cast<size_t>(q_rows) * 192 * 2);
  const size_t sk = round256(static_cast<size_t>(kv_rows) * 192 * 2);
  const size_t sv = round256(static_cast<size_t>(kv_rows) * 128 * 2);
  if (sq + sk + sv + 256 > EA_NOALLOC_SCRATCH_BYTES) return EA_EINVAL;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EA_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return EA_EUNSUPPORTED;
  uint8_t* base = nullptr;
  int num_sms = 0;
  int rc = noalloc_setup(dev, &base, &num_sms);
  if (rc != EA_OK) return rc;
  const size_t q_bytes = static_cast<size_t>(q_rows) * 64 * 4;
  const size_t kv_bytes = static_cast<size_t>(kv_rows) * 64 * 4;
  const size_t lse_bytes = static_cast<size_t>(B) * Hq * N * 4;
  if (check_range(q, q_bytes) || check_range(k, kv_bytes) || check_range(v, kv_bytes) || check_range(o, q_bytes) ||
      check_range(lse, lse_bytes) || (status && check_range(status, sizeof(int))))
    return EA_EINVAL;

  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_ptr);
  uint16_t* qs = reinterpret_cast<uint16_t*>(base);
  uint16_t* ks = reinterpret_cast<uint16_t*>(base + sq);
  uint16_t* vs = reinterpret_cast<uint16_t*>(base + sq + sk);
  // Timeout record when the caller passes no status word (never read back).
  int* err_slot = reinterpret_cast<int*>(base + EA_NOALLOC_SCRATCH_BYTES - 256);
  if (status && cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return EA_ECUDA;

  ea::FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.err = status ? status : err_slot;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.causal = causal;
  p.window = window > 0 ? window : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_qblk = static_cast<int>(num_qblk);
  p.num_work = static_cast<int>(B * Hq * num_qblk);
  p.order = g_order == 1 ? 1 : 0;
  p.skip_first_kv = 0;
  p.timeout_ns = g_timeout_ns;

  DeviceState ds;
  ds.num_sms = num_sms;
  rc = launch_split({q, qs, q_rows}, {k, ks, kv_rows}, {v, vs, kv_rows}, ds.num_sms, stream);
  if (rc != EA_OK) return rc;
  CUtensorMap tq, tk, tv;
  if (make_map(&tq, qs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 192, Hq, N, B) ||
      make_map(&tk, ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 192, Hkv, N, B) ||
      make_map(&tv, vs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, Hkv, N, B))
    return EA_EINVAL;
  return launch_attention<ea::KernelCfg<2, 192, 128, ea::kOutF32Split>>(tq, tk, tv, p, ds, stream);
}

#include "backward_api.cuh"  // attn_bwd
