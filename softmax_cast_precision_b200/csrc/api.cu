// api.cu -- the C ABI of libfp8attn (declared in include/fp8attn.h): argument
// validation, TMA tensor-map construction and kernel launch (forward,
// quantisation, decode and backward).  Every tensor
// (the decode workspace included) is caller-owned device memory; the only
// device memory the library touches besides it is a per-call 256-byte
// scheduler block from the stream-ordered allocator (the persistent kernel's
// calls at d = 128), the module-static scratch array of fp8attn_fwd_noalloc
// and a module-static error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/fp8attn.h"
#include "fwd_v1.cuh"
#include "fwd_v2.cuh"
#include "quantize.cuh"
#include "decode.cuh"
#include "bwd.cuh"

namespace fp8attn {

// Device error word set by bounded waits that run out (one per process and
// device image; read and cleared by fp8attn_check_error).
__device__ uint32_t g_error_word;

// Scratch of fp8attn_fwd_noalloc: word 0 is the persistent kernel's work-unit
// counter.  One array per device image, shared by every such call.
static __device__ __align__(256) unsigned int g_noalloc_scratch[FP8ATTN_NOALLOC_SCRATCH_BYTES / sizeof(unsigned int)];

namespace {

// How long a device-side wait of the persistent kernel may last before it
// gives up and reports FP8ATTN_ERR_TIMEOUT.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Test switch (fp8attn_test_withhold_load): when non-zero, the next launch
// of the persistent kernel skips its first K tile load and waits at most
// this many nanoseconds.
std::atomic<unsigned long long> g_test_withhold_ns{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A [Z, rows, D] byte tensor (D contiguous) read in boxes of box_rows x D,
// swizzled so that the tile lands in the layout the tcgen05 descriptors
// describe (128-byte swizzle for 128-byte rows, 64-byte for 64-byte rows).
bool make_map(CUtensorMap* map, const void* ptr, int D, int rows, int Z, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(Z)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(D) * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMapSwizzle swz = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A [Z, rows, 128] bfloat16 tensor read in boxes of 128 rows x 64 columns
// (one 128-byte swizzle panel per box; a 128 x 128 tile takes two boxes).
bool make_map_bf16(CUtensorMap* map, const void* ptr, int rows, int Z) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(Z)};
  cuuint64_t strides[2] = {256, 256ull * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Packs host signs (d values of +-1) into bit words: bit i set for -1.
// Returns false if a value is not +-1.
bool pack_signs(const float* signs, int d, uint32_t (&bits)[4]) {
  bits[0] = bits[1] = bits[2] = bits[3] = 0u;
  for (int i = 0; i < d; ++i) {
    if (signs[i] == -1.0f) {
      bits[i >> 5] |= 1u << (i & 31);
    } else if (signs[i] != 1.0f) {
      return false;
    }
  }
  return true;
}


int validate(const void* q, const void* k, const void* v, int B, int H, int Hkv, int N, int d, float p_scale,
             int kv_order) {
  if (B < 0 || N < 0 || H < 1 || Hkv < 1 || H % Hkv != 0) return FP8ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FP8ATTN_ERR_UNSUPPORTED;
  // S in [2^-64, 2^64]: the kernels carry S * l and 2^(x + log2 S) in float32.
  if (!(p_scale >= 0x1p-64f) || !(p_scale <= 0x1p64f)) return FP8ATTN_ERR_INVALID_ARG;
  if (kv_order != 0 && kv_order != 1) return FP8ATTN_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535) return FP8ATTN_ERR_UNSUPPORTED;  // grid y/z limits
  const int64_t zq = static_cast<int64_t>(B) * H;
  if (zq * N > (int64_t(1) << 40)) return FP8ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * N * H == 0) return FP8ATTN_OK;
  if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v)) return FP8ATTN_ERR_INVALID_ARG;
  return FP8ATTN_OK;
}

// Per-device stream-ordered pool for the per-call scheduler counter.  Its
// release threshold is unbounded, so blocks freed back to it stay mapped and
// later allocations cost no device-side work (the device's default pool
// unmaps freed memory at every synchronisation, which made calls slow and
// erratic).
cudaMemPool_t sched_pool() {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    uint64_t threshold = ~0ull;
    if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &threshold) != cudaSuccess) return nullptr;
    pools[dev] = pool;
  }
  return pools[dev];
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Persistent warp-specialised kernel (d = 128): one CTA per SM.  `sched`
// is the work-unit counter, already zero on `stream`; p.stream_flags (if
// set) and p.heads_per_piece describe a streamed call.
template <bool COUNT, bool SCALED = false, bool QK16 = false>
int launch_v2_on(const void* q, const void* k, const void* v, FwdParams p, cudaStream_t stream, unsigned int* sched) {
  using C = V2Config;
  constexpr int kSmem = V2Layout<QK16>::SMEM_BYTES;
  CUtensorMap tq, tk, tv;
  const bool maps_ok = QK16 ? (make_map_bf16(&tq, q, p.N, p.B * p.H) && make_map_bf16(&tk, k, p.N, p.B * p.Hkv))
                            : (make_map(&tq, q, 128, p.N, p.B * p.H, 128) &&
                               make_map(&tk, k, 128, p.N, p.B * p.Hkv, 128));
  if (!maps_ok || !make_map(&tv, v, 128, p.N, p.B * p.Hkv, 128)) return FP8ATTN_ERR_CUDA;
  // Streamed calls take their own instance (plain forward pass only).
  if (p.stream_flags != nullptr && (COUNT || SCALED || QK16)) return FP8ATTN_ERR_UNSUPPORTED;
  auto kern = p.stream_flags != nullptr ? fwd_v2_kernel<false, false, false, true> : fwd_v2_kernel<COUNT, SCALED, QK16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  // The warpgroups re-split the block's registers with setmaxnreg; that split
  // is only valid for the launch register count it was computed for.
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return FP8ATTN_ERR_CUDA;
  if (attr.numRegs != C::LAUNCH_REGS) return FP8ATTN_ERR_UNSUPPORTED;
  uint32_t* err_word = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err_word), g_error_word) != cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  const int sms = num_sms();
  if (sms <= 0) return FP8ATTN_ERR_CUDA;
  p.num_q_tiles = (p.N + 127) / 128;
  p.num_kv_tiles = (p.N + 127) / 128;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  const unsigned long long withhold = g_test_withhold_ns.exchange(0ull);
  if (withhold != 0ull) {
    p.wait_limit_ns = withhold;
    p.test_withhold_k = 1;
  }
  const int num_pairs = (p.N + 255) / 256;
  const int64_t units = static_cast<int64_t>(p.B) * p.H * num_pairs;
  const int grid = static_cast<int>(units < sms ? units : sms);
  // Scheduling groups: about two waves of units per group, capped so that the
  // K and V of the heads a group touches (and of the next group, which
  // overlaps it) stay well inside L2 (126 MB on B200).
  const int64_t kv_head_bytes = (QK16 ? 3ll : 2ll) * p.N * 128;
  int gh = (2 * grid + num_pairs - 1) / num_pairs;
  while (gh > 1 && ((gh + p.h_per_kv - 1) / p.h_per_kv + 1) * kv_head_bytes > (48ll << 20)) --gh;
  p.group_heads = gh < 1 ? 1 : (gh > p.B * p.H ? p.B * p.H : gh);
  // A streamed call needs the units in piece order: whole groups per piece.
  if (p.stream_flags != nullptr)
    while (p.heads_per_piece % p.group_heads != 0) --p.group_heads;
  p.sched = sched;
  kern<<<grid, C::THREADS, kSmem, stream>>>(tq, tk, tv, p, err_word);
  return cudaGetLastError() == cudaSuccess ? FP8ATTN_OK : FP8ATTN_ERR_CUDA;
}

// The same with its work-unit counter in a 256-byte block from the library's
// stream-ordered pool for the duration of the call, so that concurrent calls
// on other streams never share it.
template <bool COUNT, bool SCALED = false, bool QK16 = false>
int launch_v2(const void* q, const void* k, const void* v, FwdParams p, cudaStream_t stream) {
  void* sched = nullptr;
  cudaMemPool_t pool = sched_pool();
  if (!pool || cudaMallocFromPoolAsync(&sched, 256, pool, stream) != cudaSuccess) return FP8ATTN_ERR_CUDA;
  int status = FP8ATTN_OK;
  if (cudaMemsetAsync(sched, 0, sizeof(unsigned int), stream) != cudaSuccess)
    status = FP8ATTN_ERR_CUDA;
  else
    status = launch_v2_on<COUNT, SCALED, QK16>(q, k, v, p, stream, static_cast<unsigned int*>(sched));
  if (cudaFreeAsync(sched, stream) != cudaSuccess) status = FP8ATTN_ERR_CUDA;
  return status;
}

template <int D, bool COUNT>
int launch(const void* q, const void* k, const void* v, FwdParams p, cudaStream_t stream) {
  using C = V1Config<D>;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, D, p.N, p.B * p.H, C::BM) || !make_map(&tk, k, D, p.N, p.B * p.Hkv, C::BN) ||
      !make_map(&tv, v, D, p.N, p.B * p.Hkv, C::BN))
    return FP8ATTN_ERR_CUDA;
  auto kern = fwd_v1_kernel<D, COUNT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  uint32_t* err_word = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err_word), g_error_word) != cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  p.num_q_tiles = (p.N + C::BM - 1) / C::BM;
  p.num_kv_tiles = (p.N + C::BN - 1) / C::BN;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  dim3 grid(p.num_q_tiles, p.H, p.B);
  kern<<<grid, 128, C::SMEM_BYTES, stream>>>(tq, tk, tv, p, err_word);
  return cudaGetLastError() == cudaSuccess ? FP8ATTN_OK : FP8ATTN_ERR_CUDA;
}

FwdParams base_params(int B, int H, int Hkv, int N, int causal, float p_scale, int kv_order) {
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.h_per_kv = H / Hkv;
  p.causal = causal ? 1 : 0;
  p.reverse = kv_order;
  p.p_scale = p_scale;
  p.log2_p_scale = static_cast<float>(std::log2(static_cast<double>(p_scale)));
  p.wait_limit_ns = kWaitLimitNs;
  return p;
}

// ---- allocation-free entry point (fp8attn_fwd_noalloc) ----

// Per-device state of the allocation-free entry point, filled once by its
// first call on that device.
struct NoallocDevice {
  bool ready;
  unsigned int* scratch;  // device address of g_noalloc_scratch
  uint32_t* err_word;     // device address of g_error_word
  int sms;
};

int noalloc_setup(NoallocDevice** out) {
  static std::mutex mu;
  static NoallocDevice devs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  NoallocDevice& s = devs[dev];
  if (!s.ready) {
    if (!get_encode_fn()) return FP8ATTN_ERR_CUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&s.scratch), g_noalloc_scratch) != cudaSuccess)
      return FP8ATTN_ERR_CUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&s.err_word), g_error_word) != cudaSuccess)
      return FP8ATTN_ERR_CUDA;
    // Load both forward kernels and set their shared-memory limits now, so
    // that later calls do no module loading.
    auto k2 = fwd_v2_kernel<false>;
    auto k1 = fwd_v1_kernel<64, false>;
    cudaFuncAttributes attr;
    if (cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, V2Layout<false>::SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncGetAttributes(&attr, k2) != cudaSuccess)
      return FP8ATTN_ERR_CUDA;
    if (attr.numRegs != V2Config::LAUNCH_REGS) return FP8ATTN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, V1Config<64>::SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncGetAttributes(&attr, k1) != cudaSuccess)
      return FP8ATTN_ERR_CUDA;
    s.sms = num_sms();
    if (s.sms <= 0) return FP8ATTN_ERR_CUDA;
    s.ready = true;
  }
  *out = &s;
  return FP8ATTN_OK;
}

// The persistent kernel with its work-unit counter in g_noalloc_scratch
// (zeroed on the stream before the launch) instead of a pool block.
int launch_v2_noalloc(const void* q, const void* k, const void* v, FwdParams p, cudaStream_t stream,
                      const NoallocDevice& dev) {
  using C = V2Config;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, 128, p.N, p.B * p.H, 128) || !make_map(&tk, k, 128, p.N, p.B * p.Hkv, 128) ||
      !make_map(&tv, v, 128, p.N, p.B * p.Hkv, 128))
    return FP8ATTN_ERR_CUDA;
  p.num_q_tiles = (p.N + 127) / 128;
  p.num_kv_tiles = (p.N + 127) / 128;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  const int num_pairs = (p.N + 255) / 256;
  const int64_t units = static_cast<int64_t>(p.B) * p.H * num_pairs;
  const int grid = static_cast<int>(units < dev.sms ? units : dev.sms);
  const int64_t kv_head_bytes = 2ll * p.N * 128;
  int gh = (2 * grid + num_pairs - 1) / num_pairs;
  while (gh > 1 && ((gh + p.h_per_kv - 1) / p.h_per_kv + 1) * kv_head_bytes > (48ll << 20)) --gh;
  p.group_heads = gh < 1 ? 1 : (gh > p.B * p.H ? p.B * p.H : gh);
  if (cudaMemsetAsync(dev.scratch, 0, sizeof(unsigned int), stream) != cudaSuccess) return FP8ATTN_ERR_CUDA;
  p.sched = dev.scratch;
  fwd_v2_kernel<false><<<grid, C::THREADS, V2Layout<false>::SMEM_BYTES, stream>>>(tq, tk, tv, p, dev.err_word);
  return cudaGetLastError() == cudaSuccess ? FP8ATTN_OK : FP8ATTN_ERR_CUDA;
}


// ---- streamed host entry point (fp8attn_fwd_host) ----

using StreamValueFn = CUresult (*)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);

StreamValueFn get_stream_value_fn(const char* name) {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &fn, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<StreamValueFn>(fn);
}

// Per-device copy streams, fork/join events and flag blocks of
// fp8attn_fwd_host, made once.  The streams are non-blocking, so that they
// never wait for the legacy default stream on which the kernel may be
// running.  Stream memory operations reject stream-ordered (pool)
// allocations, so the 512-byte blocks holding a call's work-unit counter,
// ready words and flags come from one cudaMalloc: a ring of kHostBlocks, each
// handed to a new call only after the stream of its previous call has passed
// the event recorded at that call's end.
constexpr int kHostBlocks = 8;
struct HostStreams {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t fork = nullptr, in_done = nullptr, out_done = nullptr;
  cudaEvent_t block_free[kHostBlocks] = {};
  unsigned int* blocks = nullptr;  // kHostBlocks x kPieceBlockBytes
  int next = 0;
  StreamValueFn write32 = nullptr, wait32 = nullptr;
  bool ready = false;
};

int host_streams(HostStreams** out) {
  static HostStreams devs[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  HostStreams& h = devs[dev];
  if (!h.ready) {
    h.write32 = get_stream_value_fn("cuStreamWriteValue32");
    h.wait32 = get_stream_value_fn("cuStreamWaitValue32");
    if (!h.write32 || !h.wait32) return FP8ATTN_ERR_UNSUPPORTED;
    if (cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&h.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h.in_done, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h.out_done, cudaEventDisableTiming) != cudaSuccess ||
        cudaMalloc(reinterpret_cast<void**>(&h.blocks), kHostBlocks * kPieceBlockBytes) != cudaSuccess)
      return FP8ATTN_ERR_CUDA;
    for (int i = 0; i < kHostBlocks; ++i)
      if (cudaEventCreateWithFlags(&h.block_free[i], cudaEventDisableTiming) != cudaSuccess) return FP8ATTN_ERR_CUDA;
    h.ready = true;
  }
  *out = &h;
  return FP8ATTN_OK;
}

// Takes the next flag block of the ring (its previous call's end is passed
// on `s` before the block is touched); returns its index.
int take_host_block(HostStreams* h, cudaStream_t s) {
  static std::mutex mu;
  int slot;
  {
    std::lock_guard<std::mutex> lock(mu);
    slot = h->next;
    h->next = (h->next + 1) % kHostBlocks;
  }
  return cudaStreamWaitEvent(s, h->block_free[slot], 0) == cudaSuccess ? slot : -1;
}

}  // namespace
}  // namespace fp8attn

extern "C" int fp8attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                                float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_dev,
                                int B, int H, int Hkv, int N, int d, int causal, float p_scale, int kv_order,
                                int pieces, void* stream) {
  using namespace fp8attn;
  int st = validate(q_dev, k_dev, v_dev, B, H, Hkv, N, d, p_scale, kv_order);
  if (st != FP8ATTN_OK) return st;
  if (pieces < 0 || pieces > kMaxPieces) return FP8ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * H * N == 0) return FP8ATTN_OK;
  if (!q_host || !k_host || !v_host || !o_host || !o_dev || !aligned16(o_dev) || (lse_host == nullptr) != (lse_dev == nullptr) ||
      (lse_dev && (reinterpret_cast<uintptr_t>(lse_dev) & 3u)))
    return FP8ATTN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t row = static_cast<size_t>(N) * d;  // elements of one (b, h) slab
  const size_t zq = static_cast<size_t>(B) * H, zkv = static_cast<size_t>(B) * Hkv;
  auto h2d = [&](void* dst, const void* src, size_t bytes, cudaStream_t cs) {
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, cs) == cudaSuccess;
  };
  auto d2h = [&](void* dst, const void* src, size_t bytes, cudaStream_t cs) {
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, cs) == cudaSuccess;
  };
  FwdParams p = base_params(B, H, Hkv, N, causal, p_scale, kv_order);
  p.o = o_dev;
  p.lse = lse_dev;
  if (d != 128 || pieces == 1) {
    // One piece: copies in, the pass, copies out, in order on the stream.
    if (!h2d(q_dev, q_host, zq * row, s) || !h2d(k_dev, k_host, zkv * row, s) || !h2d(v_dev, v_host, zkv * row, s))
      return FP8ATTN_ERR_CUDA;
    st = d == 128 ? launch_v2<false>(q_dev, k_dev, v_dev, p, s) : launch<64, false>(q_dev, k_dev, v_dev, p, s);
    if (st != FP8ATTN_OK) return st;
    if (!d2h(o_host, o_dev, zq * row * 2, s) || (lse_dev && !d2h(lse_host, lse_dev, zq * N * sizeof(float), s)))
      return FP8ATTN_ERR_CUDA;
    return FP8ATTN_OK;
  }
  HostStreams* hs = nullptr;
  st = host_streams(&hs);
  if (st != FP8ATTN_OK) return st;
  // Pieces of whole (b, kv head) slabs with their query heads: the units the
  // pass waits for and reports.
  const int want = pieces == 0 ? 24 : pieces;
  const int kv_per_piece = static_cast<int>((zkv + want - 1) / want);
  const int n_pieces = static_cast<int>((zkv + kv_per_piece - 1) / kv_per_piece);
  const int rep = H / Hkv;
  p.heads_per_piece = kv_per_piece * rep;
  // Copies move runs of neighbouring pieces: one piece first (so that the pass
  // starts early), then two, then three at a time, then two and one last (so
  // that little is left to compute and copy out after the last copy in).
  // Fewer, larger copies keep the host link busy; short ones at both ends
  // shorten the time when only one direction of it is in use.
  int group_end[kMaxPieces];
  int n_groups = 0;
  {
    int c = 0;
    auto add = [&](int len) {
      c += len;
      group_end[n_groups++] = c;
    };
    if (n_pieces < 6) {
      for (int i = 0; i < n_pieces; ++i) add(1);
    } else {
      add(1);
      add(2);
      for (int mid = n_pieces - 6; mid > 0; mid -= std::min(3, mid)) add(std::min(3, mid));
      add(2);
      add(1);
    }
  }
  // The block holds the work-unit counter (word 0) and the piece words.
  const int slot = take_host_block(hs, s);
  if (slot < 0) return FP8ATTN_ERR_CUDA;
  unsigned int* flags = hs->blocks + (kPieceBlockBytes / 4) * slot;
  const CUdeviceptr fl = reinterpret_cast<CUdeviceptr>(flags);
  p.stream_flags = flags;
  bool ok = cudaMemsetAsync(flags, 0, kPieceBlockBytes, s) == cudaSuccess && cudaEventRecord(hs->fork, s) == cudaSuccess &&
            cudaStreamWaitEvent(hs->in, hs->fork, 0) == cudaSuccess &&
            cudaStreamWaitEvent(hs->out, hs->fork, 0) == cudaSuccess;
  // Slabs of the pieces [c0, c1): kv slabs [k0, k0 + nk), query slabs [k0, k0 + nk) * rep.
  auto slabs = [&](int c0, int c1, size_t& k0, size_t& nk) {
    k0 = static_cast<size_t>(c0) * kv_per_piece;
    nk = std::min<size_t>(static_cast<size_t>(c1) * kv_per_piece, zkv) - k0;
  };
  // Copies in: each run, then the ready words of its pieces.
  for (int g = 0, c0 = 0; ok && g < n_groups; c0 = group_end[g++]) {
    size_t k0, nk;
    slabs(c0, group_end[g], k0, nk);
    const size_t q0 = k0 * rep, nq = nk * rep;
    ok = h2d(static_cast<uint8_t*>(q_dev) + q0 * row, static_cast<const uint8_t*>(q_host) + q0 * row, nq * row, hs->in) &&
         h2d(static_cast<uint8_t*>(k_dev) + k0 * row, static_cast<const uint8_t*>(k_host) + k0 * row, nk * row, hs->in) &&
         h2d(static_cast<uint8_t*>(v_dev) + k0 * row, static_cast<const uint8_t*>(v_host) + k0 * row, nk * row, hs->in);
    for (int c = c0; ok && c < group_end[g]; ++c)
      ok = hs->write32(reinterpret_cast<CUstream>(hs->in), fl + 4 * (kPieceReady + c), 1u, 0) == CUDA_SUCCESS;
  }
  // (Recorded whatever happened above, so that the join below also covers
  // copies and ready words queued before a failure.)
  const bool in_recorded = cudaEventRecord(hs->in_done, hs->in) == cudaSuccess;
  ok = ok && in_recorded;
  // The pass, before any copy out is queued: a copy out of pageable memory
  // returns only when done, and must not wait for a kernel not yet launched.
  if (ok) st = launch_v2_on<false>(q_dev, k_dev, v_dev, p, s, flags);
  if (!ok && st == FP8ATTN_OK) st = FP8ATTN_ERR_CUDA;
  // Copies out: each run once the flags of all its pieces are up (the kernel
  // raises every flag, also when it gives up, so these waits always end once
  // it has run).
  for (int g = 0, c0 = 0; st == FP8ATTN_OK && g < n_groups; c0 = group_end[g++]) {
    for (int c = c0; st == FP8ATTN_OK && c < group_end[g]; ++c)
      if (hs->wait32(reinterpret_cast<CUstream>(hs->out), fl + 4 * (kPieceFlag + c), 1u, 0 /* GEQ */) != CUDA_SUCCESS)
        st = FP8ATTN_ERR_CUDA;
    size_t k0, nk;
    slabs(c0, group_end[g], k0, nk);
    const size_t q0 = k0 * rep, nq = nk * rep;
    if (st == FP8ATTN_OK &&
        (!d2h(static_cast<uint8_t*>(o_host) + q0 * row * 2, static_cast<const uint8_t*>(o_dev) + q0 * row * 2,
              nq * row * 2, hs->out) ||
         (lse_dev && !d2h(lse_host + q0 * N, lse_dev + q0 * N, nq * N * sizeof(float), hs->out))))
      st = FP8ATTN_ERR_CUDA;
  }
  // Join: the stream continues once the copies out (and in) are done; the
  // block may be handed out again once the stream is past that point.
  if (cudaEventRecord(hs->out_done, hs->out) != cudaSuccess || cudaStreamWaitEvent(s, hs->out_done, 0) != cudaSuccess ||
      cudaStreamWaitEvent(s, hs->in_done, 0) != cudaSuccess || cudaEventRecord(hs->block_free[slot], s) != cudaSuccess)
    st = FP8ATTN_ERR_CUDA;
  return st;
}

using namespace fp8attn;

extern "C" int fp8attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                           int N, int d, int causal, float p_scale, int kv_order, void* stream) {
  int st = validate(q, k, v, B, H, Hkv, N, d, p_scale, kv_order);
  if (st != FP8ATTN_OK) return st;
  if (static_cast<int64_t>(B) * H * N == 0) return FP8ATTN_OK;
  if (!o || !aligned16(o) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))) return FP8ATTN_ERR_INVALID_ARG;
  FwdParams p = base_params(B, H, Hkv, N, causal, p_scale, kv_order);
  p.o = o;
  p.lse = lse;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_v2<false>(q, k, v, p, s) : launch<64, false>(q, k, v, p, s);
}

extern "C" int fp8attn_pzero_count(const void* q, const void* k, const void* v, unsigned long long* counts, int B,
                                   int H, int Hkv, int N, int d, int causal, float p_scale, int kv_order, int n_sink,
                                   void* stream) {
  int st = validate(q, k, v, B, H, Hkv, N, d, p_scale, kv_order);
  if (st != FP8ATTN_OK) return st;
  if (n_sink < 0) return FP8ATTN_ERR_INVALID_ARG;
  const int64_t nheads = static_cast<int64_t>(B) * H;
  if (nheads == 0) return FP8ATTN_OK;
  if (!counts || (reinterpret_cast<uintptr_t>(counts) & 7u)) return FP8ATTN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(counts, 0, sizeof(unsigned long long) * nheads, s) != cudaSuccess) return FP8ATTN_ERR_CUDA;
  if (N == 0) return FP8ATTN_OK;
  FwdParams p = base_params(B, H, Hkv, N, causal, p_scale, kv_order);
  p.counts = counts;
  p.n_sink = n_sink;
  return d == 128 ? launch_v2<true>(q, k, v, p, s) : launch<64, true>(q, k, v, p, s);
}

extern "C" int fp8attn_fwd_scaled(const void* q, const void* k, const void* v, void* o, float* lse,
                                  const float* q_scales, const float* k_scales, const float* v_scales,
                                  const float* signs, int B, int H, int Hkv, int N, int d, int causal, float p_scale,
                                  int kv_order, void* stream) {
  int st = validate(q, k, v, B, H, Hkv, N, d, p_scale, kv_order);
  if (st != FP8ATTN_OK) return st;
  if (d != 128) return FP8ATTN_ERR_UNSUPPORTED;
  FwdParams p = base_params(B, H, Hkv, N, causal, p_scale, kv_order);
  if (signs != nullptr) {
    if (!pack_signs(signs, d, p.sign_bits)) return FP8ATTN_ERR_INVALID_ARG;
    p.unrotate = 1;
  }
  if (static_cast<int64_t>(B) * H * N == 0) return FP8ATTN_OK;
  if (!o || !aligned16(o) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))) return FP8ATTN_ERR_INVALID_ARG;
  auto aligned4 = [](const void* ptr) { return ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; };
  if (!aligned4(q_scales) || !aligned4(k_scales) || !aligned4(v_scales)) return FP8ATTN_ERR_INVALID_ARG;
  p.o = o;
  p.lse = lse;
  p.q_scales = q_scales;
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  return launch_v2<false, true>(q, k, v, p, static_cast<cudaStream_t>(stream));
}

extern "C" int fp8attn_fwd_bf16qk(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                  int Hkv, int N, int d, int causal, float p_scale, int kv_order, void* stream) {
  int st = validate(q, k, v, B, H, Hkv, N, d, p_scale, kv_order);
  if (st != FP8ATTN_OK) return st;
  if (d != 128) return FP8ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * N == 0) return FP8ATTN_OK;
  if (!o || !aligned16(o) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))) return FP8ATTN_ERR_INVALID_ARG;
  FwdParams p = base_params(B, H, Hkv, N, causal, p_scale, kv_order);
  p.o = o;
  p.lse = lse;
  return launch_v2<false, false, true>(q, k, v, p, static_cast<cudaStream_t>(stream));
}

extern "C" int fp8attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                   int Hkv, int N, int d, int causal, float p_scale, int kv_order, void* stream) {
  int st = validate(q, k, v, B, H, Hkv, N, d, p_scale, kv_order);
  if (st != FP8ATTN_OK) return st;
  if (static_cast<int64_t>(B) * H * N == 0) return FP8ATTN_OK;
  if (!o || !aligned16(o) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))) return FP8ATTN_ERR_INVALID_ARG;
  if (d == 128 && static_cast<int64_t>(B) * H * ((N + 255) / 256) > FP8ATTN_NOALLOC_MAX_UNITS)
    return FP8ATTN_ERR_SCRATCH_LIMIT;
  NoallocDevice* dev = nullptr;
  st = noalloc_setup(&dev);
  if (st != FP8ATTN_OK) return st;
  FwdParams p = base_params(B, H, Hkv, N, causal, p_scale, kv_order);
  p.o = o;
  p.lse = lse;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_v2_noalloc(q, k, v, p, s, *dev) : launch<64, false>(q, k, v, p, s);
}

namespace fp8attn {
namespace {

template <int E, int MODE>
int launch_quantize_ring(const QuantParams& p, cudaStream_t s, uint32_t* err_word) {
  const int nunits = p.Z * p.nblocks;
  if (nunits == 0) return FP8ATTN_OK;
  const int smem = quant_stages(p) * quant_stage_bytes(p);
  if (cudaFuncSetAttribute(quantize_kernel<E, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  const int sms = num_sms();
  if (sms <= 0) return FP8ATTN_ERR_CUDA;
  const int grid = std::min(nunits, 2 * sms);
  quantize_kernel<E, MODE><<<grid, kQuantWarps * 32, smem, s>>>(p, err_word);
  return cudaGetLastError() == cudaSuccess ? FP8ATTN_OK : FP8ATTN_ERR_CUDA;
}

template <int E>
int launch_quantize(QuantParams p, cudaStream_t s) {
  uint32_t* err_word = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err_word), g_error_word) != cudaSuccess) return FP8ATTN_ERR_CUDA;
  if (p.block_rows > 0) return launch_quantize_ring<E, 0>(p, s, err_word);
  if (cudaMemsetAsync(p.scales, 0, sizeof(float) * static_cast<size_t>(p.Z), s) != cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  p.block_rows = 128;
  p.nblocks = (p.N + 127) / 128;
  int st = launch_quantize_ring<E, 1>(p, s, err_word);
  if (st == FP8ATTN_OK) st = launch_quantize_ring<E, 2>(p, s, err_word);
  if (st != FP8ATTN_OK) return st;
  quantize_finish_kernel<<<(p.Z + 255) / 256, 256, 0, s>>>(p.scales, p.Z);
  return cudaGetLastError() == cudaSuccess ? FP8ATTN_OK : FP8ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace fp8attn

extern "C" int fp8attn_quantize(const void* x, int x_dtype, void* xq, float* scales, int Z, int N, int d,
                                int block_rows, const float* signs, void* stream) {
  if (Z < 0 || N < 0 || (d != 64 && d != 128) || (x_dtype != 0 && x_dtype != 1) || block_rows < 0 ||
      block_rows > 128)
    return (d != 64 && d != 128) ? FP8ATTN_ERR_UNSUPPORTED : FP8ATTN_ERR_INVALID_ARG;
  if (Z > 65535) return FP8ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(Z) * N * d > (int64_t(1) << 40)) return FP8ATTN_ERR_UNSUPPORTED;
  QuantParams p;
  std::memset(&p, 0, sizeof(p));
  if (signs != nullptr) {
    if (!pack_signs(signs, d, p.sign_bits)) return FP8ATTN_ERR_INVALID_ARG;
    p.rotate = 1;
  }
  if (Z == 0 || (N == 0 && block_rows > 0)) return FP8ATTN_OK;
  if (!scales || (reinterpret_cast<uintptr_t>(scales) & 3u)) return FP8ATTN_ERR_INVALID_ARG;
  if (N > 0 && (!x || !xq || !aligned16(x) || !aligned16(xq))) return FP8ATTN_ERR_INVALID_ARG;
  p.x = x;
  p.xq = static_cast<uint8_t*>(xq);
  p.scales = scales;
  p.Z = Z;
  p.N = N;
  p.d = d;
  p.block_rows = block_rows;
  p.nblocks = block_rows > 0 ? (N + block_rows - 1) / block_rows : 1;
  // The persistent CTAs number the blocks of all slabs in 32-bit integers.
  if (block_rows > 0 && static_cast<int64_t>(Z) * p.nblocks > (int64_t(1) << 30)) return FP8ATTN_ERR_UNSUPPORTED;
  p.x_f32 = x_dtype;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_quantize<64>(p, s) : launch_quantize<32>(p, s);
}

extern "C" unsigned long long fp8attn_decode_workspace_bytes(int B, int H, int N, int split_tiles) {
  if (B <= 0 || H <= 0 || N <= 0 || split_tiles <= 0) return 0;
  const int64_t ntiles = (static_cast<int64_t>(N) + 127) / 128;
  const int64_t splits = (ntiles + split_tiles - 1) / split_tiles;
  return static_cast<unsigned long long>(B) * H * splits * fp8attn::kDecodePartStride * sizeof(float);
}

extern "C" int fp8attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                              unsigned long long workspace_bytes, int B, int H, int Hkv, int N, int d,
                              float p_scale, int kv_order, int split_tiles, void* stream) {
  using namespace fp8attn;
  if (B < 0 || N < 0 || H < 1 || Hkv < 1 || H % Hkv != 0 || split_tiles < 1) return FP8ATTN_ERR_INVALID_ARG;
  if (d != 128 || H / Hkv > kDecodeMaxG) return FP8ATTN_ERR_UNSUPPORTED;
  if (!(p_scale >= 0x1p-64f) || !(p_scale <= 0x1p64f)) return FP8ATTN_ERR_INVALID_ARG;
  if (kv_order != 0 && kv_order != 1) return FP8ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * Hkv > 65535 || static_cast<int64_t>(B) * H > 0x7fffffff)
    return FP8ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H == 0) return FP8ATTN_OK;
  if (N == 0) return FP8ATTN_ERR_INVALID_ARG;  // a query with no key has no softmax
  if (!q || !k || !v || !o || !workspace || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !aligned16(workspace) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FP8ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < fp8attn_decode_workspace_bytes(B, H, N, split_tiles)) return FP8ATTN_ERR_INVALID_ARG;
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const uint8_t*>(q);
  p.k = static_cast<const uint8_t*>(k);
  p.v = static_cast<const uint8_t*>(v);
  p.part = static_cast<float*>(workspace);
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.G = H / Hkv;
  p.ntiles = (N + 127) / 128;
  p.split_tiles = split_tiles;
  p.splits = (p.ntiles + split_tiles - 1) / split_tiles;
  p.reverse = kv_order;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  p.log2_p_scale = static_cast<float>(std::log2(static_cast<double>(p_scale)));
  CUtensorMap tk, tv;
  if (!make_map(&tk, k, 128, N, B * Hkv, 128) || !make_map(&tv, v, 128, N, B * Hkv, 128)) return FP8ATTN_ERR_CUDA;
  uint32_t* err_word = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err_word), g_error_word) != cudaSuccess) return FP8ATTN_ERR_CUDA;
  if (cudaFuncSetAttribute(decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeLayout::SMEM_BYTES) !=
      cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  decode_split_kernel<<<dim3(p.splits, B * Hkv), 128, DecodeLayout::SMEM_BYTES, s>>>(tk, tv, p, err_word);
  decode_combine_kernel<<<B * H, 128, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? FP8ATTN_OK : FP8ATTN_ERR_CUDA;
}

extern "C" int fp8attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dout, float* dq, float* dk, float* dv, float* delta, int B, int H, int Hkv,
                           int N, int d, int causal, float p_scale, void* stream) {
  using namespace fp8attn;
  if (B < 0 || N < 0 || H < 1 || Hkv < 1 || H % Hkv != 0) return FP8ATTN_ERR_INVALID_ARG;
  if (d != 128) return FP8ATTN_ERR_UNSUPPORTED;
  if (!(p_scale >= 0x1p-64f) || !(p_scale <= 0x1p64f)) return FP8ATTN_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535) return FP8ATTN_ERR_UNSUPPORTED;  // grid y/z limits
  const int64_t rows = static_cast<int64_t>(B) * H * N;
  if (rows > (int64_t(1) << 34)) return FP8ATTN_ERR_UNSUPPORTED;  // row-dot grid: rows / 8 blocks
  if (rows == 0) return FP8ATTN_OK;
  auto a16 = [](const void* ptr) { return ptr != nullptr && aligned16(ptr); };
  auto a4 = [](const void* ptr) { return ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; };
  if (!a16(q) || !a16(k) || !a16(v) || !a16(o) || !a16(dout) || !a16(dq) || !a16(dk) || !a16(dv) || !a4(lse) ||
      !a4(delta))
    return FP8ATTN_ERR_INVALID_ARG;
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.delta = delta;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.h_per_kv = H / Hkv;
  p.causal = causal ? 1 : 0;
  p.num_tiles = (N + 127) / 128;
  p.p_scale = p_scale;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  p.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(128.0));
  // The dQ kernel reads bfloat16 copies of K and V, made into the dK and dV
  // buffers (4 bytes per element; the copies take the first half) before the
  // dK/dV kernel, which runs last, writes its results there.
  CUtensorMap tq, tq64, tk, tv, tdo, tkb, tvb;
  if (!make_map(&tq, q, 128, N, B * H, 128) || !make_map(&tq64, q, 128, N, B * H, 64) ||
      !make_map(&tk, k, 128, N, B * Hkv, 128) || !make_map(&tv, v, 128, N, B * Hkv, 128) ||
      !make_map_bf16(&tdo, dout, N, B * H) || !make_map_bf16(&tkb, dk, N, B * Hkv) ||
      !make_map_bf16(&tvb, dv, N, B * Hkv))
    return FP8ATTN_ERR_CUDA;
  uint32_t* err_word = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err_word), g_error_word) != cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  if (cudaFuncSetAttribute(bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DkdvLayout::SMEM_BYTES) !=
          cudaSuccess ||
      cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DqLayout::SMEM_BYTES) !=
          cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = num_sms();
  if (sms <= 0) return FP8ATTN_ERR_CUDA;
  bwd_delta_kernel<<<static_cast<unsigned int>((rows + 7) / 8), 256, 0, s>>>(p);
  const int64_t kv16 = static_cast<int64_t>(B) * Hkv * N * 8;  // 16-code groups of K (and of V)
  const unsigned int widen_grid = static_cast<unsigned int>(std::min<int64_t>((kv16 + 255) / 256, 8LL * sms));
  bwd_widen_kernel<<<widen_grid, 256, 0, s>>>(static_cast<const uint8_t*>(k), reinterpret_cast<uint16_t*>(dk), kv16);
  bwd_widen_kernel<<<widen_grid, 256, 0, s>>>(static_cast<const uint8_t*>(v), reinterpret_cast<uint16_t*>(dv), kv16);
  bwd_dq_kernel<<<dim3(p.num_tiles, H, B), 128 * kBwdGroups, DqLayout::SMEM_BYTES, s>>>(tq, tk, tkb, tvb, tdo, p,
                                                                                     err_word);
  bwd_dkdv_kernel<<<dim3(p.num_tiles, Hkv, B), kDkdvThreads, DkdvLayout::SMEM_BYTES, s>>>(tq64, tk, tv, tdo, p,
                                                                                        err_word);
  return cudaGetLastError() == cudaSuccess ? FP8ATTN_OK : FP8ATTN_ERR_CUDA;
}

extern "C" int fp8attn_kv_tile(int d) {
  if (d == 128) return V1Config<128>::BN;
  if (d == 64) return V1Config<64>::BN;
  return 0;
}

extern "C" const char* fp8attn_status_str(int status) {
  switch (status) {
    case FP8ATTN_OK:
      return "ok";
    case FP8ATTN_ERR_INVALID_ARG:
      return "invalid argument";
    case FP8ATTN_ERR_UNSUPPORTED:
      return "unsupported configuration";
    case FP8ATTN_ERR_CUDA:
      return "CUDA error";
    case FP8ATTN_ERR_TIMEOUT:
      return "device wait timed out";
    case FP8ATTN_ERR_SCRATCH_LIMIT:
      return "problem too large for the allocation-free entry point's fixed scratch";
    default:
      return "unknown status";
  }
}

extern "C" int fp8attn_check_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP8ATTN_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return FP8ATTN_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return FP8ATTN_ERR_CUDA;
    return FP8ATTN_ERR_TIMEOUT;
  }
  return FP8ATTN_OK;
}

extern "C" int fp8attn_test_withhold_load(unsigned long long wait_limit_ns) {
  if (wait_limit_ns == 0ull || wait_limit_ns > kWaitLimitNs) return FP8ATTN_ERR_INVALID_ARG;
  g_test_withhold_ns.store(wait_limit_ns);
  return FP8ATTN_OK;
}

extern "C" int fp8attn_version(void) { return 100; }
