// Dense W4A16 GEMM entry point that allocates nothing (INT4, INT3, INT2,
// INT8, MXFP4_A16 or MXINT4 weights, as hq_gemm_w4a16).
//
// Some callers cannot allocate device memory at the point where they run a
// layer: an inference engine that plans every buffer up front and then
// forbids allocation on its serving path, a host that is executing inside
// someone else's memory pool, or code that must not grow its footprint
// after start-up.  For them, hq_gemm_w4a16_static keeps the scratch the
// stream-K split of K needs (per-tile counters and per-CTA fp32 partial
// sums) in one file-scope device array instead of a caller workspace.
//
// Properties of the array (kHqStaticScratchBytes, 16 MiB):
//   * it exists once per device that loads this library and is held until
//     the process exits;
//   * a call whose launch plan needs more scratch than that is refused with
//     HQ_ERR_WORKSPACE_TOO_SMALL before anything is launched (a smaller
//     token tile through `hq_tuning` needs less);
//   * every call uses the same array, so calls that overlap on the GPU
//     (different streams, no ordering) race on it; calls ordered on one
//     stream do not;
//   * it is laid out as a workspace (error word, the fixed tile-counter
//     region, then partial sums); the tile counters start at zero, as the
//     array does, and every call that completes leaves them at zero again;
//   * its first word records the first device-side error of any call
//     (a bounded wait that ran out) until hq_static_check_device_status
//     reads it; that call then zeroes the error word and the counters,
//     which a call that gave up may have left behind.
// Host code cannot use the array's name as a device address: the first call
// in each CUDA context looks the address up with cudaGetSymbolAddress (with
// that context current) and caches it per context, so the first call in a
// context should come before any stream capture.
#include <cuda_runtime.h>

#include <mutex>

#include "hq_internal.h"

namespace hq {

namespace {

constexpr size_t kHqStaticScratchBytes = 16u << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kHqStaticScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current context (0 when none is current or the driver
// cannot say).  A context destroyed and created again (cudaDeviceReset)
// gets a new id, and its module, with this array, may load elsewhere.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  static CtxGetIdFn get_id = []() -> CtxGetIdFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetIdFn>(p);
  }();
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_static_scratch in the current context, looked up once
// per context (keyed by its unique id), or nullptr when the lookup fails.
void* static_scratch_address() {
  static std::mutex mu;
  constexpr int kSlots = 64;
  static unsigned long long ids[kSlots] = {};
  static void* addrs[kSlots] = {};
  static int next = 0;
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long id = current_context_id();
  if (id != 0) {
    for (int i = 0; i < kSlots; ++i)
      if (ids[i] == id) return addrs[i];
  }
  void* ptr = nullptr;
  // makes the device's primary context current if no context was
  if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
  if (id == 0) id = current_context_id();
  if (id != 0) {
    ids[next] = id;
    addrs[next] = ptr;
    next = (next + 1) % kSlots;
  }
  return ptr;
}

}  // namespace

}  // namespace hq

using namespace hq;

extern "C" hq_status hq_gemm_w4a16_static(const hq_quant_desc* d, const void* packed_w_dev, const void* a_dev,
                                          int32_t m, void* c_dev, const hq_tuning* t, hq_stream_t stream) {
  if (!d) return HQ_ERR_INVALID_ARG;
  if (d->layout_version != HQ_LAYOUT_VERSION) return HQ_ERR_LAYOUT_VERSION;
  if (m < 0) return HQ_ERR_INVALID_ARG;
  hq_status st = check_w4_call(d, t, false);
  if (st != HQ_OK) return st;
  if (m == 0) return HQ_OK;
  if (!packed_w_dev || !a_dev || !c_dev) return HQ_ERR_INVALID_ARG;
  auto aligned16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!aligned16(packed_w_dev) || !aligned16(a_dev) || !aligned16(c_dev)) return HQ_ERR_ALIGNMENT;
  DeviceInfo dev{};
  st = device_info(&dev);
  if (st != HQ_OK) return st;
  W4Config cfg = w4_plan(dev, *d, m, false, t);
  // a whole-tile plan with a stream-K tail falls back to whole tiles when
  // its partial sums would not fit the scratch array
  if (cfg.splits != 0 && cfg.dp_tiles > 0 && w4_workspace_bytes(*d, m, cfg, false) > kHqStaticScratchBytes)
    cfg = w4_whole_tiles(dev, *d, m, cfg);
  const size_t need = w4_workspace_bytes(*d, m, cfg, false);
  if (need > kHqStaticScratchBytes) return HQ_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = static_scratch_address();
  if (!scratch) return HQ_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The tile counters are zero here, as in a workspace: the array starts
  // zero-filled, every call that completes leaves them at zero, and
  // hq_static_check_device_status clears them after a call that did not
  // (nothing runs between the previous kernel on the stream and this one,
  // so the launch overlap of consecutive calls holds)
  return w4_launch(*d, cfg, packed_w_dev, a_dev, m, c_dev, nullptr, scratch, s);
}

extern "C" hq_status hq_static_check_device_status(hq_stream_t stream) {
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  void* scratch = static_scratch_address();
  if (!scratch) return HQ_ERR_CUDA;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return HQ_ERR_CUDA;
  uint32_t err = 0;
  if (cudaMemcpy(&err, scratch, sizeof(err), cudaMemcpyDeviceToHost) != cudaSuccess) return HQ_ERR_CUDA;
  if (err != 0) {
    // a call that ran out of a bounded wait may have left tile counters
    // behind: zero them and the error word for the next call
    if (cudaMemset(scratch, 0, kWsScratchOff) != cudaSuccess) return HQ_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return HQ_ERR_CUDA;
  }
  return static_cast<hq_status>(err);
}
