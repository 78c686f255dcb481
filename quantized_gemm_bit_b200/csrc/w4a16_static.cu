// Dense W4A16 GEMM entry point that allocates nothing (INT4 or MXFP4_A16
// weights, as hq_gemm_w4a16).
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
//   * each call clears the part that must start at zero (error word and
//     tile counters) on its stream before the kernel.
// Host code cannot use the array's name as a device address: the first call
// on each device looks the address up with cudaGetSymbolAddress (with that
// device current) and caches it, so the first call on a device should come
// before any stream capture.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "hq_internal.h"

namespace hq {

namespace {

constexpr size_t kHqStaticScratchBytes = 16u << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kHqStaticScratchBytes];

// Device address of g_static_scratch on the current device (looked up once
// per device), or nullptr when the lookup fails.
void* static_scratch_address(int device) {
  static std::mutex mu;
  static void* addr[64] = {};
  if (device < 0 || device >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[device] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
    addr[device] = ptr;
  }
  return addr[device];
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
  void* scratch = static_scratch_address(dev.device);
  if (!scratch) return HQ_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // error word and tile counters start at zero (the partial sums need not)
  const size_t tiles = (size_t)((d->n + kTileN - 1) / kTileN) * (size_t)((m + cfg.ntok - 1) / cfg.ntok);
  const size_t zero_bytes = std::min(need, sizeof(WsHeader) + ((4 * tiles * sizeof(int32_t) + 255) / 256) * 256);
  if (cudaMemsetAsync(scratch, 0, zero_bytes, s) != cudaSuccess) return HQ_ERR_CUDA;
  return w4_launch(*d, cfg, packed_w_dev, a_dev, m, c_dev, nullptr, scratch, s);
}
