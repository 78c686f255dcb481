// C-ABI entry points: argument validation, planning and dispatch.
// Every check happens on the host before any launch; a failing call returns
// a status and leaves all memory untouched.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "hq_internal.h"

namespace hq {

hq_status device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HQ_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    DeviceInfo di{};
    di.device = dev;
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return HQ_ERR_NO_DEVICE;
    di.num_sms = v;
    cudaDeviceGetAttribute(&di.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&di.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    di.max_smem_optin = (size_t)v;
    cache[dev] = di;
    have[dev] = true;
  }
  *out = cache[dev];
  // The kernels are built for sm_100a only.
  if (out->cc_major != 10 || out->cc_minor != 0) return HQ_ERR_NO_DEVICE;
  return HQ_OK;
}

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

hq_status check_desc(const hq_quant_desc* d) {
  if (!d) return HQ_ERR_INVALID_ARG;
  if (d->layout_version != HQ_LAYOUT_VERSION) return HQ_ERR_LAYOUT_VERSION;
  if (d->n < 1 || d->k < 1 || d->num_experts < 1) return HQ_ERR_INVALID_ARG;
  switch (d->fmt) {
    case HQ_FMT_INT4:
      if (d->group_size != 128 || d->k % 128 != 0) return HQ_ERR_UNSUPPORTED;
      if (d->has_zero_point != 0 && d->has_zero_point != 1) return HQ_ERR_INVALID_ARG;
      if (d->num_experts > 1024) return HQ_ERR_UNSUPPORTED;
      return HQ_OK;
    case HQ_FMT_MXFP4:
      if (d->group_size != 32 || d->k % 128 != 0 || d->has_zero_point || d->num_experts != 1)
        return HQ_ERR_UNSUPPORTED;
      return HQ_OK;
    case HQ_FMT_NVFP4:
      if (d->group_size != 16 || d->k % 256 != 0 || d->has_zero_point || d->num_experts != 1)
        return HQ_ERR_UNSUPPORTED;
      return HQ_OK;
    case HQ_FMT_MXFP4_A16:
      if (d->group_size != 32 || d->k % 128 != 0 || d->has_zero_point || d->num_experts > 1024)
        return HQ_ERR_UNSUPPORTED;
      return HQ_OK;
    case HQ_FMT_MXINT4:
      if (d->group_size != 32 || d->k % 128 != 0 || d->has_zero_point || d->num_experts > 1024)
        return HQ_ERR_UNSUPPORTED;
      return HQ_OK;
    case HQ_FMT_INT3:
    case HQ_FMT_INT2:
    case HQ_FMT_INT8:
      if (d->group_size != 128 || d->k % 128 != 0) return HQ_ERR_UNSUPPORTED;
      if (d->has_zero_point != 0 && d->has_zero_point != 1) return HQ_ERR_INVALID_ARG;
      if (d->num_experts > 1024) return HQ_ERR_UNSUPPORTED;
      return HQ_OK;
    default:
      return HQ_ERR_INVALID_ARG;
  }
}

// Formats the W4A16 kernels read (dequantized in registers, bf16 MMA).
bool w4_format(const hq_quant_desc* d) {
  return d->fmt == HQ_FMT_INT4 || d->fmt == HQ_FMT_INT3 || d->fmt == HQ_FMT_INT2 || d->fmt == HQ_FMT_INT8 ||
         d->fmt == HQ_FMT_MXFP4_A16 || d->fmt == HQ_FMT_MXINT4;
}

// Tuning checks shared by the W4A16 entry points (dense: split_k free;
// grouped: at most one CTA per tile).
hq_status check_w4_tuning(const hq_quant_desc* d, const hq_tuning* t, bool grouped) {
  if (!t) return HQ_OK;
  if (t->tile_m && t->tile_m != 16 && t->tile_m != 32 && t->tile_m != 64 && t->tile_m != 128 && t->tile_m != 256)
    return HQ_ERR_UNSUPPORTED;
  if ((t->tile_n && t->tile_n != 128) || (t->tile_k && t->tile_k != 128) || t->split_k < 0 || t->stages < 0 ||
      t->cta_group < 0 || t->cta_group > 2 || t->variant < 0 || t->variant > 3 ||
      (t->flags & ~HQ_TUNE_NO_EARLY_WEIGHTS) != 0)
    return HQ_ERR_UNSUPPORTED;
  if (grouped && t->split_k > 1) return HQ_ERR_UNSUPPORTED;
  // CTA pairs: dense 256-token whole tiles of 256-row weight tiles
  if (t->cta_group == 2 && (grouped || d->n % 256 != 0 || (t->tile_m && t->tile_m != 256) || t->split_k != 0))
    return HQ_ERR_UNSUPPORTED;
  // the exact-weight kernel factors a 128-K group scale out of the sum:
  // the MX formats' scale per 32 K leaves none
  if ((d->fmt == HQ_FMT_MXFP4_A16 || d->fmt == HQ_FMT_MXINT4) && t->variant == 2) return HQ_ERR_UNSUPPORTED;
  return HQ_OK;
}

}  // namespace

// ---- the caller's per-shape tuning table
namespace {
std::mutex g_table_mu;
std::vector<hq_tuning_entry> g_table;
}  // namespace

const hq_tuning* tuning_from_table(const hq_quant_desc& d, int m, hq_tuning* tmp) {
  std::lock_guard<std::mutex> lock(g_table_mu);
  for (const hq_tuning_entry& e : g_table) {
    if (e.fmt == d.fmt && e.n == d.n && e.k == d.k && e.num_experts == d.num_experts && m >= e.m_min &&
        m <= e.m_max) {
      *tmp = e.tuning;
      return tmp;
    }
  }
  return nullptr;
}

hq_status check_w4_call(const hq_quant_desc* d, const hq_tuning* t, bool grouped) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (!w4_format(d) || (grouped ? d->num_experts < 2 : d->num_experts != 1)) return HQ_ERR_INVALID_ARG;
  return check_w4_tuning(d, t, grouped);
}

// Packed size per format (the layouts are written out in hq_pack.cpp).
size_t packed_size_impl(const hq_quant_desc& d);
hq_status pack_impl(const hq_quant_desc& d, const void* codes, const void* scales, const void* zeros, float g,
                    void* out);
hq_status pack_gated_impl(const hq_quant_desc& d, const void* codes, const void* scales, const void* zeros,
                          void* out);

}  // namespace hq

using namespace hq;

extern "C" {

int hq_layout_version(void) { return HQ_LAYOUT_VERSION; }

const char* hq_status_string(hq_status s) {
  switch (s) {
    case HQ_OK: return "ok";
    case HQ_ERR_INVALID_ARG: return "invalid argument";
    case HQ_ERR_UNSUPPORTED: return "unsupported shape, format or tuning";
    case HQ_ERR_ALIGNMENT: return "pointer not aligned (16 B for data, 256 B for workspaces)";
    case HQ_ERR_WORKSPACE_TOO_SMALL: return "buffer or workspace too small";
    case HQ_ERR_LAYOUT_VERSION: return "descriptor from another packed-layout version";
    case HQ_ERR_CUDA: return "CUDA runtime or launch error";
    case HQ_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case HQ_ERR_DEVICE_BAD_OFFSETS: return "expert ids or offsets out of range on the device";
    case HQ_ERR_NO_DEVICE: return "no sm_100 device is current";
  }
  return "unknown status";
}

hq_status hq_quant_desc_init(hq_quant_desc* d, int32_t fmt, int32_t n, int32_t k, int32_t group_size,
                             int32_t has_zero_point, int32_t num_experts) {
  if (!d) return HQ_ERR_INVALID_ARG;
  hq_quant_desc t{};
  t.layout_version = HQ_LAYOUT_VERSION;
  t.fmt = fmt;
  t.n = n;
  t.k = k;
  t.group_size = group_size;
  t.has_zero_point = has_zero_point;
  t.num_experts = num_experts;
  hq_status st = check_desc(&t);
  if (st != HQ_OK) return st;
  *d = t;
  return HQ_OK;
}

size_t hq_packed_size(const hq_quant_desc* d) {
  if (check_desc(d) != HQ_OK) return 0;
  return packed_size_impl(*d);
}

hq_status hq_pack_weights(const hq_quant_desc* d, const void* codes_host, const void* scales_host,
                          const void* zeros_host, float global_scale, void* out_host, size_t out_bytes) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (!codes_host || !scales_host || !out_host) return HQ_ERR_INVALID_ARG;
  if (d->fmt == HQ_FMT_INT4 || d->fmt == HQ_FMT_INT3 || d->fmt == HQ_FMT_INT2 || d->fmt == HQ_FMT_INT8) {
    if ((d->has_zero_point != 0) != (zeros_host != nullptr)) return HQ_ERR_INVALID_ARG;
  } else if (zeros_host) {
    return HQ_ERR_INVALID_ARG;
  }
  if (out_bytes < packed_size_impl(*d)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  return pack_impl(*d, codes_host, scales_host, zeros_host, global_scale, out_host);
}

hq_status hq_pack_weights_gated(const hq_quant_desc* d, const void* codes_host, const void* scales_host,
                                const void* zeros_host, void* out_host, size_t out_bytes) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (!w4_format(d) || d->n % 128 != 0) return HQ_ERR_UNSUPPORTED;
  if (!codes_host || !scales_host || !out_host) return HQ_ERR_INVALID_ARG;
  if ((d->fmt == HQ_FMT_MXFP4_A16 || d->fmt == HQ_FMT_MXINT4) ? zeros_host != nullptr
                                                               : (d->has_zero_point != 0) != (zeros_host != nullptr))
    return HQ_ERR_INVALID_ARG;
  if (out_bytes < packed_size_impl(*d)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  return pack_gated_impl(*d, codes_host, scales_host, zeros_host, out_host);
}

size_t hq_workspace_size(const hq_quant_desc* d, int32_t m, const hq_tuning* t) {
  if (check_desc(d) != HQ_OK || m < 0) return 0;
  DeviceInfo dev{};
  if (device_info(&dev) != HQ_OK) {
    // no sm_100 device current: size for a 148-SM part so the answer is
    // still an upper bound the caller can allocate
    dev.num_sms = 148;
  }
  if (!w4_format(d)) {
    BsConfig cfg = bs_plan(dev, *d, m < 1 ? 1 : m, t);
    return bs_workspace_bytes(*d, m < 1 ? 1 : m, cfg);
  }
  const bool grouped = d->num_experts > 1;
  W4Config cfg = w4_plan(dev, *d, m < 1 ? 1 : m, grouped, t);
  return w4_workspace_bytes(*d, m < 1 ? 1 : m, cfg, grouped);
}

hq_status hq_gemm_w4a16(const hq_quant_desc* d, const void* packed_w_dev, const void* a_dev, int32_t m,
                        void* c_dev, const hq_tuning* t, void* ws_dev, size_t ws_bytes, hq_stream_t stream) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (!w4_format(d) || d->num_experts != 1) return HQ_ERR_INVALID_ARG;
  if (m < 0) return HQ_ERR_INVALID_ARG;
  if (m == 0) return HQ_OK;
  if (!packed_w_dev || !a_dev || !c_dev || !ws_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(packed_w_dev, 16) || !aligned(a_dev, 16) || !aligned(c_dev, 16) || !aligned(ws_dev, 256))
    return HQ_ERR_ALIGNMENT;
  st = check_w4_tuning(d, t, false);
  if (st != HQ_OK) return st;
  DeviceInfo dev{};
  st = device_info(&dev);
  if (st != HQ_OK) return st;
  W4Config cfg = w4_plan(dev, *d, m, false, t);
  if (ws_bytes < w4_workspace_bytes(*d, m, cfg, false)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  return w4_launch(*d, cfg, packed_w_dev, a_dev, m, c_dev, nullptr, ws_dev, reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_grouped_gemm_moe(const hq_quant_desc* d, const void* packed_w_dev, const void* a_sorted_dev,
                              const int32_t* expert_offsets_dev, int32_t total_rows, void* c_sorted_dev,
                              const hq_tuning* t, void* ws_dev, size_t ws_bytes, hq_stream_t stream) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (!w4_format(d) || d->num_experts < 2) return HQ_ERR_INVALID_ARG;
  if (total_rows < 0) return HQ_ERR_INVALID_ARG;
  if (total_rows == 0) return HQ_OK;
  if (!packed_w_dev || !a_sorted_dev || !expert_offsets_dev || !c_sorted_dev || !ws_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(packed_w_dev, 16) || !aligned(a_sorted_dev, 16) || !aligned(c_sorted_dev, 16) ||
      !aligned(expert_offsets_dev, 4) || !aligned(ws_dev, 256))
    return HQ_ERR_ALIGNMENT;
  st = check_w4_tuning(d, t, true);
  if (st != HQ_OK) return st;
  DeviceInfo dev{};
  st = device_info(&dev);
  if (st != HQ_OK) return st;
  W4Config cfg = w4_plan(dev, *d, total_rows, true, t);
  if (ws_bytes < w4_workspace_bytes(*d, total_rows, cfg, true)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  return w4_launch(*d, cfg, packed_w_dev, a_sorted_dev, total_rows, c_sorted_dev, expert_offsets_dev, ws_dev,
                   reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_grouped_gemm_moe_swiglu(const hq_quant_desc* d, const void* packed_w_dev, const void* a_sorted_dev,
                                     const int32_t* expert_offsets_dev, int32_t total_rows, void* h_sorted_dev,
                                     const hq_tuning* t, void* ws_dev, size_t ws_bytes, hq_stream_t stream) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (!w4_format(d) || d->num_experts < 2) return HQ_ERR_INVALID_ARG;
  if (d->n % 128 != 0) return HQ_ERR_UNSUPPORTED;
  if (total_rows < 0) return HQ_ERR_INVALID_ARG;
  if (total_rows == 0) return HQ_OK;
  if (!packed_w_dev || !a_sorted_dev || !expert_offsets_dev || !h_sorted_dev || !ws_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(packed_w_dev, 16) || !aligned(a_sorted_dev, 16) || !aligned(h_sorted_dev, 16) ||
      !aligned(expert_offsets_dev, 4) || !aligned(ws_dev, 256))
    return HQ_ERR_ALIGNMENT;
  st = check_w4_tuning(d, t, true);
  if (st != HQ_OK) return st;
  DeviceInfo dev{};
  st = device_info(&dev);
  if (st != HQ_OK) return st;
  W4Config cfg = w4_plan(dev, *d, total_rows, true, t);
  if (ws_bytes < w4_workspace_bytes(*d, total_rows, cfg, true)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  return w4_launch(*d, cfg, packed_w_dev, a_sorted_dev, total_rows, h_sorted_dev, expert_offsets_dev, ws_dev,
                   reinterpret_cast<cudaStream_t>(stream), 1);
}

namespace {
hq_status check_bs_tuning(const hq_quant_desc* d, const hq_tuning* t) {
  if (!t) return HQ_OK;
  if (t->tile_m && t->tile_m != 16 && t->tile_m != 32 && t->tile_m != 64 && t->tile_m != 128 && t->tile_m != 256)
    return HQ_ERR_UNSUPPORTED;
  if ((t->tile_n && t->tile_n != 128) || t->tile_k || t->split_k < 0 || t->stages < 0 || t->cta_group < 0 ||
      t->cta_group > 2 || t->variant != 0 || (t->flags & ~HQ_TUNE_NO_EARLY_WEIGHTS) != 0)
    return HQ_ERR_UNSUPPORTED;
  // CTA pairs: 256-row weight tiles, 128- or 256-token tiles, whole tiles
  if (t->cta_group == 2 && (d->n % 256 != 0 || (t->tile_m && t->tile_m < 128) || t->split_k != 0))
    return HQ_ERR_UNSUPPORTED;
  return HQ_OK;
}
}  // namespace

hq_status hq_gemm_mxfp4_a8(const hq_quant_desc* d, const void* packed_w_dev, const void* a_e4m3_dev,
                           const float* a_scale_dev, int32_t m, void* c_dev, const hq_tuning* t, void* ws_dev,
                           size_t ws_bytes, hq_stream_t stream) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (d->fmt != HQ_FMT_MXFP4 || m < 0) return HQ_ERR_INVALID_ARG;
  if (m == 0) return HQ_OK;
  if (!packed_w_dev || !a_e4m3_dev || !a_scale_dev || !c_dev || !ws_dev) return HQ_ERR_INVALID_ARG;
  // the unpacking weight copy needs a 32-byte aligned blob
  if (!aligned(packed_w_dev, 256) || !aligned(a_e4m3_dev, 16) || !aligned(a_scale_dev, 4) || !aligned(c_dev, 16) ||
      !aligned(ws_dev, 256))
    return HQ_ERR_ALIGNMENT;
  st = check_bs_tuning(d, t);
  if (st != HQ_OK) return st;
  DeviceInfo dev{};
  st = device_info(&dev);
  if (st != HQ_OK) return st;
  BsConfig cfg = bs_plan(dev, *d, m, t);
  if (ws_bytes < bs_workspace_bytes(*d, m, cfg)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  return bs_launch(*d, cfg, packed_w_dev, a_e4m3_dev, nullptr, a_scale_dev, 1.f, m, c_dev, ws_dev,
                   reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_gemm_nvfp4(const hq_quant_desc* d, const void* packed_w_dev, const void* a_fp4_dev,
                        const void* a_sf_dev, float a_global, int32_t m, void* c_dev, const hq_tuning* t,
                        void* ws_dev, size_t ws_bytes, hq_stream_t stream) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (d->fmt != HQ_FMT_NVFP4 || m < 0) return HQ_ERR_INVALID_ARG;
  if (m == 0) return HQ_OK;
  if (!packed_w_dev || !a_fp4_dev || !a_sf_dev || !c_dev || !ws_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(packed_w_dev, 256) || !aligned(a_fp4_dev, 16) || !aligned(a_sf_dev, 16) || !aligned(c_dev, 16) ||
      !aligned(ws_dev, 256))
    return HQ_ERR_ALIGNMENT;
  st = check_bs_tuning(d, t);
  if (st != HQ_OK) return st;
  DeviceInfo dev{};
  st = device_info(&dev);
  if (st != HQ_OK) return st;
  BsConfig cfg = bs_plan(dev, *d, m, t);
  if (ws_bytes < bs_workspace_bytes(*d, m, cfg)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  return bs_launch(*d, cfg, packed_w_dev, a_fp4_dev, a_sf_dev, nullptr, a_global, m, c_dev, ws_dev,
                   reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_quantize_fp8_rows(const void* x_bf16_dev, int32_t rows, int32_t k, void* q_e4m3_dev,
                               float* scale_dev, hq_stream_t stream) {
  if (rows < 0 || k < 1 || k % 8 != 0) return HQ_ERR_INVALID_ARG;
  if (rows == 0) return HQ_OK;
  if (!x_bf16_dev || !q_e4m3_dev || !scale_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(x_bf16_dev, 16) || !aligned(q_e4m3_dev, 8) || !aligned(scale_dev, 4)) return HQ_ERR_ALIGNMENT;
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  return fp8_rows_launch(x_bf16_dev, rows, k, q_e4m3_dev, scale_dev, reinterpret_cast<cudaStream_t>(stream));
}

size_t hq_quantize_nvfp4_workspace_size(int32_t rows, int32_t k) {
  if (rows < 0 || k < 1) return 0;
  return nvfp4_quant_ws_bytes(rows, k);
}

hq_status hq_quantize_nvfp4(const void* x_bf16_dev, int32_t rows, int32_t k, void* codes_dev, void* sf_dev,
                            float* global_dev, void* ws_dev, size_t ws_bytes, hq_stream_t stream) {
  if (rows < 0 || k < 1 || k % 16 != 0) return HQ_ERR_INVALID_ARG;
  if (rows == 0) return HQ_OK;
  if (!x_bf16_dev || !codes_dev || !sf_dev || !global_dev || !ws_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(x_bf16_dev, 16) || !aligned(codes_dev, 8) || !aligned(global_dev, 4) || !aligned(ws_dev, 256))
    return HQ_ERR_ALIGNMENT;
  if (ws_bytes < nvfp4_quant_ws_bytes(rows, k)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  return nvfp4_quant_launch(x_bf16_dev, rows, k, codes_dev, sf_dev, global_dev, ws_dev,
                            reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_moe_topk(const float* logits_dev, int32_t t, int32_t e, int32_t k, int32_t* topk_ids_dev,
                      hq_stream_t stream) {
  if (t < 0 || k < 1 || k > 16 || e < k || e > 1024) return HQ_ERR_INVALID_ARG;
  if (t == 0) return HQ_OK;
  if (!logits_dev || !topk_ids_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(logits_dev, 4) || !aligned(topk_ids_dev, 4)) return HQ_ERR_ALIGNMENT;
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  return moe_topk_launch(logits_dev, t, e, k, topk_ids_dev, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_moe_topk_softmax(const float* logits_dev, int32_t t, int32_t e, int32_t k, int32_t* topk_ids_dev,
                              float* topk_weights_dev, hq_stream_t stream) {
  if (t < 0 || k < 1 || k > 16 || e < k || e > 1024) return HQ_ERR_INVALID_ARG;
  if (t == 0) return HQ_OK;
  if (!logits_dev || !topk_ids_dev || !topk_weights_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(logits_dev, 4) || !aligned(topk_ids_dev, 4) || !aligned(topk_weights_dev, 4)) return HQ_ERR_ALIGNMENT;
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  return moe_topk_launch(logits_dev, t, e, k, topk_ids_dev, topk_weights_dev, reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_moe_swiglu(const void* gate_up_dev, int32_t rows, int32_t inter, void* h_dev, hq_stream_t stream) {
  if (rows < 0 || inter < 1 || inter % 8 != 0) return HQ_ERR_INVALID_ARG;
  if (rows == 0) return HQ_OK;
  if (!gate_up_dev || !h_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(gate_up_dev, 16) || !aligned(h_dev, 16)) return HQ_ERR_ALIGNMENT;
  return moe_swiglu_launch(gate_up_dev, rows, inter, h_dev, reinterpret_cast<cudaStream_t>(stream));
}

size_t hq_moe_combine_workspace_size(int32_t t, int32_t k) {
  if (t < 0 || k < 1) return 0;
  return moe_combine_ws_bytes(t, k);
}

hq_status hq_moe_combine(const void* y_sorted_dev, const int32_t* sorted_src_dev, const float* topk_weights_dev,
                         int32_t t, int32_t k, int32_t hidden, void* out_dev, void* ws_dev, size_t ws_bytes,
                         hq_stream_t stream) {
  if (t < 0 || k < 1 || k > 16 || hidden < 1 || hidden % 8 != 0) return HQ_ERR_INVALID_ARG;
  if ((long long)t * k > 0x7fffffffLL) return HQ_ERR_INVALID_ARG;
  if (t == 0) return HQ_OK;
  if (!y_sorted_dev || !sorted_src_dev || !topk_weights_dev || !out_dev || !ws_dev) return HQ_ERR_INVALID_ARG;
  if (!aligned(y_sorted_dev, 16) || !aligned(out_dev, 16) || !aligned(sorted_src_dev, 4) ||
      !aligned(topk_weights_dev, 4) || !aligned(ws_dev, 256))
    return HQ_ERR_ALIGNMENT;
  if (ws_bytes < moe_combine_ws_bytes(t, k)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  return moe_combine_launch(y_sorted_dev, sorted_src_dev, topk_weights_dev, t, k, hidden, out_dev, ws_dev,
                            reinterpret_cast<cudaStream_t>(stream));
}

size_t hq_moe_permute_workspace_size(int32_t t, int32_t k, int32_t e) {
  if (t < 0 || k < 1 || e < 1) return 0;
  return moe_permute_ws_bytes(t, k, e);
}

hq_status hq_moe_permute(const int32_t* topk_ids_dev, int32_t t, int32_t k, int32_t e, int32_t* sorted_src_dev,
                         int32_t* expert_offsets_dev, const void* a_dev, int32_t hidden, void* a_sorted_dev,
                         void* ws_dev, size_t ws_bytes, hq_stream_t stream) {
  if (t < 0 || k < 1 || k > 16 || e < 1 || e > 1024) return HQ_ERR_INVALID_ARG;
  if (!expert_offsets_dev || !ws_dev) return HQ_ERR_INVALID_ARG;
  if (t > 0 && (!topk_ids_dev || !sorted_src_dev)) return HQ_ERR_INVALID_ARG;
  if ((a_dev == nullptr) != (a_sorted_dev == nullptr)) return HQ_ERR_INVALID_ARG;
  if (a_dev && (hidden < 1 || hidden % 8 != 0)) return HQ_ERR_INVALID_ARG;
  if (!aligned(ws_dev, 256) || (a_dev && (!aligned(a_dev, 16) || !aligned(a_sorted_dev, 16))))
    return HQ_ERR_ALIGNMENT;
  if (ws_bytes < moe_permute_ws_bytes(t, k, e)) return HQ_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  return moe_permute_launch(topk_ids_dev, t, k, e, sorted_src_dev, expert_offsets_dev, a_dev, hidden, a_sorted_dev,
                            ws_dev, reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_tuning_table_set(const hq_tuning_entry* entries, int32_t count) {
  if (count < 0 || (count > 0 && !entries)) return HQ_ERR_INVALID_ARG;
  std::vector<hq_tuning_entry> next(entries, entries + count);
  // every entry must be a tuning the matching entry point accepts
  for (const hq_tuning_entry& e : next) {
    if (e.m_min < 0 || e.m_max < e.m_min) return HQ_ERR_INVALID_ARG;
    hq_quant_desc d{};
    hq_status st = hq_quant_desc_init(&d, e.fmt, e.n, e.k, e.fmt == HQ_FMT_INT4 || e.fmt == HQ_FMT_INT3 ||
                                                               e.fmt == HQ_FMT_INT2 || e.fmt == HQ_FMT_INT8
                                                           ? 128
                                                           : e.fmt == HQ_FMT_NVFP4 ? 16 : 32,
                                      0, e.num_experts);
    if (st != HQ_OK) return st;
    st = w4_format(&d) ? check_w4_tuning(&d, &e.tuning, d.num_experts > 1) : check_bs_tuning(&d, &e.tuning);
    if (st != HQ_OK) return st;
  }
  std::lock_guard<std::mutex> lock(g_table_mu);
  g_table.swap(next);
  return HQ_OK;
}

hq_status hq_plan_describe(const hq_quant_desc* d, int32_t m, const hq_tuning* t, hq_plan* out) {
  hq_status st = check_desc(d);
  if (st != HQ_OK) return st;
  if (!out || m < 1) return HQ_ERR_INVALID_ARG;
  const bool w16 = w4_format(d);
  st = w16 ? check_w4_tuning(d, t, d->num_experts > 1) : check_bs_tuning(d, t);
  if (st != HQ_OK) return st;
  DeviceInfo dev{};
  if (device_info(&dev) != HQ_OK) dev.num_sms = 148;   // as hq_workspace_size
  hq_tuning tmp;
  hq_plan p{};
  p.from_table = (!t && tuning_from_table(*d, m, &tmp)) ? 1 : 0;
  if (w16) {
    const bool grouped = d->num_experts > 1;
    const W4Config cfg = w4_plan(dev, *d, m, grouped, t);
    const int depth = w4_ring_depth(*d, cfg);
    const bool mx = d->fmt == HQ_FMT_MXFP4_A16 || d->fmt == HQ_FMT_MXINT4;
    p.tile_m = cfg.ntok;
    p.grid = cfg.grid;
    const bool reg = cfg.variant == 3;
    p.split = grouped ? 0 : cfg.splits == 0 || (reg && cfg.splits == 1) ? 0 : cfg.splits;
    p.whole_tiles = grouped ? 0 : cfg.dp_tiles;
    p.kernel = reg ? 4 : (!mx && cfg.ntok <= 64 && cfg.variant != 1) ? 2 : 1;
    p.cta_group = cfg.cta_group;
    p.ring_stages = depth;
    p.stages = (cfg.stages > 0 && cfg.stages < depth) ? cfg.stages : depth;
    p.workspace_bytes = w4_workspace_bytes(*d, m, cfg, grouped);
  } else {
    const BsConfig cfg = bs_plan(dev, *d, m, t);
    const int depth = bs_ring_depth(*d, cfg);
    p.tile_m = cfg.ntok;
    p.grid = cfg.grid;
    p.split = cfg.splits;
    p.kernel = 3;
    p.cta_group = cfg.cta_group;
    p.ring_stages = depth;
    p.stages = (cfg.stages > 0 && cfg.stages < depth) ? cfg.stages : depth;
    p.workspace_bytes = bs_workspace_bytes(*d, m, cfg);
  }
  *out = p;
  return HQ_OK;
}

hq_status hq_check_device_status(void* ws_dev, hq_stream_t stream) {
  if (!ws_dev) return HQ_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return HQ_ERR_CUDA;
  uint32_t err = 0;
  if (cudaMemcpy(&err, ws_dev, sizeof(err), cudaMemcpyDeviceToHost) != cudaSuccess) return HQ_ERR_CUDA;
  if (err != 0) {
    uint32_t zero = 0;
    if (cudaMemcpy(ws_dev, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return HQ_ERR_CUDA;
  }
  return static_cast<hq_status>(err);
}

hq_status hq_debug_timeout_probe(void* ws_dev, uint64_t limit_ns, hq_stream_t stream) {
  if (!ws_dev || limit_ns > 100000000ull) return HQ_ERR_INVALID_ARG;
  if (!aligned(ws_dev, 256)) return HQ_ERR_ALIGNMENT;
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  return debug_timeout_launch(ws_dev, limit_ns, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
