// Internal declarations shared by the C-ABI layer and the kernel launchers.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/hq.h"

namespace hq {

// Workspace header: the first 256 bytes of every workspace.
struct WsHeader {
  uint32_t err;        // first device-side error (hq_status), 0 = none
  uint32_t reserved[63];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");
// Workspace layout of every entry point: the header, a fixed region of
// stream-K tile counters (used by GEMM plans that split K), then scratch
// (fp32 partial sums, re-laid activation scales, histograms, block maxima,
// inverse permutations).  The counters sit at the same offsets whatever the
// call, and each call that completes sets the ones it used back to zero,
// while no call keeps data below kWsScratchOff: one workspace serves any
// sequence of calls in turn, and the scratch needs no initial value.  A
// split plan whose counters would not fit runs as whole tiles.
constexpr size_t kWsCounterBytes = 256u << 10;
constexpr size_t kWsScratchOff = sizeof(WsHeader) + kWsCounterBytes;

constexpr int kTileN = 128;      // weight rows per tile (MMA M)
constexpr int kBlockK = 128;     // K per packed record / pipeline stage
constexpr int kW4RecCodes = 8192;
inline int w4_record_bytes(bool has_zero) { return kW4RecCodes + 256 + (has_zero ? 128 : 0); }
// MXFP4 weights for the W4A16 kernels: 8192 code bytes, then one E8M0 byte
// per (row, 32-K block) of the record
constexpr int kMxA16RecBytes = kW4RecCodes + 512;
// INT3 weights: 6144 code bytes, then fp16 scales (256) and zero points
// (128, with zero points) as in the INT4 record
constexpr int kW3RecCodes = 6144;
inline int w3_record_bytes(bool has_zero) { return kW3RecCodes + 256 + (has_zero ? 128 : 0); }
// INT2 weights: 4096 code bytes, then scales and zero points as for INT4
constexpr int kW2RecCodes = 4096;
inline int w2_record_bytes(bool has_zero) { return kW2RecCodes + 256 + (has_zero ? 128 : 0); }
// INT8 weights: 16384 code bytes, then scales and zero points as for INT4
constexpr int kW8RecCodes = 16384;
inline int w8_record_bytes(bool has_zero) { return kW8RecCodes + 256 + (has_zero ? 128 : 0); }
// MXINT4 weights: 8192 code bytes (the INT4 nibble layout), then one E8M0
// byte per (row, 32-K block) as for MXFP4_A16
constexpr int kMxi4RecBytes = kW4RecCodes + 512;

constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s per wait

// Resolved launch configuration of the W4A16 kernel family.
struct W4Config {
  int ntok;     // token tile (MMA N)
  int stages;   // pipeline stages the producer keeps in flight, 0 = the kernel's ring depth
  int splits;   // 0: data parallel (whole tiles); else stream-K / split K
  int dp_tiles; // stream-K plans: tiles run whole before the shared K range
  int grid;     // CTAs
  int early_weights;  // fetch packed weights before the previous kernel completes
  int cta_group;      // 2: dense 256-token whole tiles on CTA pairs (cta_group::2 MMAs)
  int variant;  // 0: library's choice (exact weights for tiles of <= 64
                // tokens, bf16-rescaled above); 1: bf16-rescaled weights for
                // every tile; 2: exact (q - z) weights + per-group fp32
                // scaling for tiles of <= 64 tokens (bf16-rescaled above);
                // 3: dense INT4 at 1..16 tokens on the register-path kernel
                // (exact (q - z) weights in mma.sync fragments, splits = K
                // slices per weight tile, grid = tiles * splits)
  int reg_tw;   // register path: 16-row MMA tiles per warp (1: grids of fewer CTAs than SMs, else 2)
};

struct DeviceInfo {
  int device;
  int num_sms;
  int cc_major, cc_minor;
  size_t max_smem_optin;
};
hq_status device_info(DeviceInfo* out);

// The caller's tuning table (hq_tuning_table_set): the tuning of the first
// entry matching (fmt, n, k, num_experts) with m in [m_min, m_max], copied
// into *tmp, or nullptr.
const hq_tuning* tuning_from_table(const hq_quant_desc& d, int m, hq_tuning* tmp);

// Descriptor, format and tuning checks of a W4A16-family call (INT4, INT3,
// INT2, INT8, MXFP4_A16 or MXINT4 weights; grouped: num_experts >= 2, else
// exactly 1).
hq_status check_w4_call(const hq_quant_desc* d, const hq_tuning* t, bool grouped);

// W4A16 (dense or grouped) planning and launch.
W4Config w4_plan(const DeviceInfo& dev, const hq_quant_desc& d, int m, bool grouped, const hq_tuning* t);
// The same token tile with whole tiles only (no partial sums, no workspace
// beyond the header).
W4Config w4_whole_tiles(const DeviceInfo& dev, const hq_quant_desc& d, int m, W4Config cfg);
size_t w4_workspace_bytes(const hq_quant_desc& d, int m, const W4Config& cfg, bool grouped);
// swiglu: grouped only, weights packed in the gated gate+up row order; c
// receives h = silu(gate) * up, [m][d.n / 2].
hq_status w4_launch(const hq_quant_desc& d, const W4Config& cfg, const void* packed, const void* a, int m,
                    void* c, const int32_t* expert_offsets, void* ws, cudaStream_t stream, int swiglu = 0);

// Block-scaled 4-bit GEMMs (MXFP4 weights x E4M3 activations; NVFP4 x NVFP4).
struct BsConfig {
  int ntok;
  int splits;   // 0: whole tiles per CTA (no partial sums)
  int grid;
  int stages;   // pipeline stages the producer keeps in flight, 0 = the kernel's ring depth
  int early_weights;  // fetch packed weights before the previous kernel completes
  int cta_group;      // 2: CTA pairs (cta_group::2 MMAs on 256-row weight tiles)
};
BsConfig bs_plan(const DeviceInfo& dev, const hq_quant_desc& d, int m, const hq_tuning* t);
size_t bs_workspace_bytes(const hq_quant_desc& d, int m, const BsConfig& cfg);
hq_status bs_launch(const hq_quant_desc& d, const BsConfig& cfg, const void* packed, const void* a, const void* a_sf,
                    const float* a_scale, float a_global, int m, void* c, void* ws, cudaStream_t stream);

// Register-path W4A16 kernel (INT4 weights, dense, 1..16 tokens; tuning
// variant 3): CTAs per SM a plan fills (slots) for 8- or 16-token tiles, the
// K slices per weight tile, its workspace and its launch.
constexpr int reg_slots_per_sm(int nt8) { return nt8 == 1 ? 3 : 4; }
constexpr int kRegRing8 = 3, kRegRing16 = 4;   // stages of the 8- and 16-token kernels' rings
constexpr bool kRegGroupedDefault = true;       // grouped MoE: the library's choice at <= 8 tokens per expert
int reg_splits(int num_sms, const hq_quant_desc& d, int m);
size_t reg_workspace_bytes(const W4Config& cfg);
hq_status reg_launch(const hq_quant_desc& d, const W4Config& cfg, const void* packed, const void* a, int m, void* c,
                     void* ws, cudaStream_t stream);
// Grouped MoE on the register path: persistent CTAs (reg_grouped_ctas_per_sm
// per SM) over 8- or 16-token units (cfg.ntok); swiglu: gated gate+up
// weights, h written.
constexpr int reg_grouped_ctas_per_sm(int nt8) { return nt8 == 1 ? 3 : 2; }
hq_status reg_launch_grouped(const hq_quant_desc& d, const W4Config& cfg, const void* packed, const void* a,
                             int total_rows, void* c, const int32_t* expert_offsets, void* ws, cudaStream_t stream,
                             int swiglu);

// Ring depth (SMEM pipeline stages) of the kernel a plan launches.
int w4_ring_depth(const hq_quant_desc& d, const W4Config& cfg);
int bs_ring_depth(const hq_quant_desc& d, const BsConfig& cfg);

// Activation quantizers.
size_t nvfp4_quant_ws_bytes(int rows, int k);
hq_status fp8_rows_launch(const void* x, int rows, int k, void* q, float* scale, cudaStream_t s);
hq_status nvfp4_quant_launch(const void* x, int rows, int k, void* codes, void* sf, float* g, void* ws,
                             cudaStream_t s);

// MoE helpers.
size_t moe_permute_ws_bytes(int t, int k, int e);
hq_status moe_topk_launch(const float* logits, int t, int e, int k, int32_t* ids, float* weights, cudaStream_t s);
hq_status moe_swiglu_launch(const void* x, long long rows, int inter, void* h, cudaStream_t s);
size_t moe_combine_ws_bytes(int t, int k);
hq_status moe_combine_launch(const void* y_sorted, const int32_t* sorted_src, const float* weights, int t, int k,
                             int hidden, void* out, void* ws, cudaStream_t s);
hq_status moe_permute_launch(const int32_t* ids, int t, int k, int e, int32_t* sorted_src, int32_t* offsets,
                             const void* a, int hidden, void* a_sorted, void* ws, cudaStream_t s);

hq_status debug_timeout_launch(void* ws, uint64_t limit_ns, cudaStream_t s);

// Launch with programmatic stream serialization: the kernel's CTAs may start
// while the previous kernel on the stream is finishing; the kernel itself
// waits (griddepcontrol.wait) before touching anything that kernel may write.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// As launch_pdl, in clusters of two CTAs along x (grid.x even).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_pairs(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Driver entry point for tensor-map encoding (resolved once).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

}  // namespace hq
