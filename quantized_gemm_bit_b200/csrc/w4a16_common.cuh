// Device code shared by the two W4A16 kernels (w4a16.cu: dequantized and
// rescaled bf16 weights, fp32 accumulation across K in TMEM; w4a16_small.cu:
// exact (q - z) weights, per-group fp32 rescaling): the kernel parameters,
// the unit scheduler (data parallel, stream-K, grouped MoE), the grouped
// tile table built on the device, the output stores and the stream-K fixup.
//
// Method: weights are 4-bit codes with a per-group fp16 scale and an optional
// uint4 zero point, described separately from the execution choices
// ("Humming: open-source kernel library for quantized inference", summary
// paragraph 2); w = (q - z) * s.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "epilogue.cuh"
#include "hq_internal.h"
#include "ptx.cuh"

namespace hq {
namespace w4 {

constexpr int kThreads = 512;
constexpr int kRecMax = 8576;        // packed record with zero points
constexpr int kMaxExperts = 1024;

// Weight formats of the W4A16 kernels: INT4 records, MXFP4 records (8704
// bytes), INT3 records (at most 6528 bytes), INT2 records (at most 4480),
// INT8 records (at most 16768) and MXINT4 records (8704).
constexpr int kFmtInt4 = 0, kFmtMx = 1, kFmtInt3 = 2, kFmtInt2 = 3, kFmtInt8 = 4, kFmtMxi4 = 5;

// INT8 codes to exact fp32: __byte_perm places code byte j of `w` under the
// exponent of 2^23 (0x4B000000), giving 2^23 + q exactly; subtracting
// zf = 2^23 + z leaves q - z exactly.
__device__ __forceinline__ float u8_minus_zero(uint32_t w, int j, float zf) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u + (uint32_t)j)) - zf;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct W4Params {
  const uint8_t* packed;             // expert 0, record (0, 0)
  __nv_bfloat16* c;
  const int32_t* expert_offsets;     // grouped mode only
  float* partials;                   // dense: [grid][2][NTOK*128] fp32
  int32_t* counters;                 // dense: [tiles][4]
  uint32_t* err;
  uint64_t expert_bytes;
  uint64_t wait_ns;
  long long total_iters;             // dense stream-K: k-block iterations after the whole tiles
  int dp_tiles;                      // dense stream-K: tiles run whole first (a multiple of the grid)
  int m;                             // dense: rows of A; grouped: total sorted rows
  int n;                             // output columns
  int n_tiles, k_blocks, m_tiles;
  int num_experts;
  int has_zero;
  int rec_bytes;
  int grouped;
  int weights_once;                  // each weight tile is read by one CTA
  int data_parallel;                 // dense: whole tiles per unit, no partials
  int early_weights;                 // dense: fetch the first stages' weights before griddepcontrol.wait
  int cta_pairs;                     // dense, whole tiles on CTA pairs (clusters of two, 256-row weight tiles)
  int n_pairs;                       // CTA pairs: n_tiles / 2
  int stage_limit;                   // pipeline stages in flight (0 or >= the ring depth: the whole ring)
};



// One unit of work: a K range of one (expert, token tile, weight tile).
struct Unit {
  int expert;
  int nt;        // weight tile
  int row0;      // first row of A / C
  int rows;      // valid rows in this tile (<= NTOK)
  int kb0, kb1;  // k-block range
  int tile;      // dense tile index
  int partial;   // 1: other CTAs own the rest of this tile's K range
  int slot;      // partial slot of this CTA (0: its first unit, 1: its last)
};

// Unit `idx` of this CTA, or false when it has no more.  Every role walks
// the same sequence, so no role needs to hear about units from another.
template <int NTOK>
__device__ __forceinline__ bool get_unit(const W4Params& p, const int* s_prefix, const int* s_off, int total_grouped,
                                         int idx, Unit& x) {
  auto whole = [&](long long tile) {
    const int mt = (int)(tile / p.n_tiles);
    x.tile = (int)tile;
    x.nt = (int)(tile - (long long)mt * p.n_tiles);
    x.expert = 0;
    x.row0 = mt * NTOK;
    x.rows = min(NTOK, p.m - x.row0);
    x.kb0 = 0;
    x.kb1 = p.k_blocks;
    x.partial = 0;
    x.slot = 0;
  };
  if (p.cta_pairs) {
    // whole (token tile, 256-row weight tile) units over the clusters; CTA
    // rank r of the pair owns 128-row weight tile 2 * pair + r
    const long long ncl = gridDim.x / 2, cl = blockIdx.x / 2;
    const long long t = cl + (long long)idx * ncl;
    if (t >= (long long)p.m_tiles * p.n_pairs) return false;
    const int mt = (int)(t / p.n_pairs);
    x.tile = (int)t;
    x.nt = 2 * (int)(t - (long long)mt * p.n_pairs) + (int)(blockIdx.x & 1);
    x.expert = 0;
    x.row0 = mt * NTOK;
    x.rows = min(NTOK, p.m - x.row0);
    x.kb0 = 0;
    x.kb1 = p.k_blocks;
    x.partial = 0;
    x.slot = 0;
    return true;
  }
  if (!p.grouped && p.data_parallel) {
    // whole tiles, strided over the persistent CTAs
    const long long tile = (long long)blockIdx.x + (long long)idx * gridDim.x;
    if (tile >= (long long)p.m_tiles * p.n_tiles) return false;
    whole(tile);
    return true;
  }
  if (!p.grouped) {
    const long long G = gridDim.x, i = blockIdx.x;
    // first the whole tiles of the leading waves (none for plain stream-K)
    const int dp_per = p.dp_tiles / (int)G;
    if (idx < dp_per) {
      whole(i + (long long)idx * G);
      return true;
    }
    // then this CTA's share of the k-block iterations of the remaining tiles
    const int sidx = idx - dp_per;
    const long long T = p.total_iters;
    const long long beg = sk_start(i, T, G), end = sk_start(i + 1, T, G);
    const long long kb = p.k_blocks;
    const long long rel = beg / kb + sidx;
    const long long x0 = sidx == 0 ? beg : rel * kb;
    if (x0 >= end) return false;
    const long long x1 = min(end, (rel + 1) * kb);
    const long long tile = p.dp_tiles + rel;
    const int mt = (int)(tile / p.n_tiles);
    x.tile = (int)tile;
    x.nt = (int)(tile - (long long)mt * p.n_tiles);
    x.expert = 0;
    x.row0 = mt * NTOK;
    x.rows = min(NTOK, p.m - x.row0);
    x.kb0 = (int)(x0 - rel * kb);
    x.kb1 = (int)(x1 - rel * kb);
    x.partial = (x.kb0 != 0 || x.kb1 != p.k_blocks) ? 1 : 0;
    x.slot = sidx == 0 ? 0 : 1;
    return true;
  }
  const int u = blockIdx.x + idx * gridDim.x;
  if (u >= total_grouped) return false;
  // find the expert e with prefix[e] <= u < prefix[e+1] (empty experts share
  // their prefix with the next one, so the largest such e has rows)
  int lo = 0, hi = p.num_experts;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_prefix[mid] <= u) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int rows_e = s_off[e + 1] - s_off[e];
  const int mtiles = (rows_e + NTOK - 1) / NTOK;
  const int local = u - s_prefix[e];
  const int mt = local % mtiles;
  x.nt = local / mtiles;
  x.expert = e;
  x.row0 = s_off[e] + mt * NTOK;
  x.rows = min(NTOK, s_off[e + 1] - x.row0);
  x.kb0 = 0;
  x.kb1 = p.k_blocks;
  x.tile = 0;
  x.partial = 0;
  x.slot = 0;
  return true;
}

// Grouped mode: per-expert tile prefix sums from the device-resident row
// offsets (no host synchronization).  Called by every thread of the CTA;
// ends with the table visible to all of them.
template <int NTOK>
__device__ __forceinline__ void grouped_tables(const W4Params& p, int* s_off, int* s_prefix, int* s_total) {
  const int E = p.num_experts;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = p.expert_offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    bool bad = s_off[0] != 0 || s_off[E] != p.m;
    for (int e = 0; e < E; ++e) {
      s_prefix[e] = acc;
      int rows = s_off[e + 1] - s_off[e];
      if (rows < 0) { bad = true; rows = 0; }
      acc += ((rows + NTOK - 1) / NTOK) * p.n_tiles;
    }
    s_prefix[E] = acc;
    if (bad) {
      atomicCAS(p.err, 0u, (uint32_t)HQ_ERR_DEVICE_BAD_OFFSETS);
      acc = 0;
    }
    *s_total = acc;
  }
}

// Writes tokens j0 .. j0+EB-1 of one epilogue warp's 32 weight rows (row
// n = nt*128 + 32q + lane holds v[j] for token j0+j): fp32 into this CTA's
// partial slot for a partial unit, else bf16 output (store_rows_chunk); with
// SW (grouped gate+up weights in the gated row order, written as
// h = silu(gate) * up [rows][n/2]) the SwiGLU of the warp's 16 gate/up row
// pairs, 16 features of h from feature nt*64 + 16q (store_swiglu_chunk).
// SW is a kernel template parameter: the SwiGLU code would otherwise weigh
// on every other kernel's epilogue (measured ~4 % at M=4096 on B200).
template <int EB, bool SW>
__device__ __forceinline__ void store_chunk(const W4Params& p, const Unit& x, float* part, int q, int lane, int j0,
                                            const float (&v)[EB], uint16_t* sc) {
  if constexpr (SW)
    store_swiglu_chunk<EB>(p.c, p.n >> 1, x.row0, x.rows, x.nt * (kTileN / 2) + q * 16, lane, j0, v, sc);
  else
    store_rows_chunk<EB>(p.c, p.n, x.row0, x.rows, x.nt * kTileN + q * 32, q * 32 + lane, part, lane, j0, v, sc);
}

// Stream-K partial sums of a split tile.  Its contributors are the CTAs
// first..last whose k-block ranges cover it, in stream-K order, and each
// writes its fp32 partial into its own slot.  All but the last then signal
// (sk_signal) the tile counter of their epilogue warp and go on at once.
// The last contributor owns the tile's final k-blocks, which are the first
// unit of its range; it reduces the tile after its own last unit
// (sk_reduce), once the counter shows that the others have signalled --
// they have lower CTA indices, so they were dispatched first, and none of
// them waits for a CTA of higher index before signalling.  The sum runs
// over every partial in CTA order, so the result does not depend on
// timing.  (Letting whichever contributor arrives last reduce needs no
// wait, but puts a counter round trip into every contributor's pipeline,
// in the middle of its range for all but the first: measured on B200,
// M=16 K=18432 N=7168 32.6 us against 25.9 us with no fixup at all.)
__device__ __forceinline__ bool sk_is_reducer(const W4Params& p, const Unit& x) {
  return x.partial && x.kb1 == p.k_blocks;
}

static __device__ __noinline__ void sk_signal(const W4Params& p, const Unit& x, int q, int lane) {
  __threadfence();  // this lane's partial stores, visible before the signal
  __syncwarp();
  if (lane == 0) atomicAdd(p.counters + x.tile * 4 + q, 1);
}

// Not inlined: its registers stay out of the pipelined roles' allocation.
template <int NTOK, int CB = 4>
__device__ __noinline__ void sk_reduce(const W4Params& p, const Unit& x, int q, int lane) {
  const int r = q * 32 + lane;
  const int n = x.nt * kTileN + r;
  const bool n_ok = n < p.n;
  const long long T = p.total_iters, G = gridDim.x, kbl = p.k_blocks;
  const long long t0 = (long long)(x.tile - p.dp_tiles) * kbl;   // in the stream-K iteration space
  const long long first = sk_owner(t0, T, G), last = sk_owner(t0 + kbl - 1, T, G);
  int* ctr = p.counters + x.tile * 4 + q;
  if (lane == 0) {
    if (!hq_wait_count(ctr, (int)(last - first), p.wait_ns)) atomicCAS(p.err, 0u, (uint32_t)HQ_ERR_DEVICE_TIMEOUT);
    *ctr = 0;  // every other contributor has signalled: leave the counter at zero
  }
  __syncwarp();
  __threadfence();
  // 8 token rows at a time; the loads of up to CB contributors are in
  // flight together and the sum runs in contributor order (this CTA's own
  // partial, written by this lane, last)
  for (int j0 = 0; j0 < x.rows; j0 += 8) {
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (long long c0 = first; c0 <= last; c0 += CB) {
      float v[CB][8];
#pragma unroll
      for (int b = 0; b < CB; ++b) {
        if (c0 + b <= last) {
          const long long ci = c0 + b;
          const int sl = sk_start(ci, T, G) >= t0 ? 0 : 1;
          const float* src = p.partials + (((size_t)ci * 2 + sl) * NTOK + j0) * kTileN + r;
#pragma unroll
          for (int j = 0; j < 8; ++j) v[b][j] = __ldcg(src + (size_t)j * kTileN);
        }
      }
#pragma unroll
      for (int b = 0; b < CB; ++b) {
        if (c0 + b <= last) {
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] += v[b][j];
        }
      }
    }
    if (n_ok) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j0 + j < x.rows) p.c[(size_t)(x.row0 + j0 + j) * p.n + n] = __float2bfloat16_rn(acc[j]);
    }
  }
}

// Host side: the exact-weight kernel's ring depth, and its launch (16, 32 or
// 64 tokens; INT4, INT3, INT2 or INT8 records).
int small_ring_depth(int ntok, int fmt);
hq_status small_launch(int ntok, int fmt, bool swiglu, const CUtensorMap& map, const W4Params& p, int grid,
                       cudaStream_t stream);

}  // namespace w4
}  // namespace hq
