// Block-scaled 4-bit GEMMs for sm_100a: W4A8-MXFP4 (e2m1 weights with an
// E8M0 scale per 32 K, E4M3 activations with a per-token fp32 scale) and
// W4A4 NVFP4 (e2m1 with an E4M3 scale per 16 K and an fp32 tensor scale on
// each side).
//
// Method: the W4A8-MXFP4 and W4A4 combinations and the MXFP4 / NVFP4 types
// are listed on the Humming news page (section "one library, many formats",
// table row "W4A8-MXFP4, H200"); on GPUs without native MXFP4 the library
// converts the weights inside the kernel ("Humming: open-source kernel
// library for quantized inference", summary paragraph 4).  B200 has the
// native block-scaled tensor-core MMA, so here the codes go to the tensor
// core as they are and the scales ride along in TMEM.
//
// B200 design:
//   * swap-AB, as in the W4A16 kernel: 128 weight rows are the MMA's M side
//     (A operand), the token tile (16..256) is its N side (B operand); both
//     staged by TMA with the 128-byte swizzle.  MXFP4 weights use the TMA
//     type that unpacks 16 four-bit codes into a 16-byte slot, the layout
//     tcgen05.mma.kind::mxf8f6f4 reads; NVFP4 stays packed for
//     kind::mxf4nvf4.
//   * weight scales come from the packed blob, already in the 32x16-byte
//     order tcgen05.cp .32x128b.warpx4 copies into TMEM; NVFP4 activation
//     scales are loaded row-major by TMA and reordered in shared memory by
//     one warp; MXFP4 activations carry no block scale (their E8M0 scale is
//     1, set once in TMEM) and the per-token fp32 scale is applied in the
//     epilogue.
//   * warp roles: 0 producer, 1 MMA issuer (tcgen05.cp of the stage's scales
//     then its MMAs, in issue order), 2 TMEM allocator, 3 scale reorder
//     (NVFP4), 4-7 epilogue.  Dense stream-K with the deterministic
//     last-contributor reduction, as in the W4A16 kernel.
#include <cuda_bf16.h>

#include <algorithm>

#include "epilogue.cuh"
#include "hq_internal.h"
#include "ptx.cuh"

namespace hq {

namespace {

constexpr int kBsThreads = 384;    // 12 warps
constexpr int kBsTileN = 128;
constexpr int kBsEpiWarps = 8;
constexpr int kBsEB = 16;          // tokens per transposed output store

enum BsFmt { kMX = 0, kNV = 1 };

// MXFP4 stages of small token tiles carry several 128-K boxes (fewer,
// longer stages: the per-stage handshakes dominate there): three at 32
// tokens (measured on B200, M=64 K=N=7168 on 32-token tiles: 15.2 -> 14.1
// us against two), two at 16 and 64 (three gains nothing at 16); everything
// else one.
template <int FMT, int NTOK>
constexpr int bs_boxes() { return FMT == kMX && NTOK == 32 ? 3 : FMT == kMX && NTOK <= 64 ? 2 : 1; }

// CG = 2: a CTA pair (cluster of two) runs one 256-row weight tile with
// cta_group::2 MMAs; each CTA stages its own 128 weight rows and half of the
// token tile, and the scales of the whole token tile.
template <int FMT, int NTOK, int CG = 1>
struct BsCfg {
  static_assert(CG == 1 || (CG == 2 && NTOK >= 128), "CTA pairs run 128- or 256-token tiles");
  static constexpr int kBox = bs_boxes<FMT, NTOK>();        // 128-B-row boxes along K per stage
  static constexpr int kKBox = FMT == kNV ? 256 : 128;     // K elements per box: 128 B per row in SMEM
  static constexpr int kATileBox = kBsTileN * 128;         // weights in SMEM, one box
  static constexpr int kATile = kBox * kATileBox;
  // bytes the weight copy moves: NVFP4 loads packed bytes; the MXFP4 load
  // unpacks 4-bit codes into 16-byte slots and counts the packed bytes
  static constexpr int kATxBox = FMT == kNV ? kATileBox : kBsTileN * 64;
  static constexpr int kBTileBox = NTOK / CG * 128;        // this CTA's activations, one box
  static constexpr int kBTile = kBox * kBTileBox;
  static constexpr int kSfaBox = FMT == kNV ? 2048 : 512;  // weight scale chunks per box
  static constexpr int kSfa = kBox * kSfaBox;
  static constexpr int kHalves = NTOK > 128 ? 2 : 1;       // 128-token halves of the token tile
  static constexpr int kSfb = FMT == kNV ? 4 * kHalves * 512 : 0;   // activation scale chunks per stage
  static constexpr int kStageRaw = kATile + kBTile + kSfa + kSfb;
  static constexpr int kStage = (kStageRaw + 1023) / 1024 * 1024;
  static constexpr int kBarBytes = 512;
  static constexpr int kScratch = kBsEpiWarps * 32 * kBsEB * 2;   // output transposes
  static constexpr int kStages = std::min(10, (232448 - 1024 - kBarBytes - kScratch) / kStage);
  static constexpr int kAcc = NTOK <= 128 ? 2 : 1;
  static constexpr int kCols = NTOK / 2;                   // accumulator columns per epilogue warp
  // TMEM columns: accumulators, then per-stage scale slots
  static constexpr int kSfaCols = FMT == kNV ? 16 : 4 * kBox;
  static constexpr int kSfbCols = FMT == kNV ? 16 * kHalves : 0;
  static constexpr int kSfSlot = kSfaCols + kSfbCols;
  static constexpr int kSfBase = kAcc * NTOK;
  static constexpr int kSfbConst = kSfBase + kStages * kSfSlot;   // MXFP4: constant unit scales (8 cols)
  static constexpr size_t kBarOff = (size_t)kStages * kStage;
  static constexpr size_t kScrOff = kBarOff + kBarBytes;
  static constexpr size_t kSmem = 1024 + kScrOff + kScratch;
  static_assert(kStages >= 3, "pipeline depth");
  static_assert(kSfbConst + 8 <= 512, "TMEM budget");
  static_assert(8 * (2 * kStages + 5) + 16 <= kBarBytes, "barrier area");
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(kBTileBox % 1024 == 0 && kATileBox % 1024 == 0, "128-byte swizzle atoms");
};

struct BsParams {
  const uint8_t* sf_w;       // weight scale chunks (blob + codes bytes)
  const uint8_t* sf_a;       // NVFP4: activation scale chunks, [m_tiles][k_stages][kSfb] (workspace)
  __nv_bfloat16* c;
  const float* a_scale;      // MXFP4: per-token scale [m]
  const float* g_w;          // NVFP4: weight tensor scale (blob tail)
  float a_global;            // NVFP4: activation tensor scale
  float* partials;
  int32_t* counters;         // [tiles][8], one per epilogue warp
  uint32_t* err;
  uint64_t wait_ns;
  long long total_iters;
  int m, n, k;
  int n_tiles, k_stages;
  int k_boxes;               // 128-B-row boxes along K (K/256 for NVFP4, K/128 for MXFP4)
  int sf_groups;             // 512-byte scale chunks per weight tile (whole K)
  int m_tiles;
  int data_parallel;         // whole tiles per unit, no partial sums
  int early_weights;         // fetch the first stages' weights before griddepcontrol.wait
  int stage_limit;           // pipeline stages in flight (0 or >= the ring depth: the whole ring)
  int n_pairs;               // CTA pairs: 256-row weight tiles (n_tiles / 2)
  int raster;                // whole-tile order: groups of this many weight tiles (pairs) over all token tiles
};

// Whole-tile order: unit t -> (token tile, weight tile) in groups of `width`
// weight tiles, each group walking every token tile before the next group
// starts, so that the CTAs of one wave share few weight tiles (width =
// n_w is plain token-tile-major order).
__device__ __forceinline__ void raster_tile(long long t, int n_w, int m_tiles, int width, int& mt, int& wt) {
  const long long per_group = (long long)width * m_tiles;
  const long long g = t / per_group, r = t - g * per_group;
  const int w = min(width, n_w - (int)g * width);   // the last group may be narrower
  mt = (int)(r / w);
  wt = (int)g * width + (int)(r - (long long)mt * w);
}

// NVFP4 activation scales, row-major [m][K/16] bytes, re-laid into the order
// tcgen05.cp .32x128b.warpx4 copies into TMEM: per (token tile mt, stage
// ks), chunk (MMA i, token half h) is 512 bytes whose byte l*16 + 4c + j is
// the scale of token h*128 + 32c + l of the tile, K block 16*ks + 4i + j
// (zero past the tile or the last row).  One thread per 32-bit word.
__global__ void sfb_relayout_kernel(const uint32_t* __restrict__ sf, int m, int kw, int ntok, int halves,
                                    int k_stages, uint32_t* __restrict__ out, long long words) {
  for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < words;
       w += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(w & 3);
    const int l = (int)((w >> 2) & 31);
    long long rest = w >> 7;
    const int ih = (int)(rest % (4 * halves));
    rest /= 4 * halves;
    const int ks = (int)(rest % k_stages);
    const long long mt = rest / k_stages;
    const int i = ih / halves, h = ih % halves;
    const int tok = h * 128 + 32 * c + l;
    const long long row = mt * ntok + tok;
    out[w] = (tok < ntok && row < m) ? __ldg(sf + row * kw + ks * 4 + i) : 0u;
  }
}

template <int FMT, int NTOK, int CG = 1>
__device__ __forceinline__ bool bs_unit(const BsParams& p, int idx, int& tile, int& nt, int& row0, int& rows,
                                        int& ks0, int& ks1, int& partial, int& slot) {
  if constexpr (CG == 2) {
    // whole (token tile, 256-row weight tile) units over the clusters; CTA
    // rank r of the pair owns 128-row weight tile 2 * pair + r
    const long long ncl = gridDim.x / 2, cl = blockIdx.x / 2;
    const long long t = cl + (long long)idx * ncl;
    if (t >= (long long)p.m_tiles * p.n_pairs) return false;
    int mt, pnt;
    raster_tile(t, p.n_pairs, p.m_tiles, p.raster, mt, pnt);
    tile = (int)t;
    nt = 2 * pnt + (int)(blockIdx.x & 1);
    row0 = mt * NTOK;
    rows = min(NTOK, p.m - row0);
    ks0 = 0;
    ks1 = p.k_stages;
    partial = 0;
    slot = 0;
    return true;
  }
  if (p.data_parallel) {
    const long long t = (long long)blockIdx.x + (long long)idx * gridDim.x;
    if (t >= (long long)p.m_tiles * p.n_tiles) return false;
    int mt;
    raster_tile(t, p.n_tiles, p.m_tiles, p.raster, mt, nt);
    tile = (int)t;
    row0 = mt * NTOK;
    rows = min(NTOK, p.m - row0);
    ks0 = 0;
    ks1 = p.k_stages;
    partial = 0;
    slot = 0;
    return true;
  }
  const long long T = p.total_iters, G = gridDim.x, i = blockIdx.x;
  const long long beg = sk_start(i, T, G), end = sk_start(i + 1, T, G);
  const long long kst = p.k_stages;
  const long long t = beg / kst + idx;
  const long long x0 = idx == 0 ? beg : t * kst;
  if (x0 >= end) return false;
  const long long x1 = min(end, (t + 1) * kst);
  const int mt = (int)(t / p.n_tiles);
  tile = (int)t;
  nt = (int)(t - (long long)mt * p.n_tiles);
  row0 = mt * NTOK;
  rows = min(NTOK, p.m - row0);
  ks0 = (int)(x0 - t * kst);
  ks1 = (int)(x1 - t * kst);
  partial = (ks0 != 0 || ks1 != p.k_stages) ? 1 : 0;
  slot = idx == 0 ? 0 : 1;
  return true;
}

// Stream-K partial sums, as in the W4A16 kernels: one counter per (tile,
// epilogue warp).  Every contributor of a split tile writes its partial
// slot; all but the last signal and go on; the last (the owner of the
// tile's final k-stages, the first unit of its range) reduces the tile
// after its own last unit, once the others -- all of lower CTA index --
// have signalled: every partial in CTA order (8 tokens at a time, the
// loads of up to CB contributors in flight together), then the scaled
// output.
__device__ __noinline__ void bs_signal(const BsParams& p, int tile, int wslot, int lane) {
  __threadfence();  // this lane's partial stores, visible before the signal
  __syncwarp();
  if (lane == 0) atomicAdd(p.counters + tile * kBsEpiWarps + wslot, 1);
}

template <int FMT, int NTOK, int CB>
__device__ __noinline__ void bs_reduce(const BsParams& p, int tile, int nt, int row0, int rows, int tok0, int wslot,
                                       int r, int lane, float alpha) {
  constexpr int NC = BsCfg<FMT, NTOK>::kCols;
  const int rows_w = rows - tok0;
  const long long T = p.total_iters, G = gridDim.x, kst = p.k_stages;
  const long long t0 = (long long)tile * kst;
  const long long first = sk_owner(t0, T, G), last = sk_owner(t0 + kst - 1, T, G);
  int* ctr = p.counters + tile * kBsEpiWarps + wslot;
  if (lane == 0) {
    if (!hq_wait_count(ctr, (int)(last - first), p.wait_ns)) atomicCAS(p.err, 0u, (uint32_t)HQ_ERR_DEVICE_TIMEOUT);
    *ctr = 0;  // every other contributor has signalled: leave the counter at zero
  }
  __syncwarp();
  __threadfence();
  const int n = nt * kBsTileN + r;
  for (int j0 = 0; j0 < NC && j0 < rows_w; j0 += 8) {
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (long long c0 = first; c0 <= last; c0 += CB) {
      float w[CB][8];
#pragma unroll
      for (int b = 0; b < CB; ++b) {
        if (c0 + b <= last) {
          const long long ci = c0 + b;
          const int sl = sk_start(ci, T, G) >= t0 ? 0 : 1;
          const float* srcp = p.partials + (((size_t)ci * 2 + sl) * NTOK + tok0 + j0) * kBsTileN + r;
#pragma unroll
          for (int j = 0; j < 8; ++j) w[b][j] = __ldcg(srcp + (size_t)j * kBsTileN);
        }
      }
#pragma unroll
      for (int b = 0; b < CB; ++b) {
        if (c0 + b <= last) {
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] += w[b][j];
        }
      }
    }
    if (n < p.n) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j0 + j < rows_w) {
          const int tk = tok0 + j0 + j;
          const float sc = FMT == kNV ? alpha : __ldg(p.a_scale + row0 + tk);
          p.c[(size_t)(row0 + tk) * p.n + n] = __float2bfloat16_rn(acc[j] * sc);
        }
      }
    }
  }
}

template <int FMT, int NTOK, int CG>
__global__ void __launch_bounds__(kBsThreads, 1)
    blockscaled_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_a,
                       const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                       const BsParams p) {
  using C = BsCfg<FMT, NTOK, CG>;
  constexpr int S = C::kStages;
  constexpr int ACC = C::kAcc;
  constexpr int NC = C::kCols;
  // bytes of a stage with nb boxes (this CTA's share)
  auto stage_tx = [](int nb) -> uint32_t {
    return (uint32_t)(nb * (C::kATxBox + C::kBTileBox + C::kSfaBox) + C::kSfb);
  };
  // boxes of stage ks (the last one of an odd box count has one)
  auto stage_boxes = [&](int ks) -> int { return min(C::kBox, p.k_boxes - ks * C::kBox); };

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  uint16_t* scratch = reinterpret_cast<uint16_t*>(smem + C::kScrOff);   // 16-byte aligned

  auto sA = [&](int s) { return smem + s * C::kStage; };
  auto sB = [&](int s) { return smem + s * C::kStage + C::kATile; };
  auto sSfa = [&](int s) { return smem + s * C::kStage + C::kATile + C::kBTile; };
  auto sSfb = [&](int s) { return sSfa(s) + C::kSfa; };

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  // CTA pairs: rank 0 issues the pair's MMAs; every stage's copies of both
  // CTAs complete on rank 0's full barrier
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kBsEpiWarps * CG);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_w);
    prefetch_tensormap(&tmap_a);
    if (CG == 2) {
      prefetch_tensormap(&tmap_sfa);
      if (FMT == kNV) prefetch_tensormap(&tmap_sfb);
    }
  }
  if (threadIdx.x == 0) pdl_launch_dependents();
  if constexpr (CG == 2) {
    // MXFP4 activations carry no block scale: 32 rows x 16 bytes of E8M0 127
    // (= 1.0) that rank 0 copies into both CTAs' TMEM before its first MMA
    if (FMT == kMX && threadIdx.x < 128) reinterpret_cast<uint32_t*>(scratch)[threadIdx.x] = 0x7F7F7F7Fu;
    // the pair's TMEM is allocated by both CTAs together; the barriers and
    // the allocation are visible to both CTAs after the cluster barrier
    if (warp == 2) {
      tmem_alloc_pair(s_tmem, 512);
      tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
  } else {
    __syncthreads();   // barriers visible to every role
  }

  int tile, nt, row0, rows, ks0, ks1, partial, slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp, one lane issues)
    const bool leader = elect_one();
    const uint64_t pol_w = policy_evict_first();
    // rank 0's full barrier of stage s, as a cluster address (pairs)
    auto full_cl = [&](int s) -> uint32_t { return CG == 2 ? mapa_u32(&full[s], 0) : 0u; };
    // weights of stage it: codes (K coordinate in elements for the MXFP4
    // unpacking type, in bytes for NVFP4) and their scale chunks
    auto load_weights = [&](int s, int ks, int nt_) {
      const int nb = stage_boxes(ks);
      const int chunks = FMT == kNV ? 4 : 1;   // 512-byte scale chunks per box
      if constexpr (CG == 2) {
        const uint32_t fb = full_cl(s);
        for (int b = 0; b < nb; ++b) {
          const int kbox = ks * C::kBox + b;
          tma_load_2d_pair(sA(s) + b * C::kATileBox, &tmap_w, FMT == kNV ? kbox * 128 : kbox * C::kKBox,
                           nt_ * kBsTileN, fb);
        }
        // scale chunks as rows of 128 words
        tma_load_2d_pair(sSfa(s), &tmap_sfa, 0, nt_ * p.sf_groups + ks * C::kBox * chunks, fb);
      } else {
        for (int b = 0; b < nb; ++b) {
          const int kbox = ks * C::kBox + b;
          tma_load_2d(sA(s) + b * C::kATileBox, &tmap_w, FMT == kNV ? kbox * 128 : kbox * C::kKBox, nt_ * kBsTileN,
                      &full[s]);
        }
        const uint8_t* src = p.sf_w + ((size_t)nt_ * p.sf_groups + (size_t)ks * C::kBox * chunks) * 512;
        bulk_g2s(sSfa(s), src, (uint32_t)(nb * C::kSfaBox), &full[s], pol_w);
      }
    };
    // Phase 1, before the previous kernel on the stream has finished: the
    // packed weights of the first S stages (no kernel writes them)
    uint32_t n_pre = 0;
    const uint32_t lim = (p.stage_limit > 0 && p.stage_limit < S) ? (uint32_t)p.stage_limit : (uint32_t)S;
    for (int idx = 0; p.early_weights && n_pre < lim &&
                      bs_unit<FMT, NTOK, CG>(p, idx, tile, nt, row0, rows, ks0, ks1, partial, slot);
         ++idx) {
      for (int ks = ks0; ks < ks1 && n_pre < lim; ++ks, ++n_pre) {
        if (leader) {
          // rank 0 expects the bytes of both CTAs of a pair
          if (rank == 0) mbar_arrive_expect_tx(&full[n_pre], CG * stage_tx(stage_boxes(ks)));
          load_weights((int)n_pre, ks, nt);
        }
        __syncwarp();
      }
    }
    pdl_wait();
    // Phase 2: activations (and their scales) of those stages, then the ring
    uint32_t it = 0;
    bool ok = true;
    for (int idx = 0; ok && bs_unit<FMT, NTOK, CG>(p, idx, tile, nt, row0, rows, ks0, ks1, partial, slot); ++idx) {
      for (int ks = ks0; ks < ks1; ++ks, ++it) {
        const int s = it % S;
        if (!wait_stage_free<S>(empty, it, lim, p.wait_ns, s_abort)) {
          if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        if (leader) {
          if (it >= n_pre) {
            if (rank == 0) mbar_arrive_expect_tx(&full[s], CG * stage_tx(stage_boxes(ks)));
            load_weights(s, ks, nt);
          }
          if constexpr (CG == 2) {
            const uint32_t fb = full_cl(s);
            // this CTA's half of the token tile
            for (int b = 0; b < stage_boxes(ks); ++b)
              tma_load_2d_pair(sB(s) + b * C::kBTileBox, &tmap_a, (ks * C::kBox + b) * 128,
                               row0 + (int)rank * (NTOK / 2), fb);
            if (FMT == kNV)
              tma_load_2d_pair(sSfb(s), &tmap_sfb, 0, ((row0 / NTOK) * p.k_stages + ks) * (C::kSfb / 512), fb);
          } else {
            for (int b = 0; b < stage_boxes(ks); ++b)
              tma_load_2d(sB(s) + b * C::kBTileBox, &tmap_a, (ks * C::kBox + b) * 128, row0, &full[s]);
            if (FMT == kNV) {
              const uint8_t* sfb = p.sf_a + ((size_t)(row0 / NTOK) * p.k_stages + ks) * C::kSfb;
              bulk_g2s(sSfb(s), sfb, C::kSfb, &full[s], policy_evict_last());
            }
          }
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      if constexpr (CG == 2) {
        // this CTA's copies complete on rank 0's barriers: give the last
        // ones issued time to land before the CTA can exit
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 50000) {
        }
      } else {
        const uint32_t first = it > (uint32_t)S ? it - S : 0;
        for (uint32_t j = first; j < it; ++j) hq_wait(&full[j % S], (j / S) & 1, p.wait_ns, nullptr);
      }
    }
  } else {
  // The producer needs no TMEM, so it starts loading at once; the other
  // roles wait here for the allocation (and, for MXFP4, the unit scales).
  if (CG == 1 && warp == 2) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  pdl_wait();   // outputs, partials and counters may be in use by the previous kernel
  tc_fence_before();
  named_bar(1, kBsThreads - 32);
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  if (CG == 1 && FMT == kMX) {
    if (warp >= 4 && warp < 8) {
      // activations carry no block scale: E8M0 127 (= 1.0) in every byte
      tmem_st_x8(tmem_base + (((warp & 3) * 32) << 16) + C::kSfbConst, 0x7F7F7F7Fu);
      tmem_wait_st();
    }
    tc_fence_before();
    named_bar(2, kBsThreads - 32);
    tc_fence_after();
  }
  if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one fixed lane issues)
    // (pairs: rank 0 only, for both CTAs)
    const bool leader = elect_one();
    uint32_t it = 0, uc = 0;
    bool ok = rank == 0;
    if (CG == 2 && FMT == kMX && ok) {
      // the unit scales: 8 columns, as the one-CTA kernel stores them
      if (leader) {
        tmem_cp_sf_pair(tmem_base + C::kSfbConst, smem_desc_sf(smem_u32(scratch)));
        tmem_cp_sf_pair(tmem_base + C::kSfbConst + 4, smem_desc_sf(smem_u32(scratch)));
      }
      __syncwarp();
    }
    for (int idx = 0; ok && bs_unit<FMT, NTOK, CG>(p, idx, tile, nt, row0, rows, ks0, ks1, partial, slot);
         ++idx, ++uc) {
      const int ab = uc % ACC;
      const uint32_t aph = (uc / ACC) & 1;
      // (pairs: the epilogue warps of both CTAs arrive)
      if (!(CG == 2 ? hq_wait_warp_cl(&acc_empty[ab], aph ^ 1, p.wait_ns, s_abort)
                    : hq_wait_warp(&acc_empty[ab], aph ^ 1, p.wait_ns, s_abort))) {
        if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + ab * NTOK;
      for (int ks = ks0; ks < ks1; ++ks, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!hq_wait_warp(&full[s], ph, p.wait_ns, s_abort)) {
          if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA(s));
        const uint32_t b_base = smem_u32(sB(s));
        const uint32_t sf_col = C::kSfBase + s * C::kSfSlot;
        if (leader) {
          // descriptors: the K step (32 B) and the scale chunks (512 B) only
          // move the low word's 14-bit start-address field, which cannot
          // overflow inside shared memory
          const uint64_t ad = smem_desc_sw128(a_base), bd = smem_desc_sw128(b_base);
          auto step = [](uint64_t desc, uint32_t bytes) {
            return (desc & 0xFFFFFFFF00000000ull) | (uint64_t)((uint32_t)desc + (bytes >> 4));
          };
          const uint32_t acc0 = ks > ks0 ? 1u : 0u;
          if (FMT == kNV) {
            const uint64_t fa = smem_desc_sf(smem_u32(sSfa(s))), fb = smem_desc_sf(smem_u32(sSfb(s)));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t sfa_t = tmem_base + sf_col + 4 * i;
              const uint32_t sfb_t = tmem_base + sf_col + 16 + 4 * C::kHalves * i;
              constexpr uint32_t kId = idesc_block_scaled(1, 1, 0, 128 * CG, NTOK, 0, 0);
              if constexpr (CG == 2) {
                tmem_cp_sf_pair(sfa_t, step(fa, 512 * i));
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                  tmem_cp_sf_pair(sfb_t + 4 * h, step(fb, 512 * (i * C::kHalves + h)));
                mma_mxf4nvf4_pair(d_tmem, step(ad, 32 * i), step(bd, 32 * i), kId, sfa_t, sfb_t, i > 0 ? 1u : acc0);
              } else {
                tmem_cp_sf(sfa_t, step(fa, 512 * i));
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                  tmem_cp_sf(sfb_t + 4 * h, step(fb, 512 * (i * C::kHalves + h)));
                mma_mxf4nvf4(d_tmem, step(ad, 32 * i), step(bd, 32 * i), kId, sfa_t, sfb_t, i > 0 ? 1u : acc0);
              }
            }
          } else {
            const uint64_t fa = smem_desc_sf(smem_u32(sSfa(s)));
            const int nb = stage_boxes(ks);
#pragma unroll
            for (int b = 0; b < C::kBox; ++b) {
              if (b < nb) {
                const uint32_t sfa_t = tmem_base + sf_col + 4 * b;
                if constexpr (CG == 2)
                  tmem_cp_sf_pair(sfa_t, step(fa, 512 * b));
                else
                  tmem_cp_sf(sfa_t, step(fa, 512 * b));
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  // byte i of each scale column holds the scale of 32-K block i
                  const uint32_t id = idesc_block_scaled(5, 0, 1, 128 * CG, NTOK, (uint32_t)i, 0);
                  const uint64_t a_d = step(ad, b * C::kATileBox + 32 * i), b_d = step(bd, b * C::kBTileBox + 32 * i);
                  const uint32_t acc = (b > 0 || i > 0) ? 1u : acc0;
                  if constexpr (CG == 2)
                    mma_mxf8f6f4_pair(d_tmem, a_d, b_d, id, sfa_t, tmem_base + C::kSfbConst, acc);
                  else
                    mma_mxf8f6f4(d_tmem, a_d, b_d, id, sfa_t, tmem_base + C::kSfbConst, acc);
                }
              }
            }
          }
          // the stage's slot in both CTAs of a pair is free once these MMAs are done
          if constexpr (CG == 2)
            tc_commit_pair(&empty[s]);
          else
            tc_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (leader) {
        if constexpr (CG == 2)
          tc_commit_pair(&acc_full[ab]);
        else
          tc_commit(&acc_full[ab]);
      }
      __syncwarp();
    }
    if (leader && (CG == 1 || rank == 0)) {
      if constexpr (CG == 2)
        tc_commit_pair_local(drain);
      else
        tc_commit(drain);
      hq_wait(drain, 0, p.wait_ns, nullptr);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (8 warps)
    // warp 4 + 4*hc + q owns weight rows 32q..32q+31 and tokens
    // hc*NC .. hc*NC+NC-1 of the tile.  It copies its accumulator columns
    // into registers and hands the accumulator back to the MMA at once, then
    // scales and stores while the next unit's MMAs run.
    const uint32_t q = warp & 3;
    const int hc = (int)(warp - 4) >> 2;
    const int r = (int)(q * 32 + lane);
    const uint32_t lane_addr = (q * 32) << 16;
    const int wslot = hc * 4 + (int)q;
    uint16_t* scr = scratch + (warp - 4) * (32 * kBsEB);
    const float alpha = FMT == kNV ? p.a_global * __ldg(p.g_w) : 1.f;
    uint32_t uc = 0;
    bool ok = true;
    int pend_tile = -1, pend_nt = 0, pend_row0 = 0, pend_rows = 0;   // the split tile this CTA reduces last
    for (int idx = 0; bs_unit<FMT, NTOK, CG>(p, idx, tile, nt, row0, rows, ks0, ks1, partial, slot); ++idx, ++uc) {
      const int ab = uc % ACC;
      const uint32_t aph = (uc / ACC) & 1;
      if (!hq_wait(&acc_full[ab], aph, p.wait_ns, s_abort)) {
        raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[NC];
      const uint32_t src = tmem_base + lane_addr + ab * NTOK + hc * NC;
      if constexpr (NC == 8) {
        tmem_ld_x8(src, *reinterpret_cast<uint32_t(*)[8]>(v));
      } else {
#pragma unroll
        for (int j0 = 0; j0 < NC; j0 += 16) tmem_ld_x16(src + j0, *reinterpret_cast<uint32_t(*)[16]>(v + j0));
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // (pairs: the accumulator's owner is rank 0's MMA issuer)
        if constexpr (CG == 2)
          mbar_arrive_cluster(mapa_u32(&acc_empty[ab], 0));
        else
          mbar_arrive(&acc_empty[ab]);
      }

      const int tok0 = hc * NC;                       // first token of this warp's run
      const int rows_w = rows - tok0;                 // valid tokens in the run (may be <= 0)
      float* part = partial ? p.partials + (((size_t)blockIdx.x * 2 + slot) * NTOK + tok0) * kBsTileN : nullptr;
      constexpr int EB = NC < kBsEB ? NC : kBsEB;
#pragma unroll
      for (int j0 = 0; j0 < NC; j0 += EB) {
        float f[EB];
        if (FMT == kMX && !partial) {
          // per-token scales: lane j reads token j of the run, then broadcast
          const int tk = tok0 + j0 + (int)(lane % EB);
          const float mine = tk < rows ? __ldg(p.a_scale + row0 + tk) : 0.f;
#pragma unroll
          for (int j = 0; j < EB; ++j) f[j] = __uint_as_float(v[j0 + j]) * __shfl_sync(0xffffffffu, mine, j);
        } else {
#pragma unroll
          for (int j = 0; j < EB; ++j) f[j] = partial ? __uint_as_float(v[j0 + j]) : __uint_as_float(v[j0 + j]) * alpha;
        }
        store_rows_chunk<EB>(p.c, p.n, row0 + tok0, rows_w, nt * kBsTileN + (int)q * 32, r, part, (int)lane, j0, f,
                             scr);
      }
      if (CG == 1 && partial) {
        if (ks1 == p.k_stages) {
          pend_tile = tile;
          pend_nt = nt;
          pend_row0 = row0;
          pend_rows = rows;
        } else {
          bs_signal(p, tile, wslot, (int)lane);
        }
      }
    }
    // (the 256-token tile keeps 128 accumulator registers per thread: fewer
    // contributors in flight there)
    if (CG == 1 && ok && pend_tile >= 0)
      bs_reduce<FMT, NTOK, (NTOK > 128 ? 1 : 4)>(p, pend_tile, pend_nt, pend_row0, pend_rows, hc * NC, wslot, r,
                                                 (int)lane, alpha);
  }

  }  // non-producer roles

  tc_fence_before();
  __syncthreads();
  // a pair's CTAs leave together: rank 0's MMAs read the other CTA's shared
  // memory and write its TMEM until rank 0 has drained them
  if constexpr (CG == 2) cluster_sync();
  tc_fence_after();
  if (warp == 2) {
    if constexpr (CG == 2)
      tmem_dealloc_pair(*s_tmem, 512);
    else
      tmem_dealloc(*s_tmem, 512);
  }
}

template <int FMT, int NTOK, int CG>
bool bs_smem_attr() {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && attr_set[dev]) return true;
  if (cudaFuncSetAttribute(blockscaled_kernel<FMT, NTOK, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)BsCfg<FMT, NTOK, CG>::kSmem) != cudaSuccess)
    return false;
  if (dev < 64) attr_set[dev] = true;
  return true;
}

template <int FMT, int NTOK, int CG>
hq_status bs_launch_t(const CUtensorMap& mw, const CUtensorMap& ma, const CUtensorMap& msfa, const CUtensorMap& msfb,
                      const BsParams& p, int grid, cudaStream_t stream) {
  auto kern = blockscaled_kernel<FMT, NTOK, CG>;
  const size_t smem = BsCfg<FMT, NTOK, CG>::kSmem;
  if (!bs_smem_attr<FMT, NTOK, CG>()) return HQ_ERR_CUDA;
  const cudaError_t e = CG == 2 ? launch_pdl_pairs(kern, dim3(grid), dim3(kBsThreads), smem, stream, mw, ma, msfa, msfb, p)
                                : launch_pdl(kern, dim3(grid), dim3(kBsThreads), smem, stream, mw, ma, msfa, msfb, p);
  return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

// Clusters of two of the CTA-pair kernel that are resident at once (0 when
// the query fails), per device.
template <int FMT, int NTOK>
int bs_pair_slots_t() {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  if (!bs_smem_attr<FMT, NTOK, 2>()) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kBsThreads);
  cfg.dynamicSmemBytes = BsCfg<FMT, NTOK, 2>::kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, blockscaled_kernel<FMT, NTOK, 2>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev < 64) cached[dev] = n;
  return n;
}
int bs_pair_slots(bool nv, int ntok) {
  if (nv) return ntok == 128 ? bs_pair_slots_t<kNV, 128>() : bs_pair_slots_t<kNV, 256>();
  return ntok == 128 ? bs_pair_slots_t<kMX, 128>() : bs_pair_slots_t<kMX, 256>();
}

// 128-B-row boxes along K, and pipeline stages (bs_boxes boxes each).
long long bs_k_boxes(const hq_quant_desc& d) { return d.k / (d.fmt == HQ_FMT_NVFP4 ? 256 : 128); }
long long bs_k_stages(const hq_quant_desc& d, int ntok) {
  const int box = d.fmt != HQ_FMT_MXFP4 ? 1 : ntok == 32 ? 3 : ntok <= 64 ? 2 : 1;   // bs_boxes<FMT, NTOK>()
  return (bs_k_boxes(d) + box - 1) / box;
}

int bs_tiles(const hq_quant_desc& d, int m, int ntok) {
  return ((d.n + kBsTileN - 1) / kBsTileN) * ((m + ntok - 1) / ntok);
}

}  // namespace

namespace {
BsConfig bs_plan_rules(const DeviceInfo& dev, const hq_quant_desc& d, int m, const hq_tuning* t) {
  BsConfig cfg{};
  // no tuning from the caller: the caller's per-shape table first, then the rules below
  hq_tuning from_table;
  if (!t) t = tuning_from_table(d, m, &from_table);
  cfg.early_weights = (t && (t->flags & HQ_TUNE_NO_EARLY_WEIGHTS)) ? 0 : 1;
  cfg.stages = t ? t->stages : 0;
  cfg.cta_group = 1;
  if (t && t->cta_group == 2) {
    // CTA pairs: whole 256-row weight tiles of 128 or 256 tokens, one per
    // resident cluster at a time
    cfg.cta_group = 2;
    cfg.ntok = t->tile_m ? t->tile_m : (m <= 128 ? 128 : 256);
    cfg.splits = 0;
    const long long pair_tiles = (long long)(d.n / 256) * ((m + cfg.ntok - 1) / cfg.ntok);
    const long long slots = bs_pair_slots(d.fmt == HQ_FMT_NVFP4, cfg.ntok);
    cfg.grid = (int)(2 * std::max<long long>(1, std::min<long long>(slots > 0 ? slots : dev.num_sms / 2, pair_tiles)));
    return cfg;
  }
  int ntok = (t && t->tile_m) ? t->tile_m : 0;
  if (!ntok) ntok = m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : m <= 128 ? 128 : 256;
  auto dp_eff = [&](int nt) {
    const long long tl = bs_tiles(d, m, nt);
    const long long waves = (tl + dev.num_sms - 1) / dev.num_sms;
    return (double)tl / (double)(waves * dev.num_sms);
  };
  if (t && t->split_k > 0) {
    const long long ks = bs_k_stages(d, ntok);
    cfg.ntok = ntok;
    cfg.splits = t->split_k;
    cfg.grid = (int)std::max<long long>(1, std::min<long long>((long long)bs_tiles(d, m, ntok) * t->split_k,
                                                                (long long)bs_tiles(d, m, ntok) * ks));
    return cfg;
  }
  // Whole tiles when they fill the SMs well, a token tile dropping to a
  // smaller one for that (one step when that fills >= 85 % of the SMs; down
  // to 32 tokens for >= 70 %); else an even K split when whole tiles fill
  // under half the SMs; else stream-K.  Measured on B200 (K=N=7168), the
  // fp32 partial tiles of a shared K range cost more than idle SMs here:
  // MXFP4 M=256: 128-token whole tiles on 112 SMs 23.1 us, 256-token
  // stream-K 36.8 us; M=64: 32-token whole tiles 14.5 us, stream-K 17.5;
  // M=16: two K halves per tile on 112 SMs 11.7 us, stream-K 12.8.
  const bool fixed_tile = t && t->tile_m;
  int pick = 0;
  if (!fixed_tile) {
    for (int nt = ntok; nt >= ntok / 2 && nt >= 64 && !pick; nt /= 2)
      if (dp_eff(nt) >= 0.85) pick = nt;
    for (int nt = ntok; nt >= 32 && !pick; nt /= 2)
      if (dp_eff(nt) >= 0.7) pick = nt;
    if (pick) ntok = pick;
  }
  cfg.ntok = ntok;
  const long long ks = bs_k_stages(d, ntok);
  const long long tiles = bs_tiles(d, m, ntok);
  if (pick || dp_eff(ntok) >= 0.85) {
    cfg.splits = 0;
    cfg.grid = (int)std::min<long long>(dev.num_sms, tiles);
    // 128/256-token whole tiles run on CTA pairs when the pairs' waves are
    // as full (the caller may ask for one CTA per tile with cta_group 1).
    // Measured on B200, one CTA per tile -> pairs: NVFP4 8192^3 244 -> 204
    // us, M=16384 K=7168 N=18432 990 -> 898 us, M=256 K=N=8192 20.7 ->
    // 17.9 us; MXFP4 K=N=7168 M=4096 159 -> 147 us, M=2048 128 -> 109 us,
    // M=256 23.2 -> 21.5 us.
    if (ntok >= 128 && d.n % 256 == 0 && !(t && t->cta_group == 1)) {
      const long long pair_tiles = (long long)(d.n / 256) * ((m + ntok - 1) / ntok);
      const long long slots = bs_pair_slots(d.fmt == HQ_FMT_NVFP4, ntok);
      if (slots > 0) {
        const long long waves = (pair_tiles + slots - 1) / slots;
        if ((double)pair_tiles / (double)(waves * slots) >= dp_eff(ntok) - 0.02) {
          cfg.cta_group = 2;
          cfg.grid = (int)(2 * std::min<long long>(slots, pair_tiles));
        }
      }
    }
    return cfg;
  }
  if (tiles * 2 <= dev.num_sms && tiles * (dev.num_sms / tiles) >= 0.7 * dev.num_sms) {
    cfg.splits = (int)(dev.num_sms / tiles);
    cfg.grid = (int)std::min<long long>(tiles * cfg.splits, tiles * ks);
    return cfg;
  }
  cfg.splits = 1;
  cfg.grid = (int)std::max<long long>(1, std::min<long long>(dev.num_sms, tiles * ks / 4));
  return cfg;
}
}  // namespace

BsConfig bs_plan(const DeviceInfo& dev, const hq_quant_desc& d, int m, const hq_tuning* t) {
  BsConfig cfg = bs_plan_rules(dev, d, m, t);
  // eight tile counters per output tile, in the workspace's fixed counter region
  if (cfg.splits != 0 && (size_t)bs_tiles(d, m, cfg.ntok) * kBsEpiWarps * sizeof(int32_t) > kWsCounterBytes) {
    cfg.splits = 0;
    cfg.cta_group = 1;
    cfg.grid = (int)std::min<long long>(dev.num_sms, (long long)bs_tiles(d, m, cfg.ntok));
  }
  return cfg;
}

// Workspace: header | the fixed stream-K counter region (8 counters per
// tile, when K is split) | partial tiles (2 per CTA, when K is split) |
// NVFP4 activation scales re-laid for the MMA.  Scratch always starts past
// the counter region, so no call's data lies where another call's counters
// do.
struct BsWsLayout {
  size_t counters, partials, sfb, total;
};
BsWsLayout bs_ws_layout(const hq_quant_desc& d, int m, const BsConfig& cfg) {
  BsWsLayout L{};
  L.counters = sizeof(WsHeader);
  size_t off = kWsScratchOff;
  L.partials = off;
  if (cfg.splits != 0) off += (size_t)cfg.grid * 2 * cfg.ntok * kBsTileN * sizeof(float);
  L.sfb = off;
  if (d.fmt == HQ_FMT_NVFP4) {
    const size_t halves = cfg.ntok > 128 ? 2 : 1;
    off += (size_t)((m + cfg.ntok - 1) / cfg.ntok) * (d.k / 256) * 4 * halves * 512;
  }
  L.total = (cfg.splits != 0 || d.fmt == HQ_FMT_NVFP4) ? off : sizeof(WsHeader);
  return L;
}

int bs_ring_depth(const hq_quant_desc& d, const BsConfig& cfg) {
  const bool nv = d.fmt == HQ_FMT_NVFP4;
  if (cfg.cta_group == 2)
    return cfg.ntok == 128 ? (nv ? BsCfg<kNV, 128, 2>::kStages : BsCfg<kMX, 128, 2>::kStages)
                           : (nv ? BsCfg<kNV, 256, 2>::kStages : BsCfg<kMX, 256, 2>::kStages);
  switch (cfg.ntok) {
    case 16: return nv ? BsCfg<kNV, 16>::kStages : BsCfg<kMX, 16>::kStages;
    case 32: return nv ? BsCfg<kNV, 32>::kStages : BsCfg<kMX, 32>::kStages;
    case 64: return nv ? BsCfg<kNV, 64>::kStages : BsCfg<kMX, 64>::kStages;
    case 128: return nv ? BsCfg<kNV, 128>::kStages : BsCfg<kMX, 128>::kStages;
    default: return nv ? BsCfg<kNV, 256>::kStages : BsCfg<kMX, 256>::kStages;
  }
}

size_t bs_workspace_bytes(const hq_quant_desc& d, int m, const BsConfig& cfg) {
  return bs_ws_layout(d, m, cfg).total;
}

hq_status bs_launch(const hq_quant_desc& d, const BsConfig& cfg, const void* packed, const void* a,
                    const void* a_sf, const float* a_scale, float a_global, int m, void* c, void* ws,
                    cudaStream_t stream) {
  const bool nv = d.fmt == HQ_FMT_NVFP4;
  const int n_tiles = (d.n + kBsTileN - 1) / kBsTileN;
  const int np = n_tiles * kBsTileN;
  const size_t codes_bytes = (size_t)np * d.k / 2;
  BsParams p{};
  p.sf_w = static_cast<const uint8_t*>(packed) + codes_bytes;
  p.c = static_cast<__nv_bfloat16*>(c);
  p.a_scale = a_scale;
  p.sf_groups = nv ? d.k / 64 : d.k / 128;
  p.g_w = reinterpret_cast<const float*>(p.sf_w + (size_t)n_tiles * p.sf_groups * 512);
  p.a_global = a_global;
  p.err = static_cast<uint32_t*>(ws);
  p.wait_ns = kDefaultWaitNs;
  p.m = m;
  p.n = d.n;
  p.k = d.k;
  p.n_tiles = n_tiles;
  p.k_boxes = (int)bs_k_boxes(d);
  p.k_stages = (int)bs_k_stages(d, cfg.ntok);
  const size_t tiles = (size_t)bs_tiles(d, m, cfg.ntok);
  p.total_iters = (long long)tiles * p.k_stages;
  p.m_tiles = (m + cfg.ntok - 1) / cfg.ntok;
  p.data_parallel = cfg.splits == 0 ? 1 : 0;
  p.early_weights = cfg.early_weights;
  p.stage_limit = cfg.stages;
  p.n_pairs = n_tiles / 2;
  // Whole-tile order: token-tile-major, except on CTA pairs when the packed
  // weights outgrow L2's comfortable share (> 48 MB, about 3/8 of it): then
  // groups of 16 pair tiles, so that a wave's clusters share 15 MB of weights
  // instead of streaming the whole matrix past the outputs' stores.
  // Measured on B200: NVFP4 M=16384 K=7168 N=18432 (66 MB) 900 -> 817 us;
  // at NVFP4 8192^3 (34 MB) and MXFP4 K=N=7168 groups of 4-16 were 0-5 %
  // slower than token-tile-major.
  p.raster = n_tiles;
  if (cfg.cta_group == 2) p.raster = codes_bytes > (size_t)48 << 20 ? std::min(16, p.n_pairs) : p.n_pairs;
  const BsWsLayout L = bs_ws_layout(d, m, cfg);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  p.counters = reinterpret_cast<int32_t*>(wsb + L.counters);
  p.partials = reinterpret_cast<float*>(wsb + L.partials);
  p.sf_a = wsb + L.sfb;

  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return HQ_ERR_CUDA;
  CUtensorMap mw{}, ma{};
  cuuint32_t estr[2] = {1, 1};
  // weights: codes [NP][K/2] bytes
  {
    cuuint64_t dims[2] = {nv ? (cuuint64_t)d.k / 2 : (cuuint64_t)d.k, (cuuint64_t)np};
    cuuint64_t strides[1] = {(cuuint64_t)d.k / 2};
    cuuint32_t box[2] = {128, (cuuint32_t)kBsTileN};
    CUresult cr = enc(&mw, nv ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2,
                      const_cast<void*>(packed), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return HQ_ERR_CUDA;
  }
  // activations: NVFP4 [M][K/2] bytes, MXFP4 E4M3 [M][K] bytes
  {
    const cuuint64_t row_bytes = nv ? (cuuint64_t)d.k / 2 : (cuuint64_t)d.k;
    cuuint64_t dims[2] = {row_bytes, (cuuint64_t)m};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {128, (cuuint32_t)(cfg.ntok / cfg.cta_group)};
    CUresult cr = enc(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return HQ_ERR_CUDA;
  }
  // NVFP4 activation scales: re-laid into the MMA's chunk order in the
  // workspace (a few MB at most), read by the kernel with bulk copies
  if (nv) {
    const int halves = cfg.ntok > 128 ? 2 : 1;
    const long long words = (long long)p.m_tiles * p.k_stages * 4 * halves * 128;
    const int blocks = (int)std::min<long long>((words + 255) / 256, 4LL * 148);
    sfb_relayout_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint32_t*>(a_sf), m, d.k / 64, cfg.ntok,
                                                     halves, p.k_stages, reinterpret_cast<uint32_t*>(wsb + L.sfb), words);
    if (cudaGetLastError() != cudaSuccess) return HQ_ERR_CUDA;
  }

  // CTA pairs: the scale chunks come by tensor copy (their completion is
  // counted on the other CTA's barrier), as rows of 128 32-bit words
  CUtensorMap msfa{}, msfb{};
  if (cfg.cta_group == 2) {
    {
      cuuint64_t dims[2] = {128, (cuuint64_t)n_tiles * p.sf_groups};
      cuuint64_t strides[1] = {512};
      cuuint32_t box[2] = {128, (cuuint32_t)(nv ? 4 : 1)};
      CUresult cr = enc(&msfa, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(p.sf_w), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (cr != CUDA_SUCCESS) return HQ_ERR_CUDA;
    }
    if (nv) {
      const int chunks = 4 * (cfg.ntok > 128 ? 2 : 1);   // 512-byte chunks per (token tile, stage)
      cuuint64_t dims[2] = {128, (cuuint64_t)p.m_tiles * p.k_stages * chunks};
      cuuint64_t strides[1] = {512};
      cuuint32_t box[2] = {128, (cuuint32_t)chunks};
      CUresult cr = enc(&msfb, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, wsb + L.sfb, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (cr != CUDA_SUCCESS) return HQ_ERR_CUDA;
    }
    if (cfg.ntok == 128)
      return nv ? bs_launch_t<kNV, 128, 2>(mw, ma, msfa, msfb, p, cfg.grid, stream)
                : bs_launch_t<kMX, 128, 2>(mw, ma, msfa, msfb, p, cfg.grid, stream);
    if (cfg.ntok == 256)
      return nv ? bs_launch_t<kNV, 256, 2>(mw, ma, msfa, msfb, p, cfg.grid, stream)
                : bs_launch_t<kMX, 256, 2>(mw, ma, msfa, msfb, p, cfg.grid, stream);
    return HQ_ERR_UNSUPPORTED;
  }

#define HQ_BS_CASE(F, NT) \
  case NT: return bs_launch_t<F, NT, 1>(mw, ma, msfa, msfb, p, cfg.grid, stream);
  if (nv) {
    switch (cfg.ntok) {
      HQ_BS_CASE(kNV, 16) HQ_BS_CASE(kNV, 32) HQ_BS_CASE(kNV, 64) HQ_BS_CASE(kNV, 128) HQ_BS_CASE(kNV, 256)
      default: return HQ_ERR_UNSUPPORTED;
    }
  }
  switch (cfg.ntok) {
    HQ_BS_CASE(kMX, 16) HQ_BS_CASE(kMX, 32) HQ_BS_CASE(kMX, 64) HQ_BS_CASE(kMX, 128) HQ_BS_CASE(kMX, 256)
    default: return HQ_ERR_UNSUPPORTED;
  }
#undef HQ_BS_CASE
}

}  // namespace hq
