// Dense and grouped (MoE) W4A16 GEMM for sm_100a with the INT4 dequantization
// fused into the kernel.
//
// Method: the weights are stored as 4-bit codes with a per-group fp16 scale
// and an optional uint4 zero point, described separately ("Humming:
// open-source kernel library for quantized inference", summary paragraph 2)
// and converted inside the kernel; the dense small-batch W4A16 case and the
// grouped MoE W4A16 case are the two rows of the comparison table on the
// Humming news page (section "one library, many formats").
//
// B200 design (this library's own):
//   * swap-AB: 128 weight rows form the MMA's M side and are the A operand,
//     read by tcgen05.mma straight from tensor memory (TMEM); the tokens are
//     the MMA's N side (16..256) and the B operand, staged by TMA into
//     shared memory with the 128-byte swizzle.  Dequantized weights never
//     touch shared memory.
//   * warp roles (16 warps): warp 0 issues the copies (one bulk copy of the
//     packed record, two TMA boxes of activations per 128-K stage), warp 1
//     issues the MMAs, warp 2 owns the TMEM allocation, warps 4-7 drain the
//     fp32 accumulators (epilogue), warps 8-15 unpack and rescale codes into
//     TMEM.  Stages are tied together by mbarriers; every wait is bounded.
//   * small M: split-K over CTAs; each split writes an fp32 partial and the
//     last split of a tile (found with one atomic counter, no spinning)
//     reduces all partials in split order, so results are bit-identical
//     from run to run.
//   * grouped mode: one launch covers every expert; the tile scheduler is
//     built on the device from the per-expert row offsets.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdio>

#include "hq_internal.h"
#include "ptx.cuh"

namespace hq {

namespace {

constexpr int kThreads = 512;
constexpr int kRecMax = 8576;        // packed record with zero points
constexpr int kMaxExperts = 1024;

struct W4Params {
  const uint8_t* packed;             // expert 0, record (0, 0)
  __nv_bfloat16* c;
  const int32_t* expert_offsets;     // grouped mode only
  float* partials;
  int32_t* counters;
  uint32_t* err;
  uint64_t expert_bytes;
  uint64_t wait_ns;
  int m;                             // dense: rows of A; grouped: total sorted rows
  int n;                             // output columns
  int n_tiles, k_blocks, m_tiles, splits;
  int num_experts;
  int has_zero;
  int rec_bytes;
  int grouped;
};

struct Unit {
  int expert;
  int nt;        // weight tile
  int row0;      // first row of A / C
  int rows;      // valid rows in this tile (<= NTOK)
  int kb0, kb1;  // k-block range
  int tile;      // dense tile index (split-K bookkeeping)
  int split;
};

template <int NTOK>
struct Smem {
  static constexpr int kATile = NTOK * 256;  // two 64-wide K boxes of NTOK rows x 128 B
};

__device__ __forceinline__ void raise_error(uint32_t* err, volatile int* abort_flag, uint32_t code) {
  atomicCAS(err, 0u, code);
  *abort_flag = 1;
}

template <int NTOK>
__device__ __forceinline__ bool decode_unit(const W4Params& p, const int* s_prefix, const int* s_off, int u,
                                            Unit& x) {
  if (!p.grouped) {
    int per_m = p.n_tiles * p.splits;
    int mt = u / per_m;
    int rem = u - mt * per_m;
    x.nt = rem / p.splits;
    x.split = rem - x.nt * p.splits;
    x.expert = 0;
    x.row0 = mt * NTOK;
    x.rows = min(NTOK, p.m - x.row0);
    x.kb0 = (int)((long long)x.split * p.k_blocks / p.splits);
    x.kb1 = (int)((long long)(x.split + 1) * p.k_blocks / p.splits);
    x.tile = mt * p.n_tiles + x.nt;
    return true;
  }
  // grouped: find the expert e with prefix[e] <= u < prefix[e+1]
  int lo = 0, hi = p.num_experts;  // invariant: prefix[lo] <= u < prefix[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (s_prefix[mid] <= u) lo = mid; else hi = mid;
  }
  int e = lo;
  int rows_e = s_off[e + 1] - s_off[e];
  int mtiles = (rows_e + NTOK - 1) / NTOK;
  int local = u - s_prefix[e];
  int mt = local % mtiles;
  x.nt = local / mtiles;
  x.expert = e;
  x.row0 = s_off[e] + mt * NTOK;
  x.rows = min(NTOK, s_off[e + 1] - x.row0);
  x.kb0 = 0;
  x.kb1 = p.k_blocks;
  x.tile = 0;
  x.split = 0;
  return true;
}

template <int NTOK, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    w4a16_kernel(const __grid_constant__ CUtensorMap tmap_a, const W4Params p) {
  constexpr int ACC_BUFS = (NTOK <= 128) ? 2 : 1;
  constexpr int kATile = Smem<NTOK>::kATile;
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, NTOK);
  static_assert(64 * STAGES + ACC_BUFS * NTOK <= 512, "TMEM budget");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                  // STAGES * kATile
  uint8_t* sR = smem + STAGES * kATile;                // STAGES * kRecMax
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + STAGES * kRecMax);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* aready = bars + 2 * STAGES;
  uint64_t* acc_full = bars + 3 * STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_total = const_cast<int*>(reinterpret_cast<volatile int*>(s_abort + 1));
  int* s_prefix = s_total + 1;                          // [kMaxExperts + 1]
  int* s_off = s_prefix + (kMaxExperts + 1);           // [kMaxExperts + 1]

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&aready[s], 8);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_a);
  if (warp == 2) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }

  // Unit count: dense is static; grouped builds per-expert tile prefix sums
  // from the device-resident row offsets.
  if (!p.grouped) {
    if (threadIdx.x == 0) *s_total = p.m_tiles * p.n_tiles * p.splits;
  } else {
    const int E = p.num_experts;
    for (int i = threadIdx.x; i <= E; i += kThreads) s_off[i] = p.expert_offsets[i];
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = *s_total;

  auto a_col = [](int s) -> uint32_t { return (uint32_t)(s * 64); };
  auto acc_col = [](int b) -> uint32_t { return (uint32_t)(64 * STAGES + b * NTOK); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        Unit x;
        decode_unit<NTOK>(p, s_prefix, s_off, u, x);
        const uint8_t* wbase = p.packed + (uint64_t)x.expert * p.expert_bytes +
                               (uint64_t)x.nt * p.k_blocks * p.rec_bytes;
        for (int kb = x.kb0; kb < x.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!hq_wait(&empty[s], ph ^ 1, p.wait_ns, s_abort)) {
            raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], (uint32_t)p.rec_bytes + kATile);
          bulk_g2s(sR + s * kRecMax, wbase + (uint64_t)kb * p.rec_bytes, (uint32_t)p.rec_bytes, &full[s], pol_w);
          tma_load_2d(sA + s * kATile, &tmap_a, kb * kBlockK, x.row0, &full[s]);
          tma_load_2d(sA + s * kATile + NTOK * 128, &tmap_a, kb * kBlockK + 64, x.row0, &full[s]);
        }
      }
      if (!ok) {
        // let every copy already issued land before the CTA exits
        uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j)
          hq_wait(&full[j % STAGES], (j / STAGES) & 1, p.wait_ns, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, uc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++uc) {
        Unit x;
        decode_unit<NTOK>(p, s_prefix, s_off, u, x);
        const int ab = uc % ACC_BUFS;
        const uint32_t aph = (uc / ACC_BUFS) & 1;
        if (!hq_wait(&acc_empty[ab], aph ^ 1, p.wait_ns, s_abort)) {
          raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc_col(ab);
        for (int kb = x.kb0; kb < x.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!hq_wait(&aready[s], ph, p.wait_ns, s_abort) || !hq_wait(&full[s], ph, p.wait_ns, s_abort)) {
            raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_base = smem_u32(sA + s * kATile);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint64_t bdesc = smem_desc_sw128(b_base + (j >> 2) * (NTOK * 128) + (j & 3) * 32);
            mma_bf16_ts(d_tmem, tmem_base + a_col(s) + j * 8, bdesc, kIdesc, (kb > x.kb0 || j > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&acc_full[ab]);
      }
      // make sure no MMA is still running when TMEM is released
      tc_commit(drain);
      hq_wait(drain, 0, p.wait_ns, nullptr);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = warp & 3;
    const int r = (int)(q * 32 + lane);  // weight row within the tile
    const uint32_t lane_addr = (q * 32) << 16;
    uint32_t uc = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++uc) {
      Unit x;
      decode_unit<NTOK>(p, s_prefix, s_off, u, x);
      const int ab = uc % ACC_BUFS;
      const uint32_t aph = (uc / ACC_BUFS) & 1;
      if (!hq_wait(&acc_full[ab], aph, p.wait_ns, s_abort)) {
        raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int n = x.nt * kTileN + r;
      const bool n_ok = n < p.n;
      const bool split = p.splits > 1;
      float* part = split ? p.partials + ((size_t)(x.tile * p.splits + x.split) * NTOK) * kTileN : nullptr;
#pragma unroll 1
      for (int j0 = 0; j0 < NTOK; j0 += 16) {
        uint32_t v[16];
        tmem_ld_x16(tmem_base + lane_addr + acc_col(ab) + j0, v);
        tmem_wait_ld();
        if (split) {
#pragma unroll
          for (int j = 0; j < 16; ++j) __stcg(part + (size_t)(j0 + j) * kTileN + r, __uint_as_float(v[j]));
        } else if (n_ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j0 + j < x.rows)
              p.c[(size_t)(x.row0 + j0 + j) * p.n + n] = __float2bfloat16_rn(__uint_as_float(v[j]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      if (split) {
        // Each epilogue warp owns 32 rows of the tile and its own counter:
        // the last split to finish those rows reduces every partial in
        // split order (deterministic; nobody waits on anybody).
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = (atomicAdd(p.counters + x.tile * 4 + q, 1) == p.splits - 1);
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          const float* base = p.partials + (size_t)x.tile * p.splits * NTOK * kTileN;
          for (int j = 0; j < x.rows; ++j) {
            float acc = 0.f;
            for (int sp = 0; sp < p.splits; ++sp) acc += __ldcg(base + ((size_t)sp * NTOK + j) * kTileN + r);
            if (n_ok) p.c[(size_t)(x.row0 + j) * p.n + n] = __float2bfloat16_rn(acc);
          }
          if (lane == 0) p.counters[x.tile * 4 + q] = 0;  // leave the workspace zeroed
        }
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dequantize into TMEM
    const uint32_t q = warp & 3;
    const int half = (int)(warp - 8) >> 2;  // chunks {2*half, 2*half+1} of each 128-K block
    const int r = (int)(q * 32 + lane);
    const uint32_t lane_addr = (q * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      Unit x;
      decode_unit<NTOK>(p, s_prefix, s_off, u, x);
      for (int kb = x.kb0; kb < x.kb1; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        // the TMEM stage s is free once empty[s] completed for the previous
        // round, which the producer already waited on before refilling s
        if (!hq_wait(&full[s], ph, p.wait_ns, s_abort)) {
          raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* rec = sR + s * kRecMax;
        const __half sc = reinterpret_cast<const __half*>(rec + kW4RecCodes)[r];
        const uint32_t z = p.has_zero ? rec[kW4RecCodes + 256 + r] : 8u;
        const __nv_bfloat16 sb = __float2bfloat16_rn(__half2float(sc));
        const uint32_t sbits = (uint32_t)__bfloat16_as_ushort(sb);
        const uint32_t s2 = sbits | (sbits << 16);
        const __nv_bfloat16 zb = __float2bfloat16_rn((float)(128 + z));
        const uint32_t zbits = (uint32_t)__bfloat16_as_ushort(zb);
        const uint32_t z2 = zbits | (zbits << 16);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = half * 2 + cc;
          const uint4 raw = *reinterpret_cast<const uint4*>(rec + (c * 128 + r) * 16);
          const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t out[16];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t x2 = lop3_and_or(wv[w] >> (4 * j), 0x000F000Fu, 0x43004300u);  // 128 + q
              out[w * 4 + j] = bf16x2_mul(bf16x2_sub(x2, z2), s2);
            }
          }
          tmem_st_x16(tmem_base + lane_addr + a_col(s) + c * 16, out);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&aready[s]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, 512);
}

template <int NTOK, int STAGES>
size_t smem_bytes() {
  return (size_t)STAGES * (Smem<NTOK>::kATile + kRecMax) + 1024 /*align*/ + 256 /*barriers*/ +
         2 * (kMaxExperts + 1) * sizeof(int) + 64;
}

template <int NTOK, int STAGES>
hq_status launch_t(const CUtensorMap& map, const W4Params& p, int grid, cudaStream_t stream) {
  auto kern = w4a16_kernel<NTOK, STAGES>;
  const size_t smem = smem_bytes<NTOK, STAGES>();
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return HQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  kern<<<grid, kThreads, smem, stream>>>(map, p);
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

}  // namespace

int w4_stages_for(int ntok) {
  switch (ntok) {
    case 16: return 7;
    case 32: return 7;
    case 64: return 6;
    case 128: return 4;
    default: return 3;
  }
}

W4Config w4_plan(const DeviceInfo& dev, const hq_quant_desc& d, int m, bool grouped, const hq_tuning* t) {
  W4Config cfg{};
  const int n_tiles = (d.n + kTileN - 1) / kTileN;
  const int k_blocks = d.k / kBlockK;
  int ntok = (t && t->tile_m) ? t->tile_m : 0;
  if (!ntok) {
    if (grouped) {
      // average rows per expert decides the token tile
      long long avg = (long long)m / std::max(1, d.num_experts);
      ntok = avg <= 16 ? 16 : avg <= 32 ? 32 : avg <= 64 ? 64 : 128;
    } else {
      ntok = m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : m <= 128 ? 128 : 256;
    }
  }
  cfg.ntok = ntok;
  cfg.stages = w4_stages_for(ntok);
  if (t && t->stages) cfg.stages = t->stages;
  if (grouped) {
    cfg.splits = 1;
    cfg.grid = dev.num_sms;
    return cfg;
  }
  const int m_tiles = (m + ntok - 1) / ntok;
  const long long tiles = (long long)m_tiles * n_tiles;
  int splits = 1;
  if (t && t->split_k) {
    splits = t->split_k;
  } else if (tiles < dev.num_sms) {
    splits = (int)(dev.num_sms / tiles);
    splits = std::max(1, std::min(splits, k_blocks / 4));
  }
  splits = std::max(1, std::min(splits, k_blocks));
  cfg.splits = splits;
  long long units = tiles * splits;
  cfg.grid = (int)std::min<long long>(units, dev.num_sms);
  return cfg;
}

size_t w4_workspace_bytes(const hq_quant_desc& d, int m, const W4Config& cfg, bool grouped) {
  size_t bytes = sizeof(WsHeader);
  if (grouped || cfg.splits <= 1) return bytes;
  const int n_tiles = (d.n + kTileN - 1) / kTileN;
  const int m_tiles = (m + cfg.ntok - 1) / cfg.ntok;
  const size_t tiles = (size_t)n_tiles * m_tiles;
  bytes += ((4 * tiles * sizeof(int32_t) + 255) / 256) * 256;           // counters, 4 per tile
  bytes += tiles * (size_t)cfg.splits * cfg.ntok * kTileN * sizeof(float);  // partials
  return bytes;
}

hq_status w4_launch(const hq_quant_desc& d, const W4Config& cfg, const void* packed, const void* a, int m,
                    void* c, const int32_t* expert_offsets, void* ws, cudaStream_t stream) {
  const bool grouped = expert_offsets != nullptr;
  W4Params p{};
  p.packed = static_cast<const uint8_t*>(packed);
  p.c = static_cast<__nv_bfloat16*>(c);
  p.expert_offsets = expert_offsets;
  p.err = static_cast<uint32_t*>(ws);
  p.has_zero = d.has_zero_point ? 1 : 0;
  p.rec_bytes = w4_record_bytes(p.has_zero);
  p.n_tiles = (d.n + kTileN - 1) / kTileN;
  p.k_blocks = d.k / kBlockK;
  p.expert_bytes = (uint64_t)p.n_tiles * p.k_blocks * p.rec_bytes;
  p.m = m;
  p.n = d.n;
  p.m_tiles = (m + cfg.ntok - 1) / cfg.ntok;
  p.splits = cfg.splits;
  p.num_experts = grouped ? d.num_experts : 1;
  p.grouped = grouped ? 1 : 0;
  p.wait_ns = kDefaultWaitNs;
  if (!grouped && cfg.splits > 1) {
    const size_t tiles = (size_t)p.n_tiles * p.m_tiles;
    uint8_t* base = static_cast<uint8_t*>(ws) + sizeof(WsHeader);
    p.counters = reinterpret_cast<int32_t*>(base);
    p.partials = reinterpret_cast<float*>(base + ((4 * tiles * sizeof(int32_t) + 255) / 256) * 256);
  }

  // Activations: bf16 [rows][K], boxes of 64 K x NTOK rows, 128-byte swizzle.
  CUtensorMap map;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return HQ_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)d.k, (cuuint64_t)m};
  cuuint64_t strides[1] = {(cuuint64_t)d.k * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)cfg.ntok};
  cuuint32_t estr[2] = {1, 1};
  CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return HQ_ERR_CUDA;

  const int grid = cfg.grid;
  switch (cfg.ntok) {
    case 16: return cfg.stages == 7 ? launch_t<16, 7>(map, p, grid, stream) : HQ_ERR_UNSUPPORTED;
    case 32: return cfg.stages == 7 ? launch_t<32, 7>(map, p, grid, stream) : HQ_ERR_UNSUPPORTED;
    case 64: return cfg.stages == 6 ? launch_t<64, 6>(map, p, grid, stream) : HQ_ERR_UNSUPPORTED;
    case 128: return cfg.stages == 4 ? launch_t<128, 4>(map, p, grid, stream) : HQ_ERR_UNSUPPORTED;
    case 256: return cfg.stages == 3 ? launch_t<256, 3>(map, p, grid, stream) : HQ_ERR_UNSUPPORTED;
    default: return HQ_ERR_UNSUPPORTED;
  }
}

}  // namespace hq
