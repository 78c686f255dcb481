// W4A16 GEMM for 1 to 16 tokens with the weights dequantized straight into
// tensor-core register fragments: the HBM-bound end of the token range.
//
// Method: weights are 4-bit codes q with a per-group fp16 scale s and an
// optional uint4 zero point z, w = (q - z) * s ("Humming: open-source kernel
// library for quantized inference", summary paragraph 2), converted inside
// the kernel (same page, paragraph 3).  As in the exact-weight kernel the
// sum over one 128-K group factors as s * sum_k (q_k - z) a_k: the tensor
// core multiplies the exact integers (q - z) (bf16 holds -15..15 exactly)
// and s is applied to each group's fp32 sum.
//
// B200 design.  At M <= 16 the launch streams K*N/2 bytes of codes and does
// almost no arithmetic per byte, so what matters is keeping enough bytes in
// flight on every SM with as few instructions per byte as possible.  The
// TMEM path (a TMA stage -> unpacking warps -> tcgen05.st -> an MMA warp ->
// scale warps) pays a chain of mbarrier handshakes per stage; here every warp
// is its own pipeline with no handshake on the weight path:
//   * each warp owns 32 weight rows (two 16-row MMA tiles) of a 128-row tile
//     and a K range, and keeps kP records (128 K each) of its codes in flight
//     in registers, loaded with plain coalesced global loads (a warp's load
//     covers whole 128-byte lines of the packed record);
//   * codes become bf16 (q - z) in registers and feed mma.sync m16n8k16
//     directly (weights as the 16-row A side, tokens as the 8-wide B side,
//     one or two 8-token tiles); each group's fp32 result is scaled into a
//     running fp32 sum;
//   * activations, shared by the CTA's four warps, are staged by TMA (128-byte
//     swizzle) in a small shared-memory ring, one mbarrier pair per stage of
//     kP records.  Lanes 8 bytes apart in K would meet in one bank; lanes of
//     the upper half of a quad read their four 16-byte pieces in an order
//     rotated by two, and load their code words in the same rotated order,
//     which makes every activation load conflict-free;
//   * the K range of a tile is split over a few CTAs so that the grid fills
//     the SMs in one wave; each CTA writes an fp32 partial tile, and the last
//     of a tile's CTAs (a counter per tile) adds the partials in slice order
//     and writes the bf16 output, so results repeat bit for bit.
// mma.sync is the older tensor-core path (on B200 a 16x8x16 MMA issues about
// every 2.7 SM cycles, near 0.44 PFLOP/s for the GPU); at 1-8 tokens the MMAs
// are a small share of the time (the bound is the codes' HBM traffic), at
// 9-16 tokens they start to show.  Measured on B200 (per launch, back to back,
// M <= 8): warps matter more than loads in flight per warp: two records in
// flight per warp with four CTAs (16 warps) per SM beat four records with
// three CTAs (22.4 against 24.5 us at K=7168 N=18432) and six with two
// (30.1); staging the codes through shared memory with cp.async (three to
// four records per warp) took 25.6-25.9 us, bulk L2 prefetches of each CTA's
// whole K slice 25.4, code loads that skip L1 no change, and the in-order
// activation reads (a 2-way bank conflict, one 16-byte code load) 2 % more.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "hq_internal.h"
#include "ptx.cuh"
#include "w4a16_common.cuh"

namespace hq {
namespace w4 {

namespace {

template <int NT8, int TW_>
struct RegCfg {
  static constexpr int kTw = TW_;               // 16-row MMA tiles per warp (1 or 2)
  static constexpr int kWarps = 8 / kTw;        // 128 weight rows per CTA
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kP = 2;                 // records per activation stage = records in flight per warp
  static constexpr int kD = kRegRing;          // activation ring depth (stages)
  static constexpr int kRows = 8 * NT8;        // tokens in the activation box
  static constexpr int kBox = kRows * 128;     // one 64-K box: kRows rows of 128 bytes
  static constexpr int kRecA = 2 * kBox;       // one record's activations
  static constexpr int kStage = kP * kRecA;
  static constexpr int kBarOff = kD * kStage;
  static constexpr int kSmem = kBarOff + 2 * kD * 8 + 16 + 1024;  // + 1 KiB for the 1024-byte alignment
  static constexpr int kNv4 = kTw * NT8;       // float4s per thread in a partial tile
  static constexpr int kCtasPerSm = reg_ctas_per_sm(TW_);
  static_assert(kBox % 1024 == 0, "a 128-byte-swizzled box starts on a 1024-byte boundary");
  static_assert(kCtasPerSm * (kSmem + 1024) <= 228 * 1024, "kCtasPerSm CTAs fit one SM's shared memory");
};

struct RegParams {
  const uint8_t* packed;   // record (0, 0)
  __nv_bfloat16* c;        // [m][n]
  float* partials;         // [grid][kNv4][kThreads] float4
  int32_t* counters;       // 4 per weight tile, the first used
  uint32_t* err;
  uint64_t wait_ns;
  int m, n;
  int k_blocks;
  int rec_bytes;
  int splits;              // CTAs per weight tile (K slices)
  int early_weights;       // load the first records' codes before the previous kernel has completed
};

__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_nc_u16(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_nc_u8(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Codes of the pair at nibble j of a word (elements k, k+1 at bits 4j and
// 16 + 4j) to the exact bf16 pair (q_k - z, q_{k+1} - z): the 0x4300 exponent
// makes bf16(128 + q), and z2 holds bf16(128 + z) twice.
__device__ __forceinline__ uint32_t code_pair(uint32_t w, int j, uint32_t z2) {
  return bf16x2_sub(lop3_and_or(w >> (4 * j), 0x000F000Fu, 0x43004300u), z2);
}

// Warp w of the CTA owns rows 16 TW w .. 16 TW (w + 1) - 1 of the 128-row
// weight tile (TW = 1 or 2): MMA tile T row g (lane / 4) is weight
// row 16 TW w + 16T + g, row g + 8 is 16 TW w + 16T + 8 + g.  Lane quad
// position qd (lane % 4) holds the 32-K chunk qd of each record for those rows.
template <int NT8, bool HASZ, int TWT>
__global__ void __launch_bounds__(RegCfg<NT8, TWT>::kThreads, RegCfg<NT8, TWT>::kCtasPerSm)
    w4a16_reg_kernel(const __grid_constant__ CUtensorMap tmap_a, const RegParams p) {
  using C = RegCfg<NT8, TWT>;
  constexpr int P = C::kP;
  constexpr int D = C::kD;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + D;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + D);
  int* s_last = const_cast<int*>(s_abort + 1);

  const int warp = (int)(threadIdx.x >> 5), lane = (int)(threadIdx.x & 31);
  const int g = lane >> 2, qd = lane & 3;
  const int tile = (int)blockIdx.x / p.splits, slice = (int)blockIdx.x - tile * p.splits;
  const int kb0 = (int)((long long)slice * p.k_blocks / p.splits);
  const int kb1 = (int)((long long)(slice + 1) * p.k_blocks / p.splits);
  const int nrec = kb1 - kb0;
  const int nstage = (nrec + P - 1) / P;

  if (threadIdx.x == 0) {
    for (int i = 0; i < D; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::kWarps);
    }
    *s_abort = 0;
    fence_mbar_init();
    pdl_launch_dependents();
    prefetch_tensormap(&tmap_a);
  }

  // ---- this thread's places in a record
  // codes of (T, h): row rw = 32 warp + 16 T + 8 h + g, chunk qd, at byte
  // (qd * 128 + rw) * 16; the upper half of a quad takes the chunk's two
  // 8-byte halves in swapped order (word slot i holds word (i + 2 (qd >> 1)) % 4)
  const int rot = (qd >> 1) * 8;
  constexpr int TW = C::kTw;
  int coff[TW][2], row[TW][2];
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      row[T][h] = 16 * TW * warp + 16 * T + 8 * h + g;
      coff[T][h] = (qd * 128 + row[T][h]) * 16;
    }
  const uint8_t* rec0 = p.packed + ((size_t)tile * p.k_blocks + kb0) * (size_t)p.rec_bytes;

  uint32_t wv[P][TW][2][4];  // [record slot][T][h][word slot]
  uint32_t sc[P][TW][2];     // fp16 scale bits of row (T, h)
  uint32_t zp[P][TW][2];     // zero point of row (T, h) (HASZ)
  auto load_rec = [&](int u, int r) {
    if (r < nrec) {
      const uint8_t* rec = rec0 + (size_t)r * p.rec_bytes;
#pragma unroll
      for (int T = 0; T < TW; ++T)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint2 lo = ldg_nc_v2(rec + coff[T][h] + rot);
          const uint2 hi = ldg_nc_v2(rec + coff[T][h] + (8 - rot));
          wv[u][T][h][0] = lo.x;
          wv[u][T][h][1] = lo.y;
          wv[u][T][h][2] = hi.x;
          wv[u][T][h][3] = hi.y;
          sc[u][T][h] = ldg_nc_u16(rec + kW4RecCodes + 2 * row[T][h]);
          if (HASZ) zp[u][T][h] = ldg_nc_u8(rec + kW4RecCodes + 256 + row[T][h]);
        }
    }
  };

  // Phase 1: the first records' codes (no kernel on the stream writes them)
  // before the previous kernel has completed, unless the caller said otherwise.
  if (p.early_weights) {
#pragma unroll
    for (int u = 0; u < P; ++u) load_rec(u, u);
  }
  __syncthreads();  // barriers initialised
  pdl_wait();       // activations, outputs, partials and counters may be in use until here
  if (!p.early_weights) {
#pragma unroll
    for (int u = 0; u < P; ++u) load_rec(u, u);
  }

  auto issue_stage = [&](int x) {  // one thread
    const int r0 = x * P;
    const int nr = min(P, nrec - r0);
    uint64_t* fb = &full[x % D];
    mbar_arrive_expect_tx(fb, (uint32_t)(nr * C::kRecA));
    uint8_t* dst = smem + (x % D) * C::kStage;
    for (int u = 0; u < nr; ++u) {
      const int kx = (kb0 + r0 + u) * kBlockK;
      tma_load_2d(dst + u * C::kRecA, &tmap_a, kx, 0, fb);
      tma_load_2d(dst + u * C::kRecA + C::kBox, &tmap_a, kx + 64, 0, fb);
    }
  };
  int issued = 0;
  if (warp == 0) {
    if (lane == 0 && nstage > 0) issue_stage(0);
    issued = nstage > 0 ? 1 : 0;
  }

  // activation addresses: token row g + 8t of box (qd >> 1); the 16-byte
  // piece of word slot i is piece 4 (qd & 1) + ((i + 2 (qd >> 1)) & 3) of the
  // row, stored at piece index ^ (row & 7) by the 128-byte swizzle
  const uint32_t sbase = smem_u32(smem);
  uint32_t aoff[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int piece = 4 * (qd & 1) + ((i + 2 * (qd >> 1)) & 3);
    aoff[i] = (uint32_t)((qd >> 1) * C::kBox + g * 128 + ((piece ^ g) << 4));
  }

  float acc[TW][NT8][4];
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int t = 0; t < NT8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[T][t][e] = 0.f;

  bool ok = true;
  for (int j = 0; j < nstage; ++j) {
    // the producer refills the slot of stage j + 1, freed at the end of stage j + 1 - D
    if (warp == 0 && j + 1 < nstage) {
      const int x = j + 1;
      if (x >= D && !hq_wait_warp(&empty[x % D], ((x / D) - 1) & 1, p.wait_ns, s_abort)) {
        if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      if (lane == 0) issue_stage(x);
      __syncwarp();
      issued = x + 1;
    }
    if (!hq_wait_warp(&full[j % D], (j / D) & 1, p.wait_ns, s_abort)) {
      if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
      ok = false;
      break;
    }
    const uint32_t sa = sbase + (uint32_t)((j % D) * C::kStage);
#pragma unroll
    for (int u = 0; u < P; ++u) {
      const int r = j * P + u;
      if (r < nrec) {
        uint32_t z2[TW][2];
#pragma unroll
        for (int T = 0; T < TW; ++T)
#pragma unroll
          for (int h = 0; h < 2; ++h) z2[T][h] = HASZ ? (0x43004300u | zp[u][T][h] | (zp[u][T][h] << 16)) : 0x43084308u;
        float d[TW][NT8][4];
#pragma unroll
        for (int T = 0; T < TW; ++T)
#pragma unroll
          for (int t = 0; t < NT8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) d[T][t][e] = 0.f;
        const uint32_t ra = sa + (uint32_t)(u * C::kRecA);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 b[NT8];
#pragma unroll
          for (int t = 0; t < NT8; ++t) b[t] = lds128(ra + aoff[i] + t * 8 * 128);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int T = 0; T < TW; ++T) {
              const uint32_t a0 = code_pair(wv[u][T][0][i], 2 * hh, z2[T][0]);
              const uint32_t a1 = code_pair(wv[u][T][1][i], 2 * hh, z2[T][1]);
              const uint32_t a2 = code_pair(wv[u][T][0][i], 2 * hh + 1, z2[T][0]);
              const uint32_t a3 = code_pair(wv[u][T][1][i], 2 * hh + 1, z2[T][1]);
#pragma unroll
              for (int t = 0; t < NT8; ++t)
                mma_16816(d[T][t], a0, a1, a2, a3, hh ? b[t].z : b[t].x, hh ? b[t].w : b[t].y);
            }
          }
        }
#pragma unroll
        for (int T = 0; T < TW; ++T) {
          const float s0 = __half2float(__ushort_as_half((unsigned short)sc[u][T][0]));
          const float s1 = __half2float(__ushort_as_half((unsigned short)sc[u][T][1]));
#pragma unroll
          for (int t = 0; t < NT8; ++t) {
            acc[T][t][0] = fmaf(s0, d[T][t][0], acc[T][t][0]);
            acc[T][t][1] = fmaf(s0, d[T][t][1], acc[T][t][1]);
            acc[T][t][2] = fmaf(s1, d[T][t][2], acc[T][t][2]);
            acc[T][t][3] = fmaf(s1, d[T][t][3], acc[T][t][3]);
          }
        }
      }
      load_rec(u, r + P);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[j % D]);
  }
  if (!ok && lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
  if (warp == 0 && lane == 0 && *s_abort) {
    // let every copy already issued land before the CTA exits
    for (int x = issued > D ? issued - D : 0; x < issued; ++x) hq_wait(&full[x % D], (x / D) & 1, p.wait_ns, nullptr);
  }

  // ---- output: feature tile * 128 + row, token 8t + 2 qd + e
  auto store = [&](float (&v)[TW][NT8][4]) {
#pragma unroll
    for (int T = 0; T < TW; ++T)
#pragma unroll
      for (int t = 0; t < NT8; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int f = tile * kTileN + row[T][e >> 1];
          const int tok = 8 * t + 2 * qd + (e & 1);
          if (f < p.n && tok < p.m) p.c[(size_t)tok * p.n + f] = __float2bfloat16_rn(v[T][t][e]);
        }
  };
  if (p.splits == 1) {
    store(acc);
    return;
  }
  // K split over p.splits CTAs: fp32 partial tile, the last CTA of the tile
  // sums the partials in slice order
  float4* mine = reinterpret_cast<float4*>(p.partials) + (size_t)blockIdx.x * C::kNv4 * C::kThreads + threadIdx.x;
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int t = 0; t < NT8; ++t)
      __stcg(mine + (T * NT8 + t) * C::kThreads, make_float4(acc[T][t][0], acc[T][t][1], acc[T][t][2], acc[T][t][3]));
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(&p.counters[4 * tile], 1);
    *s_last = prev == p.splits - 1 ? 1 : 0;
  }
  __syncthreads();
  if (!*s_last) return;
  __threadfence();
  float sum[TW][NT8][4];
  const float4* first = reinterpret_cast<const float4*>(p.partials) +
                        (size_t)tile * p.splits * C::kNv4 * C::kThreads + threadIdx.x;
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      float4 s4 = __ldcg(first + (T * NT8 + t) * C::kThreads);
      for (int sl = 1; sl < p.splits; ++sl) {
        const float4 v = __ldcg(first + ((size_t)sl * C::kNv4 + T * NT8 + t) * C::kThreads);
        s4.x += v.x;
        s4.y += v.y;
        s4.z += v.z;
        s4.w += v.w;
      }
      sum[T][t][0] = s4.x;
      sum[T][t][1] = s4.y;
      sum[T][t][2] = s4.z;
      sum[T][t][3] = s4.w;
    }
  if (threadIdx.x == 0) p.counters[4 * tile] = 0;  // back to zero for the next call
  store(sum);
}

template <int NT8, bool HASZ, int TWT>
hq_status reg_launch_t(const CUtensorMap& map, const RegParams& p, int grid, cudaStream_t stream) {
  auto kern = w4a16_reg_kernel<NT8, HASZ, TWT>;
  const size_t smem = RegCfg<NT8, TWT>::kSmem;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return HQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  return launch_pdl(kern, dim3(grid), dim3(RegCfg<NT8, TWT>::kThreads), smem, stream, map, p) == cudaSuccess
             ? HQ_OK
             : HQ_ERR_CUDA;
}

}  // namespace
}  // namespace w4

using w4::RegParams;

// CTAs per weight tile (K slices) of the register-path plan: the split that
// fills the SMs best in one wave of reg_ctas_per_sm(2) CTAs per SM (a tie
// goes to more CTAs: more bytes in flight).
int reg_splits(int num_sms, const hq_quant_desc& d) {
  const long long tiles = (d.n + kTileN - 1) / kTileN;
  const long long kbs = d.k / kBlockK;
  const long long slots = (long long)num_sms * reg_ctas_per_sm(2);
  int best = 1;
  double best_eff = -1.0;
  for (long long s = 1; s <= kbs && tiles * s <= slots; ++s) {
    const long long units = tiles * s;
    const long long waves = (units + num_sms - 1) / num_sms;
    const double eff = (double)units / (double)(waves * num_sms);
    if (eff >= best_eff - 1e-9) {
      best_eff = eff;
      best = (int)s;
    }
  }
  return best;
}

size_t reg_workspace_bytes(const W4Config& cfg) {
  if (cfg.splits <= 1) return sizeof(WsHeader);
  return sizeof(WsHeader) + kWsCounterBytes + (size_t)cfg.grid * 128 * 16 * sizeof(float);
}

hq_status reg_launch(const hq_quant_desc& d, const W4Config& cfg, const void* packed, const void* a, int m, void* c,
                     void* ws, cudaStream_t stream) {
  if (d.fmt != HQ_FMT_INT4 || m > 16 || m < 1) return HQ_ERR_UNSUPPORTED;
  RegParams p{};
  p.packed = static_cast<const uint8_t*>(packed);
  p.c = static_cast<__nv_bfloat16*>(c);
  p.err = static_cast<uint32_t*>(ws);
  uint8_t* base = static_cast<uint8_t*>(ws) + sizeof(WsHeader);
  p.counters = reinterpret_cast<int32_t*>(base);
  p.partials = reinterpret_cast<float*>(base + kWsCounterBytes);
  p.wait_ns = kDefaultWaitNs;
  p.m = m;
  p.n = d.n;
  p.k_blocks = d.k / kBlockK;
  p.rec_bytes = w4_record_bytes(d.has_zero_point != 0);
  p.splits = cfg.splits < 1 ? 1 : cfg.splits;
  p.early_weights = cfg.early_weights;
  const int n_tiles = (d.n + kTileN - 1) / kTileN;
  if (cfg.grid != n_tiles * p.splits) return HQ_ERR_INVALID_ARG;
  const int nt8 = m <= 8 ? 1 : 2;

  // Activations: bf16 [m][K], boxes of 64 K x (8 or 16) rows, 128-byte
  // swizzle; rows past m read as zeros.
  CUtensorMap map;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return HQ_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)d.k, (cuuint64_t)m};
  cuuint64_t strides[1] = {(cuuint64_t)d.k * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)(8 * nt8)};
  cuuint32_t estr[2] = {1, 1};
  CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return HQ_ERR_CUDA;
  const bool hz = d.has_zero_point != 0;
  // grids of fewer CTAs than SMs: eight warps of 16 rows per CTA (more warps
  // on each busy SM); else four warps of 32 rows at four CTAs per SM
  if (cfg.reg_tw == 1) {
    if (nt8 == 1)
      return hz ? w4::reg_launch_t<1, true, 1>(map, p, cfg.grid, stream) : w4::reg_launch_t<1, false, 1>(map, p, cfg.grid, stream);
    return hz ? w4::reg_launch_t<2, true, 1>(map, p, cfg.grid, stream) : w4::reg_launch_t<2, false, 1>(map, p, cfg.grid, stream);
  }
  if (nt8 == 1)
    return hz ? w4::reg_launch_t<1, true, 2>(map, p, cfg.grid, stream) : w4::reg_launch_t<1, false, 2>(map, p, cfg.grid, stream);
  return hz ? w4::reg_launch_t<2, true, 2>(map, p, cfg.grid, stream) : w4::reg_launch_t<2, false, 2>(map, p, cfg.grid, stream);
}

}  // namespace hq
