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
// little arithmetic per byte, so what matters is keeping enough bytes in
// flight on every SM and few instructions per byte.  The TMEM path (a TMA
// stage -> unpacking warps -> tcgen05.st -> an MMA warp -> scale warps) pays
// a chain of mbarrier handshakes per stage; here the warps that convert the
// codes also issue the MMAs, from registers:
//   * each CTA owns one 128-row weight tile and a K slice; one thread copies
//     whole records (codes, scales, zero points: one bulk copy per stage) and
//     their activation boxes (TMA, 128-byte swizzle) into a small ring of
//     shared-memory stages, one full and one empty mbarrier per stage;
//   * each warp owns 32 rows (two 16-row MMA tiles; 16 rows for grids below
//     one CTA per SM), reads its codes with ldmatrix (conflict-free, see
//     below), turns them into the exact bf16 (q - z) in registers and feeds
//     mma.sync m16n8k16 (weights = the 16-row A side, tokens = one or two
//     8-wide B tiles); each group's fp32 result is scaled into a running
//     fp32 sum;
//   * the K range of a tile is split over a few CTAs so that the grid fills
//     the SMs; each CTA writes an fp32 partial tile, and the last of a tile's
//     CTAs (a counter per tile) adds the partials in slice order and writes
//     the bf16 output, so results repeat bit for bit;
//   * grouped MoE (experts of a few tokens): persistent CTAs walk (expert,
//     weight tile, token tile) units over the whole K range, the ring
//     streaming across units (w4a16_reg_grouped_kernel, below).
// mma.sync is the older tensor-core path (on B200 a 16x8x16 MMA issues about
// every 2.7 SM cycles, near 0.44 PFLOP/s for the GPU); at 1-8 tokens the MMAs
// are a small share of the time, at 9-16 they start to show.  Measured on
// B200 (per launch, back to back, M <= 8, K=7168 N=18432): this layout 20.8
// us; codes loaded by each warp straight from global memory into registers
// (two records in flight per warp, no shared-memory hop) 22.4 us at best
// (four records at three CTAs per SM 24.5, six at two 30.1); the same through
// a per-warp cp.async ring 25.6-25.9; bulk L2 prefetches of each CTA's slice
// 25.4.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "hq_internal.h"
#include "ptx.cuh"
#include "w4a16_common.cuh"

namespace hq {
namespace w4 {

namespace {


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
  int splits;              // CTAs per weight tile (K slices); grouped: 1
  int early_weights;       // load the first records' codes before the previous kernel has completed
  // grouped MoE: experts back to back in the blob, rows of A / C sorted by expert
  const int32_t* expert_offsets;
  uint64_t expert_bytes;
  int num_experts;
  int n_tiles;
};

// One grouped unit: weight tile nt of one expert over the whole K range, for
// token rows [row0, row0 + rows) of A.
struct RegUnit {
  const uint8_t* rec0;
  int row0, rows, nt;
};

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
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

// Whole records reach shared memory by one bulk copy per stage (long
// contiguous reads, no registers held for loads in flight); each warp reads
// its codes back with ldmatrix.  In the packed record, the
// 16-byte chunk c of rows r .. r+7 is one 128-byte run, so an 8x8 b16
// "matrix" of ldmatrix is chunk c of 8 consecutive rows, and lane (g, qd)
// receives word qd of row g's chunk: exactly the quad distribution of the MMA
// fragment, with no bank conflict.  Word qd of chunk c holds K = 32c + 8qd ..
// +7, so lane (g, qd) reads activations K = 32c + 8qd .. +7 of its token; the
// token of MMA column n is sigma(n) = (n >> 1) | ((n & 1) << 2), which puts
// the two tokens of every 8-lane phase 4 rows apart under the 128-byte swizzle
// and makes those reads conflict-free too.
template <int NT8, int TW_>
struct RegCfg {
  static constexpr int kTw = TW_;
  static constexpr int kWarps = 8 / kTw;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kP = NT8 == 2 ? 1 : 2;          // records per stage
  static constexpr int kD = NT8 == 2 ? kRegRing16 : kRegRing8;   // stages
  static constexpr int kRows = 8 * NT8;
  static constexpr int kBox = kRows * 128;
  static constexpr int kRecA = 2 * kBox;
  static constexpr int kWBytes = (kP * kRecMax + 1023) / 1024 * 1024;   // codes, scales, zero points
  static constexpr int kStage = kWBytes + kP * kRecA;
  static constexpr int kBarOff = kD * kStage;
  static constexpr int kSmem = kBarOff + 2 * kD * 8 + 16 + 1024;
  static constexpr int kNv4 = kTw * NT8;
  static constexpr int kCtasPerSm = 3;
  static_assert(kBox % 1024 == 0 && kWBytes % 1024 == 0 && kStage % 1024 == 0, "1024-byte aligned boxes");
  static_assert(kCtasPerSm * (kSmem + 1024) <= 228 * 1024, "kCtasPerSm CTAs fit one SM's shared memory");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ int col_token(int n) { return (n >> 1) | ((n & 1) << 2); }

// One 128-K record of a warp's rows: codes (ldmatrix from the record at
// `wrec`), scales and zero points from shared memory, activations from the
// record's boxes at `ra`; the group's fp32 sum scaled into acc.
template <int NT8, bool HASZ, int TW>
__device__ __forceinline__ void reg_record(uint32_t wrec, uint32_t ra, uint32_t lds_row, const uint32_t (&aoff)[4],
                                           const int (&row)[TW][2], float (&acc)[TW][NT8][4]) {
  uint32_t w[TW][2][4];   // word qd of chunk c of row (T, h)
  if (TW == 2) {
#pragma unroll
    for (int c = 0; c < 4; ++c) ldsm_x4(wrec + lds_row + c * 2048, w[0][0][c], w[0][1][c], w[TW - 1][0][c], w[TW - 1][1][c]);
  } else {
#pragma unroll
    for (int cc = 0; cc < 2; ++cc)
      ldsm_x4(wrec + lds_row + cc * 4096, w[0][0][2 * cc], w[0][1][2 * cc], w[0][0][2 * cc + 1], w[0][1][2 * cc + 1]);
  }
  uint32_t z2[TW][2];
  float s[TW][2];
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      s[T][h] = __half2float(__ushort_as_half((unsigned short)lds_u16(wrec + kW4RecCodes + 2 * row[T][h])));
      const uint32_t z = HASZ ? lds_u8(wrec + kW4RecCodes + 256 + row[T][h]) : 8u;
      z2[T][h] = 0x43004300u | z | (z << 16);
    }
  float d[TW][NT8][4];
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int t = 0; t < NT8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[T][t][e] = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 b[NT8];
#pragma unroll
    for (int t = 0; t < NT8; ++t) b[t] = lds128(ra + aoff[c] + t * 8 * 128);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
      for (int T = 0; T < TW; ++T) {
        const uint32_t a0 = code_pair(w[T][0][c], 2 * hh, z2[T][0]);
        const uint32_t a1 = code_pair(w[T][1][c], 2 * hh, z2[T][1]);
        const uint32_t a2 = code_pair(w[T][0][c], 2 * hh + 1, z2[T][0]);
        const uint32_t a3 = code_pair(w[T][1][c], 2 * hh + 1, z2[T][1]);
#pragma unroll
        for (int t = 0; t < NT8; ++t)
          mma_16816(d[T][t], a0, a1, a2, a3, hh ? b[t].z : b[t].x, hh ? b[t].w : b[t].y);
      }
    }
  }
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      acc[T][t][0] = fmaf(s[T][0], d[T][t][0], acc[T][t][0]);
      acc[T][t][1] = fmaf(s[T][0], d[T][t][1], acc[T][t][1]);
      acc[T][t][2] = fmaf(s[T][1], d[T][t][2], acc[T][t][2]);
      acc[T][t][3] = fmaf(s[T][1], d[T][t][3], acc[T][t][3]);
    }
}

template <int NT8, bool HASZ, int TWT>
__global__ void __launch_bounds__(RegCfg<NT8, TWT>::kThreads, RegCfg<NT8, TWT>::kCtasPerSm)
    w4a16_reg_kernel(const __grid_constant__ CUtensorMap tmap_a, const RegParams p) {
  using C = RegCfg<NT8, TWT>;
  constexpr int P = C::kP;
  constexpr int D = C::kD;
  constexpr int TW = C::kTw;

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
  const uint8_t* rec0 = p.packed + ((size_t)tile * p.k_blocks + kb0) * (size_t)p.rec_bytes;

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
  __syncthreads();  // barriers initialised

  // stage x: records x*P .. of the slice; weights (one bulk copy) and the
  // activations' boxes complete on full[x % D]; one thread
  const uint64_t pol_w = policy_evict_first();
  auto stage_bytes = [&](int x) { return (uint32_t)(min(P, nrec - x * P) * (p.rec_bytes + C::kRecA)); };
  auto issue_weights = [&](int x) {
    const int nr = min(P, nrec - x * P);
    bulk_g2s(smem + (x % D) * C::kStage, rec0 + (size_t)x * P * p.rec_bytes, (uint32_t)(nr * p.rec_bytes),
             &full[x % D], pol_w);
  };
  auto issue_acts = [&](int x) {
    const int nr = min(P, nrec - x * P);
    uint8_t* dst = smem + (x % D) * C::kStage + C::kWBytes;
    for (int u = 0; u < nr; ++u) {
      const int kx = (kb0 + x * P + u) * kBlockK;
      tma_load_2d(dst + u * C::kRecA, &tmap_a, kx, 0, &full[x % D]);
      tma_load_2d(dst + u * C::kRecA + C::kBox, &tmap_a, kx + 64, 0, &full[x % D]);
    }
  };
  // Phase 1: the first stages' weights before the previous kernel has
  // completed (no kernel on the stream writes them), unless the caller said
  // otherwise; their activations after griddepcontrol.wait.
  const int npre = min(D, nstage);
  if (threadIdx.x == 0) {
    for (int x = 0; x < npre; ++x) {
      mbar_arrive_expect_tx(&full[x], stage_bytes(x));
      if (p.early_weights) issue_weights(x);
    }
  }
  pdl_wait();   // activations, outputs, partials and counters may be in use until here
  if (threadIdx.x == 0) {
    for (int x = 0; x < npre; ++x) {
      if (!p.early_weights) issue_weights(x);
      issue_acts(x);
    }
  }
  int issued = npre;

  int row[TW][2];
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int h = 0; h < 2; ++h) row[T][h] = 16 * TW * warp + 16 * T + 8 * h + g;
  // ldmatrix row addresses: lane L gives row L % 8 of matrix L / 8; TW = 2:
  // matrix k = (T, h) = (k / 2, k % 2) of one chunk; TW = 1: matrix k =
  // (h, chunk) = (k % 2, c0 + k / 2) of a chunk pair
  const int mk = lane >> 3, mi = lane & 7;
  const uint32_t lds_row = TW == 2 ? (uint32_t)((16 * TW * warp + 16 * (mk >> 1) + 8 * (mk & 1) + mi) * 16)
                                   : (uint32_t)(((mk >> 1) * 128 + 16 * warp + 8 * (mk & 1) + mi) * 16);
  // activation reads: token row sigma(g) (+ 8t) of box c >> 1, piece 4 (c & 1) + qd
  const int tg = col_token(g);
  uint32_t aoff[4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    aoff[c] = (uint32_t)((c >> 1) * C::kBox + tg * 128 + (((4 * (c & 1) + qd) ^ tg) << 4));
  const uint32_t sbase = smem_u32(smem);

  float acc[TW][NT8][4];
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int t = 0; t < NT8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[T][t][e] = 0.f;

  bool ok = true;
  for (int j = 0; j < nstage; ++j) {
    // the producer refills the slot of stage j + D - 1, freed at the end of stage j - 1
    if (warp == 0 && j >= 1 && j + D - 1 < nstage) {
      const int x = j + D - 1;
      if (!hq_wait_warp(&empty[x % D], ((x / D) - 1) & 1, p.wait_ns, s_abort)) {
        if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[x % D], stage_bytes(x));
        issue_weights(x);
        issue_acts(x);
      }
      __syncwarp();
      issued = x + 1;
    }
    if (!hq_wait_warp(&full[j % D], (j / D) & 1, p.wait_ns, s_abort)) {
      if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
      ok = false;
      break;
    }
    const uint32_t st = sbase + (uint32_t)((j % D) * C::kStage);
#pragma unroll
    for (int u = 0; u < P; ++u) {
      const int r = j * P + u;
      if (r < nrec)
        reg_record<NT8, HASZ, TW>(st + (uint32_t)(u * p.rec_bytes), st + (uint32_t)(C::kWBytes + u * C::kRecA),
                                  lds_row, aoff, row, acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[j % D]);
  }
  if (!ok && lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
  if (warp == 0 && lane == 0 && *s_abort) {
    // let every copy already issued land before the CTA exits
    for (int x = issued > D ? issued - D : 0; x < issued; ++x) hq_wait(&full[x % D], (x / D) & 1, p.wait_ns, nullptr);
  }

  // ---- output: feature tile * 128 + row, token 8t + sigma(2 qd + (e & 1))
  auto store = [&](float (&v)[TW][NT8][4]) {
#pragma unroll
    for (int T = 0; T < TW; ++T)
#pragma unroll
      for (int t = 0; t < NT8; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int f = tile * kTileN + row[T][e >> 1];
          const int tok = 8 * t + col_token(2 * qd + (e & 1));
          if (f < p.n && tok < p.m) p.c[(size_t)tok * p.n + f] = __float2bfloat16_rn(v[T][t][e]);
        }
  };
  if (p.splits == 1) {
    store(acc);
    return;
  }
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
  using C = RegCfg<NT8, TWT>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem) != cudaSuccess)
      return HQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  return launch_pdl(kern, dim3(grid), dim3(C::kThreads), (size_t)C::kSmem, stream, map, p) == cudaSuccess
             ? HQ_OK
             : HQ_ERR_CUDA;
}

// Grouped MoE on the register path: persistent CTAs walk (expert, weight
// tile, 8*NT8-token tile) units built on the device from the expert row
// offsets, each over the whole K range (four warps of 32 rows).  One thread
// streams the units' stages through the ring without a gap between units;
// the warps finish a unit with its stores.  SW: weights in the gated gate+up
// row order, whose 32-row groups put a warp's 16 gate rows in its MMA tile 0
// and the matching up rows in tile 1, so each thread writes
// h = silu(gate) * up for its features directly.
template <int NT8>
struct RegGrpCfg {
  using C = RegCfg<NT8, 2>;
  static constexpr int kTabOff = C::kBarOff + 128;
  static constexpr int kSmem = kTabOff + 2 * (kMaxExperts + 1) * 4 + 1024;
  static constexpr int kCtasPerSm = reg_grouped_ctas_per_sm(NT8);
  static_assert(kCtasPerSm * (kSmem + 1024) <= 228 * 1024, "kCtasPerSm CTAs fit one SM's shared memory");
};

template <int NT8, bool HASZ, bool SW>
__global__ void __launch_bounds__(128, RegGrpCfg<NT8>::kCtasPerSm)
    w4a16_reg_grouped_kernel(const __grid_constant__ CUtensorMap tmap_a, const RegParams p) {
  using C = RegCfg<NT8, 2>;
  using G = RegGrpCfg<NT8>;
  constexpr int P = C::kP;
  constexpr int D = C::kD;
  constexpr int TW = 2;
  constexpr int NTOK = 8 * NT8;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + D;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + D);
  int* s_total = const_cast<int*>(s_abort + 1);
  int* s_off = reinterpret_cast<int*>(smem + G::kTabOff);   // [num_experts + 1]
  int* s_prefix = s_off + (kMaxExperts + 1);                 // [num_experts + 1]

  const int warp = (int)(threadIdx.x >> 5), lane = (int)(threadIdx.x & 31);
  const int g = lane >> 2, qd = lane & 3;
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
  pdl_wait();   // the expert offsets, activations and outputs may be in use until here
  const int E = p.num_experts;
  for (int i = (int)threadIdx.x; i <= E; i += (int)blockDim.x) s_off[i] = p.expert_offsets[i];
  __syncthreads();   // barriers initialised, offsets loaded
  if (threadIdx.x == 0) {
    int total = 0;
    bool bad = s_off[0] != 0 || s_off[E] != p.m;
    for (int e = 0; e < E; ++e) {
      s_prefix[e] = total;
      int rows = s_off[e + 1] - s_off[e];
      if (rows < 0) { bad = true; rows = 0; }
      total += ((rows + NTOK - 1) / NTOK) * p.n_tiles;
    }
    s_prefix[E] = total;
    if (bad) {
      atomicCAS(p.err, 0u, (uint32_t)HQ_ERR_DEVICE_BAD_OFFSETS);
      total = 0;
    }
    *s_total = total;
  }
  __syncthreads();

  auto get_unit = [&](int idx, RegUnit& x) -> bool {
    const int u = (int)blockIdx.x + idx * (int)gridDim.x;
    if (u >= *s_total) return false;
    // the expert e with prefix[e] <= u < prefix[e + 1] (empty experts share
    // their prefix with the next one, so the largest such e has rows)
    int lo = 0, hi = E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_prefix[mid] <= u) lo = mid; else hi = mid;
    }
    const int rows_e = s_off[lo + 1] - s_off[lo];
    const int mtiles = (rows_e + NTOK - 1) / NTOK;
    const int local = u - s_prefix[lo];
    const int mt = local % mtiles;
    x.nt = local / mtiles;
    x.rec0 = p.packed + (size_t)lo * p.expert_bytes + (size_t)x.nt * p.k_blocks * (size_t)p.rec_bytes;
    x.row0 = s_off[lo] + mt * NTOK;
    x.rows = min(NTOK, s_off[lo + 1] - x.row0);
    return true;
  };
  const int nrec = p.k_blocks;
  const int nstage = (nrec + P - 1) / P;

  // ---- producer state (thread 0): the next stage to issue
  const uint64_t pol_w = policy_evict_first();
  RegUnit pu{};
  int pidx = 0, psj = 0;
  bool pmore = false;
  int issued = 0;
  auto issue_next = [&](int X) {   // stage psj of unit pu into ring stage X
    const int r0 = psj * P, nr = min(P, nrec - r0);
    uint64_t* fb = &full[X % D];
    uint8_t* dst = smem + (X % D) * C::kStage;
    mbar_arrive_expect_tx(fb, (uint32_t)(nr * (p.rec_bytes + C::kRecA)));
    bulk_g2s(dst, pu.rec0 + (size_t)r0 * p.rec_bytes, (uint32_t)(nr * p.rec_bytes), fb, pol_w);
    for (int u = 0; u < nr; ++u) {
      const int kx = (r0 + u) * kBlockK;
      tma_load_2d(dst + C::kWBytes + u * C::kRecA, &tmap_a, kx, pu.row0, fb);
      tma_load_2d(dst + C::kWBytes + u * C::kRecA + C::kBox, &tmap_a, kx + 64, pu.row0, fb);
    }
    if (++psj == nstage) {
      psj = 0;
      pmore = get_unit(++pidx, pu);
    }
  };
  if (threadIdx.x == 0) {
    pmore = get_unit(0, pu);
    while (issued < D && pmore) issue_next(issued++);
  }

  int row[TW][2];
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int h = 0; h < 2; ++h) row[T][h] = 32 * warp + 16 * T + 8 * h + g;
  const int mk = lane >> 3, mi = lane & 7;
  const uint32_t lds_row = (uint32_t)((32 * warp + 16 * (mk >> 1) + 8 * (mk & 1) + mi) * 16);
  const int tg = col_token(g);
  uint32_t aoff[4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    aoff[c] = (uint32_t)((c >> 1) * C::kBox + tg * 128 + (((4 * (c & 1) + qd) ^ tg) << 4));
  const uint32_t sbase = smem_u32(smem);

  float acc[TW][NT8][4];
  auto zero = [&]() {
#pragma unroll
    for (int T = 0; T < TW; ++T)
#pragma unroll
      for (int t = 0; t < NT8; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[T][t][e] = 0.f;
  };
  zero();
  RegUnit cu{};
  int cidx = 0, csj = 0;
  bool cmore = get_unit(0, cu);
  bool ok = true;
  for (int X = 0; cmore; ++X) {
    // ring stage X + D - 1 reuses the slot of stage X - 1
    if (warp == 0 && X >= 1) {
      const bool more = __shfl_sync(0xffffffffu, (lane == 0 && pmore && issued == X + D - 1) ? 1 : 0, 0) != 0;
      if (more) {
        if (!hq_wait_warp(&empty[(X - 1) % D], ((X - 1) / D) & 1, p.wait_ns, s_abort)) {
          if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        if (lane == 0) issue_next(issued++);
        __syncwarp();
      }
    }
    if (!hq_wait_warp(&full[X % D], (X / D) & 1, p.wait_ns, s_abort)) {
      if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
      ok = false;
      break;
    }
    const uint32_t st = sbase + (uint32_t)((X % D) * C::kStage);
#pragma unroll
    for (int u = 0; u < P; ++u) {
      if (csj * P + u < nrec)
        reg_record<NT8, HASZ, TW>(st + (uint32_t)(u * p.rec_bytes), st + (uint32_t)(C::kWBytes + u * C::kRecA),
                                  lds_row, aoff, row, acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[X % D]);
    if (++csj < nstage) continue;
    // ---- the unit's output: token row0 + 8t + sigma(2 qd + (e & 1))
#pragma unroll
    for (int t = 0; t < NT8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = 8 * t + col_token(2 * qd + (e & 1));
        if (tok >= cu.rows) continue;
        const size_t r = (size_t)(cu.row0 + tok);
        if constexpr (SW) {
          const int hc = p.n >> 1;
          const int f = cu.nt * (kTileN / 2) + 16 * warp + 8 * (e >> 1) + g;
          const float gv = acc[0][t][e], uv = acc[1][t][e];
          if (f < hc) p.c[r * hc + f] = __float2bfloat16_rn(__fdividef(gv, 1.f + __expf(-gv)) * uv);
        } else {
#pragma unroll
          for (int T = 0; T < TW; ++T) {
            const int f = cu.nt * kTileN + row[T][e >> 1];
            if (f < p.n) p.c[r * p.n + f] = __float2bfloat16_rn(acc[T][t][e]);
          }
        }
      }
    zero();
    csj = 0;
    cmore = get_unit(++cidx, cu);
  }
  if (!ok && lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
  if (warp == 0 && lane == 0 && *s_abort) {
    // let every copy already issued land before the CTA exits
    for (int X = issued > D ? issued - D : 0; X < issued; ++X) hq_wait(&full[X % D], (X / D) & 1, p.wait_ns, nullptr);
  }
}

template <int NT8, bool HASZ, bool SW>
hq_status reg_grouped_launch_t(const CUtensorMap& map, const RegParams& p, int grid, cudaStream_t stream) {
  auto kern = w4a16_reg_grouped_kernel<NT8, HASZ, SW>;
  using G = RegGrpCfg<NT8>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::kSmem) != cudaSuccess)
      return HQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  return launch_pdl(kern, dim3(grid), dim3(128), (size_t)G::kSmem, stream, map, p) == cudaSuccess ? HQ_OK
                                                                                                  : HQ_ERR_CUDA;
}

}  // namespace
}  // namespace w4

using w4::RegParams;

// CTAs per weight tile (K slices) of the register-path plan: the largest
// split whose grid fits reg_slots_per_sm CTAs per SM (more CTAs, more bytes in
// flight; one record per CTA at least).  Measured on B200 (back to back,
// per launch): K=18432 N=7168 M=1 at 4..10 slices 31.9 / 26.8 / 24.8 / 22.9
// / 26.6 / 25.5 us (7 best: 392 CTAs); M=16 41.1 .. 26.0 (10 best: 560 CTAs);
// K=7168 N=18432 M=1 26.0 / 20.8 / 24.5 at 2 / 3 / 4, M=16 32.4 / 29.5 / 24.8.
int reg_splits(int num_sms, const hq_quant_desc& d, int m) {
  const long long tiles = (d.n + kTileN - 1) / kTileN;
  const long long kbs = d.k / kBlockK;
  const long long slots = (long long)num_sms * reg_slots_per_sm(m <= 8 ? 1 : 2);
  return (int)std::max<long long>(1, std::min<long long>(kbs, slots / tiles));
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
  // on each busy SM); else four warps of 32 rows
  if (cfg.reg_tw == 1) {
    if (nt8 == 1)
      return hz ? w4::reg_launch_t<1, true, 1>(map, p, cfg.grid, stream) : w4::reg_launch_t<1, false, 1>(map, p, cfg.grid, stream);
    return hz ? w4::reg_launch_t<2, true, 1>(map, p, cfg.grid, stream) : w4::reg_launch_t<2, false, 1>(map, p, cfg.grid, stream);
  }
  if (nt8 == 1)
    return hz ? w4::reg_launch_t<1, true, 2>(map, p, cfg.grid, stream) : w4::reg_launch_t<1, false, 2>(map, p, cfg.grid, stream);
  return hz ? w4::reg_launch_t<2, true, 2>(map, p, cfg.grid, stream) : w4::reg_launch_t<2, false, 2>(map, p, cfg.grid, stream);
}

hq_status reg_launch_grouped(const hq_quant_desc& d, const W4Config& cfg, const void* packed, const void* a,
                             int total_rows, void* c, const int32_t* expert_offsets, void* ws, cudaStream_t stream,
                             int swiglu) {
  if (d.fmt != HQ_FMT_INT4 || d.num_experts < 2 || d.num_experts > w4::kMaxExperts || total_rows < 1)
    return HQ_ERR_UNSUPPORTED;
  if (cfg.ntok != 8 && cfg.ntok != 16) return HQ_ERR_INVALID_ARG;
  RegParams p{};
  p.packed = static_cast<const uint8_t*>(packed);
  p.c = static_cast<__nv_bfloat16*>(c);
  p.err = static_cast<uint32_t*>(ws);
  p.wait_ns = kDefaultWaitNs;
  p.m = total_rows;
  p.n = d.n;
  p.k_blocks = d.k / kBlockK;
  p.rec_bytes = w4_record_bytes(d.has_zero_point != 0);
  p.splits = 1;
  p.expert_offsets = expert_offsets;
  p.n_tiles = (d.n + kTileN - 1) / kTileN;
  p.expert_bytes = (uint64_t)p.n_tiles * p.k_blocks * p.rec_bytes;
  p.num_experts = d.num_experts;
  CUtensorMap map;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return HQ_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)d.k, (cuuint64_t)total_rows};
  cuuint64_t strides[1] = {(cuuint64_t)d.k * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)cfg.ntok};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return HQ_ERR_CUDA;
  const bool hz = d.has_zero_point != 0;
  const int grid = cfg.grid;
  if (cfg.ntok == 8) {
    if (swiglu)
      return hz ? w4::reg_grouped_launch_t<1, true, true>(map, p, grid, stream) : w4::reg_grouped_launch_t<1, false, true>(map, p, grid, stream);
    return hz ? w4::reg_grouped_launch_t<1, true, false>(map, p, grid, stream) : w4::reg_grouped_launch_t<1, false, false>(map, p, grid, stream);
  }
  if (swiglu)
    return hz ? w4::reg_grouped_launch_t<2, true, true>(map, p, grid, stream) : w4::reg_grouped_launch_t<2, false, true>(map, p, grid, stream);
  return hz ? w4::reg_grouped_launch_t<2, true, false>(map, p, grid, stream) : w4::reg_grouped_launch_t<2, false, false>(map, p, grid, stream);
}

}  // namespace hq
