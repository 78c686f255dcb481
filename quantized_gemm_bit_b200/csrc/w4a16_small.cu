// W4A16 GEMM for small token tiles (16, 32 or 64 tokens): the
// weight-bandwidth-bound regime, where the fused dequantization has to keep
// up with HBM.
//
// Method: the weights are 4-bit codes q with a per-group fp16 scale s and an
// optional uint4 zero point z, w = (q - z) * s ("Humming: open-source kernel
// library for quantized inference", summary paragraph 2), converted inside
// the kernel (same page, paragraph 3).  Because the scale is constant over a
// group of 128 K, the sum over one group factors as
//     sum_k (q_k - z) s a_k  =  s * sum_k (q_k - z) a_k ,
// so this kernel feeds the tensor core the exact small integers (q - z) (bf16
// holds -15..15 exactly) and applies s once per group and output element in
// fp32.  Compared with rescaling every weight in bf16 this takes one bf16x2
// multiply per weight pair off the dequantization warps and never rounds s
// or w to bf16.
//
// B200 design:
//   * swap-AB as in the other W4A16 kernel: 128 weight rows are the MMA's M
//     side, read from TMEM; the tokens are the N side, TMA-staged in shared
//     memory with the 128-byte swizzle;
//   * each pipeline stage holds two 128-K records; its MMAs write one fresh
//     fp32 tile D_g (128 x NTOK) per group g into a TMEM ring instead of
//     accumulating across K;
//   * warps 8 and up unpack codes in groups of four warps (one per 32-row
//     quarter; three groups for 16/32 tokens, two for 64), each group
//     owning every stage it == g (mod groups) and one TMEM weight slot, so
//     several stages are unpacked at once and the groups run ahead of the
//     MMA;
//   * warps 4-7 ("scale warps") read s for their 32 rows from the stage in
//     shared memory, then fold s * D_g into fp32 registers as each D_g
//     lands, and write the output (or the stream-K partial) when a unit
//     ends.  The order of the fp32 sum is fixed, so results repeat bit for
//     bit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "hq_internal.h"
#include "ptx.cuh"
#include "w4a16_common.cuh"

namespace hq {
namespace w4 {

namespace {

constexpr int cgcd(int a, int b) { return b == 0 ? a : cgcd(b, a % b); }

template <int NTOK, int FMT>
struct SmallCfg {
  static constexpr int kKps = 2;                        // records (groups) per stage
  static constexpr int kABlock = NTOK * 256;            // one record's activations: two 64-K boxes
  static constexpr int kATile = kKps * kABlock;
  static constexpr int kCodeBytes = FMT == kFmtInt3   ? kW3RecCodes
                                    : FMT == kFmtInt2 ? kW2RecCodes
                                    : FMT == kFmtInt8 ? kW8RecCodes
                                                      : kW4RecCodes;
  static constexpr int kRecStride = kCodeBytes + 384;  // codes, fp16 scales, zero points
  static constexpr int kRecs = kKps * kRecStride;
  static constexpr uint32_t kZSym = FMT == kFmtInt3 ? 4u : FMT == kFmtInt2 ? 2u : FMT == kFmtInt8 ? 128u : 8u;
  // Unpacking warps form kNdq groups of kGroupWarps; group g owns the
  // stages it with it % kNdq == g, and its warps split each of its stages
  // (4 row quarters x kGroupWarps / 4 parts of the stage's 32-K chunks).
  // Groups owning whole stages keep several stages in flight with few
  // synchronizations each (measured on B200 against every warp sharing
  // every stage).
  static constexpr int kNdq = NTOK == 64 ? 2 : 3;
  static constexpr int kGroupWarps = 4;
  static constexpr int kUnpackWarps = kNdq * kGroupWarps;
  static constexpr int kChunks = 4 * kKps * 4 / kGroupWarps;   // 32-K chunks per unpacking warp and stage
  static constexpr int kEpiScratch = 4 * 2048;          // warp-local transposes of the output
  static constexpr int kBarBytes = 512;
  // as many SMEM stages as fit, up to a preferred depth per token tile
  static constexpr int kSmemPref = NTOK == 16 ? 8 : NTOK == 32 ? 6 : 4;
  // (exact: the budget less the base alignment and the scratch is a
  // multiple of 128, so rounding the tables' end up to 128 stays inside it
  // whenever the unrounded end does)
  static constexpr int kSmemFit =
      (int)((232448 - 1024 - kEpiScratch - kBarBytes - 2 * (kMaxExperts + 1) * sizeof(int)) / (kATile + kRecs));
  static constexpr int kSmemStages = kSmemPref < kSmemFit ? kSmemPref : kSmemFit;
  static constexpr int kAStages = NTOK == 64 ? 2 : 3;   // TMEM ring of unpacked weights
  static constexpr int kDStages = NTOK == 16 ? 4 : 2;   // TMEM ring of per-group results
  static constexpr int kACols = kKps * 64;              // TMEM columns per weight stage
  static constexpr int kDCols = kKps * NTOK;            // TMEM columns per result stage
  static constexpr int kThreads = (8 + kUnpackWarps) * 32;
  // full barriers, one per (SMEM stage, unpacking group): iteration `it`
  // uses barrier (it % SS, it % NDQ), so every waiter sees each phase of
  // its barriers in order whatever the ring depth
  static constexpr int kFullBars = kSmemStages * kNdq;
  static constexpr int kFullPeriod = kSmemStages / cgcd(kSmemStages, kNdq) * kNdq;  // lcm
  // Warp 1 issues every MMA.  (Letting the last unpacking warp to finish a
  // stage issue that stage's MMAs measured slower on B200: single-lane issue
  // from a busy warp; so did one issuing warp per unpacking group, whose
  // unpacking then ran slower.  A clock trace of one CTA at M=16 shows each
  // stage costs the issuer ~1260 SM cycles: ~450 for one probe of its three
  // (already complete) mbarriers, ~480 to issue the 16 MMAs, the rest its
  // loop.  Several issuers would also need a result ring of at least as
  // many stages as groups, or a parity wait could mistake a phase two
  // behind for the one it waits for.)
  // byte offsets from the 1024-aligned base of dynamic shared memory
  static constexpr size_t kBarOff = (size_t)kSmemStages * (kATile + kRecs);
  static constexpr size_t kTabOff = kBarOff + kBarBytes;                          // s_prefix, s_off
  static constexpr size_t kScrOff = (kTabOff + 2 * (kMaxExperts + 1) * sizeof(int) + 127) / 128 * 128;
  static constexpr size_t kSmem = 1024 + kScrOff + kEpiScratch;
  static_assert(kABlock % 1024 == 0 && kRecStride % 16 == 0 && kBarOff % 16 == 0, "stage alignment");
  static_assert(kACols * kAStages + kDCols * kDStages <= 512, "TMEM budget");
  static_assert(kAStages % kNdq == 0, "every TMEM weight stage must always return to the same group");
  static_assert(kGroupWarps % 4 == 0 && kChunks * kGroupWarps == 16 * kKps, "chunk split");
  static_assert(8 * (kFullBars + kSmemStages + 2 * kAStages + 2 * kDStages + 1) + 16 <= kBarBytes,
                "barrier area");
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(kSmemStages >= 2, "pipeline depth");
};

// One 32-K chunk c of weight row r of a record, exact: the bf16 values
// (q - z) (bf16 holds every such integer, up to 255 in magnitude) as 16
// words of two weights (even k in the low half).  Codes of up to 4 bits:
// OR-ing a code into the mantissa of bf16 128.0 gives bf16(128 + q), and
// (128 + q) - (128 + z) is q - z exactly.  INT8 codes: 2^23 + q in fp32,
// minus 2^23 + z, is q - z exactly, and so is its conversion to bf16.
template <int FMT>
__device__ __forceinline__ void unpack_chunk(const uint8_t* rec, int c, int r, uint32_t z, uint32_t (&out)[16]) {
  const uint32_t zbits = 0x4300u + z;
  const uint32_t z2 = zbits | (zbits << 16);
  if constexpr (FMT == kFmtInt8) {
    // 16-K chunks 2c and 2c + 1 of the row, 16 code bytes each
    const float zf = 8388608.f + (float)z;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 raw = *reinterpret_cast<const uint4*>(rec + ((2 * c + h) * 128 + r) * 16);
      const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        out[8 * h + 2 * w] = pack_bf16x2(u8_minus_zero(wv[w], 0, zf), u8_minus_zero(wv[w], 1, zf));
        out[8 * h + 2 * w + 1] = pack_bf16x2(u8_minus_zero(wv[w], 2, zf), u8_minus_zero(wv[w], 3, zf));
      }
    }
  } else if constexpr (FMT == kFmtInt3) {
    // words 3c .. 3c+2 of the row: pairs 0-14 at bits 3j / 16 + 3j of word
    // 3c + i/5, pair 15 from bit p at 15 / 31 of word 3c + p
    uint32_t wv[3];
#pragma unroll
    for (int p = 0; p < 3; ++p) {
      const int q = 3 * c + p;
      wv[p] = *reinterpret_cast<const uint32_t*>(rec + ((q >> 2) * 128 + r) * 16 + 4 * (q & 3));
    }
#pragma unroll
    for (int p = 0; p < 3; ++p) {
#pragma unroll
      for (int j = 0; j < 5; ++j)
        out[5 * p + j] = bf16x2_sub(lop3_and_or(wv[p] >> (3 * j), 0x00070007u, 0x43004300u), z2);
    }
    uint32_t x2 = lop3_and_or(wv[0] >> 15, 0x00010001u, 0x43004300u);
    x2 = lop3_and_or(wv[1] >> 14, 0x00020002u, x2);
    x2 = lop3_and_or(wv[2] >> 13, 0x00040004u, x2);
    out[15] = bf16x2_sub(x2, z2);
  } else if constexpr (FMT == kFmtInt2) {
    // words 2c, 2c+1 of the row: pair i at bits 2j / 16 + 2j of word 2c + i/8
    const uint2 wv = *reinterpret_cast<const uint2*>(rec + ((c >> 1) * 128 + r) * 16 + 8 * (c & 1));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      out[j] = bf16x2_sub(lop3_and_or(wv.x >> (2 * j), 0x00030003u, 0x43004300u), z2);
      out[8 + j] = bf16x2_sub(lop3_and_or(wv.y >> (2 * j), 0x00030003u, 0x43004300u), z2);
    }
  } else {
    // 16 bytes: the nibbles of k = 2j and 2j+1 of each word at bits 4j and 16+4j
    const uint4 raw = *reinterpret_cast<const uint4*>(rec + (c * 128 + r) * 16);
    const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
      for (int j = 0; j < 4; ++j) out[w * 4 + j] = bf16x2_sub(lop3_and_or(wv[w] >> (4 * j), 0x000F000Fu, 0x43004300u), z2);
    }
  }
}

// Unpack the chunks [c0, c0 + NCH) of a stage (chunk i = record i / 4,
// 32-K chunk i % 4 of it) for weight row r into TMEM lane r: each chunk
// fills 16 columns from taddr + 16 * i.  Records at or past `nrec` (the
// ragged end of a unit) are skipped.
template <int FMT, int NCH, int CODE_BYTES, uint32_t ZSYM>
__device__ __forceinline__ void unpack_stage(const uint8_t* recs, int rec_bytes, int nrec, int c0, int r, int has_zero,
                                             uint32_t taddr) {
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int ci = c0 + i;
    const int rr = ci >> 2;
    if (rr >= nrec) break;
    const uint8_t* rec = recs + rr * rec_bytes;
    const uint32_t z = has_zero ? rec[CODE_BYTES + 256 + r] : ZSYM;
    uint32_t out[16];
    unpack_chunk<FMT>(rec, ci & 3, r, z, out);
    tmem_st_x16(taddr + ci * 16, out);
  }
}

template <int NTOK, int FMT, bool SW>
__global__ void __launch_bounds__(SmallCfg<NTOK, FMT>::kThreads, 1)
    w4a16_small_kernel(const __grid_constant__ CUtensorMap tmap_a, const W4Params p) {
  using C = SmallCfg<NTOK, FMT>;
  constexpr int SS = C::kSmemStages;
  constexpr int AS = C::kAStages;
  constexpr int DS = C::kDStages;
  constexpr int KPS = C::kKps;
  constexpr int NDQ = C::kNdq;
  constexpr int kATile = C::kATile;
  constexpr int kRecs = C::kRecs;
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, NTOK);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                               // SS * kATile (activations, 128-byte swizzle)
  uint8_t* sR = smem + SS * kATile;                 // SS * kRecs (packed weight records)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + C::kFullBars;  // MMA commit + the four scale warps
  uint64_t* aready = empty + SS;    // the owning group's unpacking warps
  uint64_t* afree = aready + AS;    // MMA commit
  uint64_t* dfull = afree + AS;     // MMA commit
  uint64_t* dempty = dfull + DS;    // four scale warps
  uint64_t* drain = dempty + DS;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_total = const_cast<int*>(s_abort + 1);
  int* s_prefix = reinterpret_cast<int*>(smem + C::kTabOff);  // [kMaxExperts + 1]
  int* s_off = s_prefix + (kMaxExperts + 1);                    // [kMaxExperts + 1]
  uint16_t* epi_scratch = reinterpret_cast<uint16_t*>(smem + C::kScrOff);  // 16-byte aligned
  auto full_bar = [&](uint32_t i) { return &full[(i % SS) * NDQ + (i % NDQ)]; };
  auto full_par = [](uint32_t i) { return (i / C::kFullPeriod) & 1; };

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0) {
    for (int f = 0; f < C::kFullBars; ++f) mbar_init(&full[f], 1);
    for (int s = 0; s < SS; ++s) mbar_init(&empty[s], 5);
    for (int t = 0; t < AS; ++t) {
      mbar_init(&aready[t], C::kGroupWarps);
      mbar_init(&afree[t], 1);
    }
    for (int d = 0; d < DS; ++d) {
      mbar_init(&dfull[d], 1);
      mbar_init(&dempty[d], 4);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    *s_total = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 0) pdl_launch_dependents();
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_a);
  // Everything but the packed weights may be written by the previous kernel
  // on the stream: grouped mode needs the expert offsets at once
  if (p.grouped) {
    pdl_wait();
    grouped_tables<NTOK>(p, s_off, s_prefix, s_total);
  }
  __syncthreads();   // barriers (and the grouped tables) visible to every role
  const int total_grouped = *s_total;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp, elected lane issues)
    const bool leader = elect_one();
    const uint64_t pol_w = p.weights_once ? policy_evict_first() : policy_evict_last();
    Unit x;
    // Phase 1, before the previous kernel has finished: the packed weights
    // of the first SS stages (no kernel writes them)
    uint32_t n_pre = 0;
    // stages in flight: the whole ring unless the caller asked for fewer
    const uint32_t lim = (p.stage_limit > 0 && p.stage_limit < SS) ? (uint32_t)p.stage_limit : (uint32_t)SS;
    if (!p.grouped) {
      for (int idx = 0; p.early_weights && n_pre < lim && get_unit<NTOK>(p, s_prefix, s_off, total_grouped, idx, x);
           ++idx) {
        const uint8_t* wbase = p.packed + (uint64_t)x.nt * p.k_blocks * p.rec_bytes;
        for (int kb = x.kb0; kb < x.kb1 && n_pre < lim; kb += KPS, ++n_pre) {
          const int nrec = min(KPS, x.kb1 - kb);
          if (leader) {
            uint64_t* fb = full_bar(n_pre);
            mbar_arrive_expect_tx(fb, (uint32_t)nrec * ((uint32_t)p.rec_bytes + C::kABlock));
            bulk_g2s(sR + n_pre * kRecs, wbase + (uint64_t)kb * p.rec_bytes, (uint32_t)(nrec * p.rec_bytes), fb,
                     pol_w);
          }
          __syncwarp();
        }
      }
      pdl_wait();
    }
    // Phase 2: the activations of those stages, then the steady ring
    uint32_t it = 0;
    bool ok = true;
    for (int idx = 0; ok && get_unit<NTOK>(p, s_prefix, s_off, total_grouped, idx, x); ++idx) {
      const uint8_t* wbase =
          p.packed + (uint64_t)x.expert * p.expert_bytes + (uint64_t)x.nt * p.k_blocks * p.rec_bytes;
      for (int kb = x.kb0; kb < x.kb1; kb += KPS, ++it) {
        const int s = it % SS;
        const int nrec = min(KPS, x.kb1 - kb);
        if (!wait_stage_free<SS>(empty, it, lim, p.wait_ns, s_abort)) {
          if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        if (leader) {
          uint64_t* fb = full_bar(it);
          if (it >= n_pre) {
            mbar_arrive_expect_tx(fb, (uint32_t)nrec * ((uint32_t)p.rec_bytes + C::kABlock));
            // the stage's records are consecutive in the blob: one bulk copy
            // (long copies stream HBM much faster than record-sized ones)
            bulk_g2s(sR + s * kRecs, wbase + (uint64_t)kb * p.rec_bytes, (uint32_t)(nrec * p.rec_bytes), fb, pol_w);
          }
          for (int r = 0; r < nrec; ++r) {
            uint8_t* a_dst = sA + s * kATile + r * C::kABlock;
            tma_load_2d(a_dst, &tmap_a, (kb + r) * kBlockK, x.row0, fb);
            tma_load_2d(a_dst + NTOK * 128, &tmap_a, (kb + r) * kBlockK + 64, x.row0, fb);
          }
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      // let every copy already issued land before the CTA exits
      const uint32_t first = it > (uint32_t)SS ? it - SS : 0;
      for (uint32_t j = first; j < it; ++j) hq_wait(full_bar(j), full_par(j), p.wait_ns, nullptr);
    }
  } else {
  // The producer needs no TMEM, so it starts loading at once; the other
  // roles wait here for the allocation.
  if (warp == 2) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  if (!p.grouped) pdl_wait();   // outputs, partials and counters may be in use by the previous kernel
  tc_fence_before();
  named_bar(1, C::kThreads - 32);
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  auto a_col = [](int t) -> uint32_t { return (uint32_t)(t * C::kACols); };
  auto d_col = [](int d) -> uint32_t { return (uint32_t)(AS * C::kACols + d * C::kDCols); };
  // MMAs of one stage (called by a single thread): record r of the stage
  // writes a fresh fp32 tile D(d, r) = W_r^T-slice x A_r, eight K=16 steps;
  // descriptors advance by constants: 32 B per 16-K step inside a 128-byte
  // swizzle row, one box (NTOK rows) per 64 K
  auto issue_stage = [&](int s, int t, int d, int nrec) {
    const uint64_t b0 = smem_desc_sw128(smem_u32(sA + s * kATile));
    const uint32_t a0 = tmem_base + a_col(t);
    const uint32_t d0 = tmem_base + d_col(d);
    for (int r = 0; r < nrec; ++r) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint64_t bdesc = b0 + (uint64_t)((r * C::kABlock + (j >> 2) * (NTOK * 128) + (j & 3) * 32) >> 4);
        mma_bf16_ts(d0 + r * NTOK, a0 + r * 64 + j * 8, bdesc, kIdesc, j > 0 ? 1u : 0u);
      }
    }
    tc_commit(&empty[s]);
    tc_commit(&afree[t]);
    tc_commit(&dfull[d]);
  };

  if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp, elected lane issues)
    // one lane, fixed for the whole kernel, issues every MMA and commit: a
    // commit tracks the tcgen05 operations of the thread that issues it
    const bool leader = elect_one();
    uint32_t it = 0;
    bool ok = true;
    Unit x;
    for (int idx = 0; ok && get_unit<NTOK>(p, s_prefix, s_off, total_grouped, idx, x); ++idx) {
      for (int kb = x.kb0; kb < x.kb1; kb += KPS, ++it) {
        const int s = it % SS, t = it % AS, d = it % DS;
        const int nrec = min(KPS, x.kb1 - kb);
        if (!hq_wait_warp_n(3, &aready[t], (it / AS) & 1, full_bar(it), full_par(it), &dempty[d],
                            ((it / DS) & 1) ^ 1, p.wait_ns, s_abort)) {
          if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) issue_stage(s, t, d, nrec);
        __syncwarp();
      }
    }
    // make sure no MMA is still running when TMEM is released
    if (leader) {
      tc_commit(drain);
      hq_wait(drain, 0, p.wait_ns, nullptr);
    }
    __syncwarp();
  } else if (warp >= 8) {
    // ------------------------------------------------------------ unpack codes (warps 8 and up)
    // warp 8 + kGroupWarps * g + 4u + q belongs to group g and unpacks rows
    // 32q .. 32q+31 of the chunks [u * NCH, (u + 1) * NCH) of every stage
    // the group owns
    constexpr int NCH = C::kChunks;
    const int wi = (int)warp - 8;
    const int g = wi / C::kGroupWarps;
    const int u = (wi % C::kGroupWarps) >> 2;
    const uint32_t q = warp & 3;
    const int c0 = u * NCH;
    const int r = (int)(q * 32 + lane);               // weight row within the tile
    const uint32_t lane_addr = (q * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    Unit x;
    for (int idx = 0; ok && get_unit<NTOK>(p, s_prefix, s_off, total_grouped, idx, x); ++idx) {
      for (int kb = x.kb0; kb < x.kb1; kb += KPS, ++it) {
        if ((int)(it % NDQ) != g) continue;
        const int s = it % SS, t = it % AS;
        const int nrec = min(KPS, x.kb1 - kb);
        // The full barrier of (stage, group) and TMEM stage t (AS % NDQ == 0)
        // only ever serve this group, and neither can move on before this
        // group's own arrival (through the MMA it enables): every phase of
        // both is observed in order
        if (!hq_wait_warp_n(2, full_bar(it), full_par(it), &afree[t], ((it / AS) & 1) ^ 1, nullptr, 0, p.wait_ns,
                            s_abort)) {
          if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        unpack_stage<FMT, NCH, C::kCodeBytes, C::kZSym>(sR + s * kRecs, p.rec_bytes, nrec, c0, r, p.has_zero,
                                                         tmem_base + lane_addr + a_col(t));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&aready[t]);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ scale warps + epilogue (warps 4-7)
    const uint32_t q = warp & 3;
    const int r = (int)(q * 32 + lane);
    const uint32_t lane_addr = (q * 32) << 16;
    constexpr int CH = NTOK >= 64 ? 32 : 16;          // TMEM columns per load batch
    uint32_t it = 0;
    bool ok = true;
    Unit x, pend;          // pend: the split tile this CTA reduces after its last unit
    bool has_pend = false;
    for (int idx = 0; ok && get_unit<NTOK>(p, s_prefix, s_off, total_grouped, idx, x); ++idx) {
      float acc[NTOK];
#pragma unroll
      for (int j = 0; j < NTOK; ++j) acc[j] = 0.f;
      for (int kb = x.kb0; kb < x.kb1; kb += KPS, ++it) {
        const int s = it % SS, d = it % DS;
        const int nrec = min(KPS, x.kb1 - kb);
        if (!hq_wait(full_bar(it), full_par(it), p.wait_ns, s_abort)) {
          raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        float sc[KPS];
#pragma unroll
        for (int rr = 0; rr < KPS; ++rr)
          sc[rr] = rr < nrec ? __half2float(reinterpret_cast<const __half*>(sR + s * kRecs + rr * p.rec_bytes +
                                                                            C::kCodeBytes)[r])
                             : 0.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (!hq_wait(&dfull[d], (it / DS) & 1, p.wait_ns, s_abort)) {
          raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int rr = 0; rr < KPS; ++rr) {
          if (rr < nrec) {
#pragma unroll
            for (int j0 = 0; j0 < NTOK; j0 += CH) {
              uint32_t v0[16], v1[16];
              const uint32_t src = tmem_base + lane_addr + d_col(d) + rr * NTOK + j0;
              tmem_ld_x16(src, v0);
              if (CH == 32) tmem_ld_x16(src + 16, v1);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < CH; ++j)
                acc[j0 + j] = fmaf(sc[rr], __uint_as_float(j < 16 ? v0[j] : v1[j - 16]), acc[j0 + j]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dempty[d]);
      }
      if (!ok) break;

      // ---- output of this unit
      float* part = x.partial ? p.partials + ((size_t)blockIdx.x * 2 + x.slot) * NTOK * kTileN : nullptr;
      uint16_t* scr = epi_scratch + q * 1024;
#pragma unroll
      for (int j0 = 0; j0 < NTOK; j0 += CH) {
        float v[CH];
#pragma unroll
        for (int j = 0; j < CH; ++j) v[j] = acc[j0 + j];
        store_chunk<CH, SW>(p, x, part, (int)q, (int)lane, j0, v, scr);
      }
      if (sk_is_reducer(p, x)) {
        pend = x;
        has_pend = true;
      } else if (x.partial) {
        sk_signal(p, x, (int)q, (int)lane);
      }
    }
    if (ok && has_pend) sk_reduce<NTOK, (C::kThreads > 512 ? 2 : 4)>(p, pend, (int)q, (int)lane);
  }

  }  // non-producer roles

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(*s_tmem, 512);
}

template <int NTOK, int FMT, bool SW>
hq_status launch_small_t(const CUtensorMap& map, const W4Params& p, int grid, cudaStream_t stream) {
  auto kern = w4a16_small_kernel<NTOK, FMT, SW>;
  using C = SmallCfg<NTOK, FMT>;
  const size_t smem = C::kSmem;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return HQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  return launch_pdl(kern, dim3(grid), dim3(C::kThreads), smem, stream, map, p) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

template <int FMT, bool SW>
hq_status small_launch_f(int ntok, const CUtensorMap& map, const W4Params& p, int grid, cudaStream_t stream) {
  switch (ntok) {
    case 16: return launch_small_t<16, FMT, SW>(map, p, grid, stream);
    case 32: return launch_small_t<32, FMT, SW>(map, p, grid, stream);
    case 64: return launch_small_t<64, FMT, SW>(map, p, grid, stream);
    default: return HQ_ERR_UNSUPPORTED;
  }
}

template <int FMT>
hq_status small_launch_sw(int ntok, bool swiglu, const CUtensorMap& map, const W4Params& p, int grid,
                          cudaStream_t stream) {
  return swiglu ? small_launch_f<FMT, true>(ntok, map, p, grid, stream)
                : small_launch_f<FMT, false>(ntok, map, p, grid, stream);
}

}  // namespace

namespace {
template <int FMT>
int small_depth_f(int ntok) {
  return ntok == 16 ? SmallCfg<16, FMT>::kSmemStages : ntok == 32 ? SmallCfg<32, FMT>::kSmemStages
                                                                  : SmallCfg<64, FMT>::kSmemStages;
}
}  // namespace

int small_ring_depth(int ntok, int fmt) {
  switch (fmt) {
    case kFmtInt3: return small_depth_f<kFmtInt3>(ntok);
    case kFmtInt2: return small_depth_f<kFmtInt2>(ntok);
    case kFmtInt8: return small_depth_f<kFmtInt8>(ntok);
    default: return small_depth_f<kFmtInt4>(ntok);
  }
}

hq_status small_launch(int ntok, int fmt, bool swiglu, const CUtensorMap& map, const W4Params& p, int grid,
                       cudaStream_t stream) {
  switch (fmt) {
    case kFmtInt4: return small_launch_sw<kFmtInt4>(ntok, swiglu, map, p, grid, stream);
    case kFmtInt3: return small_launch_sw<kFmtInt3>(ntok, swiglu, map, p, grid, stream);
    case kFmtInt2: return small_launch_sw<kFmtInt2>(ntok, swiglu, map, p, grid, stream);
    case kFmtInt8: return small_launch_sw<kFmtInt8>(ntok, swiglu, map, p, grid, stream);
    default: return HQ_ERR_UNSUPPORTED;
  }
}

}  // namespace w4
}  // namespace hq
