// Dense and grouped (MoE) W4A16 GEMM for sm_100a with the INT4 dequantization
// fused into the kernel (also run with INT3, INT2, INT8, MXFP4 or MXINT4
// weights: the same kernel with another record decode).
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
#include <cmath>
#include <cstdio>

#include "hq_internal.h"
#include "ptx.cuh"
#include "w4a16_common.cuh"

namespace hq {

using namespace w4;

namespace {

constexpr int cgcd(int a, int b) { return b == 0 ? a : cgcd(b, a % b); }

// CG = 2: a CTA pair (cluster of two) runs one 256-row weight tile with
// cta_group::2 MMAs; each CTA dequantizes its own 128 weight rows into its
// TMEM and stages half of the token tile.
template <int NTOK, int FMT = kFmtInt4, int CG = 1>
struct Cfg {
  static_assert(CG == 1 || NTOK == 256, "CTA pairs run 256-token tiles");
  // records (128-K blocks) per pipeline stage: two for the small token tiles,
  // whose MMAs are cheap, so the per-stage waits and commits are amortized
  static constexpr int kKps = NTOK <= 64 ? 2 : 1;
  static constexpr int kABlock = NTOK / CG * 256;           // one record's activations (this CTA's): two 64-K boxes
  static constexpr int kATile = kKps * kABlock;
  static constexpr int kRecStride = (FMT == kFmtMx || FMT == kFmtMxi4) ? kMxA16RecBytes
                                    : FMT == kFmtInt3                  ? kW3RecCodes + 384
                                    : FMT == kFmtInt2                  ? kW2RecCodes + 384
                                    : FMT == kFmtInt8                  ? kW8RecCodes + 384
                                                                       : kRecMax;
  static constexpr int kRecs = kKps * kRecStride;
  static constexpr int kBarBytes = (FMT == kFmtMx || FMT == kFmtMxi4) ? 384 : 512;
  static constexpr int kEpiScratch = NTOK == 256 ? 0 : 4 * 2048;
  // as many SMEM stages as fit, up to a preferred depth per token tile
  static constexpr int kSmemPref = NTOK == 16 ? 6 : NTOK == 32 ? 6 : NTOK == 64 ? 3 : NTOK == 128 ? 5 : CG == 2 ? 8 : 3;
  // (exact: the budget less the base alignment and the scratch is a
  // multiple of 128, so rounding the tables' end up to 128 stays inside it
  // whenever the unrounded end does)
  static constexpr int kSmemFit =
      (int)((232448 - 1024 - kEpiScratch - kBarBytes - 2 * (kMaxExperts + 1) * sizeof(int)) / (kATile + kRecs));
  static constexpr int kSmemStages = kSmemPref < kSmemFit ? kSmemPref : kSmemFit;
  static constexpr int kTmemStages = NTOK <= 64 ? 3 : 4;   // 64 * kKps TMEM columns each
  static constexpr int kAccBufs = NTOK <= 128 ? 2 : 1;
  // Dequantizing warpgroups own alternate stages (the epilogue warpgroup
  // joins for tiles of <= 64 tokens).  Measured slower on B200 and dropped:
  // all twelve warps sharing every three-record stage of a 16/32-token tile.
  static constexpr int kDqGroups = NTOK <= 64 ? 3 : 2;
  static constexpr int kDqWarps = 4;  // arrivals on a TMEM stage's ready barrier
  // full barriers, one per (SMEM stage, dequant group): iteration `it`
  // uses barrier (it % SS, it % NDQ), so every waiter sees each of its
  // barrier's phases in order whatever the ring depth
  static constexpr int kFullBars = kSmemStages * kDqGroups;
  static constexpr int kFullPeriod = kSmemStages / cgcd(kSmemStages, kDqGroups) * kDqGroups;  // lcm
  // (kEpiScratch: the warp-local transpose buffer for 16-byte output
  // stores; at 256 tokens it aliases the expert tables, so grouped 256-token
  // tiles use 1 KB per warp after the tables, 16 tokens at a time, when the
  // tables take at most half of their area)
  // byte offsets from the 1024-aligned base of dynamic shared memory
  static constexpr size_t kBarOff = (size_t)kSmemStages * (kATile + kRecs);
  static constexpr size_t kTabOff = kBarOff + kBarBytes;                          // s_prefix, s_off
  static constexpr size_t kScrOff = (kTabOff + 2 * (kMaxExperts + 1) * sizeof(int) + 127) / 128 * 128;
  static constexpr size_t kSmem = 1024 + kScrOff + kEpiScratch;
  static_assert(kABlock % 1024 == 0 && kRecStride % 16 == 0 && kBarOff % 16 == 0, "stage alignment");
  static_assert(kEpiScratch != 0 || 2 * (kMaxExperts + 1) * sizeof(int) >= 4 * 2048, "aliased scratch size");
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(kSmemStages >= 2, "pipeline depth");
  static_assert(64 * kKps * kTmemStages + kAccBufs * NTOK <= 512, "TMEM budget");
  static_assert(kTmemStages % kDqGroups == 0, "every TMEM stage must always return to the same dequant group");
  static_assert(8 * (kFullBars + kSmemStages + 2 * kTmemStages + 5) + 16 <= kBarBytes, "barrier area");
};

// Weight row r of one 128-K packed record: its scale and zero point as
// bf16x2 pairs.  The fp16 scale s is split exactly into s_hi = bf16(s) and
// s_lo = s - s_hi (at most three significant bits, so bf16 holds it), and
// z2 = bf16(128 + z) twice (exact).
struct RowQ {
  uint32_t shi2, slo2, z2;
};
template <int CODE_BYTES, uint32_t ZSYM>
__device__ __forceinline__ RowQ row_qparams_t(const uint8_t* rec, int r, int has_zero) {
  const float s = __half2float(reinterpret_cast<const __half*>(rec + CODE_BYTES)[r]);
  const __nv_bfloat16 hi = __float2bfloat16_rn(s);
  const uint32_t hbits = (uint32_t)__bfloat16_as_ushort(hi);
  // s - s_hi is exact in fp32 and a bf16 number: no rounding here
  const uint32_t lbits = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(s - __bfloat162float(hi)));
  const uint32_t z = has_zero ? rec[CODE_BYTES + 256 + r] : ZSYM;
  const uint32_t zbits = 0x4300u + z;
  return RowQ{hbits | (hbits << 16), lbits | (lbits << 16), zbits | (zbits << 16)};
}
__device__ __forceinline__ RowQ row_qparams(const uint8_t* rec, int r, int has_zero) {
  return row_qparams_t<kW4RecCodes, 8u>(rec, r, has_zero);
}

// bf16x2 pair of bf16(128 + q) -> the weights (q - z) * s, each rounded to
// bf16 once: d = q - z is exact, d * s_lo is exact (at most 4 + 3
// significant bits), and the fused multiply-add rounds d * s_hi + d * s_lo
// = d * s a single time.
__device__ __forceinline__ uint32_t rescale(uint32_t x2, const RowQ& qp) {
  const uint32_t d = bf16x2_sub(x2, qp.z2);
  return bf16x2_fma(d, qp.shi2, bf16x2_mul(d, qp.slo2));
}

// One 32-K chunk of row r (16 bytes of codes) -> its weights w = (q - z) * s
// as 16 words, two bf16 per 32-bit word (even k in the low half).
__device__ __forceinline__ void dequant_chunk(const uint4& raw, const RowQ& qp, uint32_t* out) {
  const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // nibbles of k = 2j and 2j+1 sit at bits 4j and 16+4j: OR-ing them
      // into the mantissa of bf16 128.0 gives bf16(128 + q)
      const uint32_t x2 = lop3_and_or(wv[w] >> (4 * j), 0x000F000Fu, 0x43004300u);
      out[w * 4 + j] = rescale(x2, qp);
    }
  }
}

// A whole 128-K record for weight row r (thread lane of warp quarter q owns
// row r = 32q + lane, TMEM lane r, columns taddr .. taddr + 63): its 64 code
// bytes and the row's scale and zero point are read from shared memory
// first (one round trip), then each 32-K chunk is dequantized and stored.
__device__ __forceinline__ void dequant_block(const uint8_t* rec, int r, int has_zero, uint32_t taddr) {
  uint4 raw[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) raw[c] = *reinterpret_cast<const uint4*>(rec + (c * 128 + r) * 16);
  const RowQ qp = row_qparams(rec, r, has_zero);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t w[16];
    dequant_chunk(raw[c], qp, w);
    tmem_st_x16(taddr + c * 16, w);
  }
}

// ---- MXFP4 weights (e2m1 codes, E8M0 scale per 32 K)
//
// One 32-bit word of a chunk holds 4 pairs of codes (k even, k odd) with
// their bits placed by the packer so that, after a rotation (pairs 0-2) or
// two (pair 3), one mask leaves a bf16x2 word whose halves carry the sign at
// bit 15, the code's two exponent bits at 8..7 and its mantissa bit at 6:
// the bf16 value e2m1(c) * 2^-126 (the code 0.5 lands as the subnormal
// 2^-127, which bf16 arithmetic keeps).
__device__ __forceinline__ uint32_t rotr32(uint32_t x, int n) { return __funnelshift_r(x, x, n); }

__device__ __forceinline__ void mx_pairs(uint32_t w, uint32_t* o) {
  constexpr uint32_t kMask = 0x81C081C0u;
  o[0] = w & kMask;
  o[1] = rotr32(w, 4) & kMask;
  o[2] = rotr32(w, 10) & kMask;
  o[3] = (rotr32(w, 30) & 0x80C080C0u) | (rotr32(w, 6) & 0x01000100u);
}

// One 32-K chunk of row r -> 16 bf16x2 words w = e2m1(c) * 2^(e - 127),
// exact (scale bytes <= 252).  ONE_MUL: the scale is below 2^1, so a single
// multiply by bf16 2^(e - 1) suffices; otherwise the codes are first brought
// to their e2m1 values (times 2^126, exact) and then scaled by 2^(e - 127)
// (2^-127 is the bf16 subnormal 0x0040).
template <bool ONE_MUL>
__device__ __forceinline__ void mx_dequant_chunk(const uint4& raw, uint32_t e, uint32_t* out) {
  const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
  const uint32_t sbits = ONE_MUL ? (e + 126u) << 7 : (e ? e << 7 : 0x40u);
  const uint32_t s2 = sbits | (sbits << 16);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t o[4];
    mx_pairs(wv[w], o);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      out[w * 4 + j] = ONE_MUL ? bf16x2_mul(o[j], s2) : bf16x2_mul(bf16x2_mul(o[j], 0x7E807E80u), s2);
  }
}

template <bool ONE_MUL>
__device__ __forceinline__ void mx_dequant_chunks(const uint4* raw, uint32_t e4, uint32_t taddr) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t w[16];
    mx_dequant_chunk<ONE_MUL>(raw[c], (e4 >> (8 * c)) & 0xFFu, w);
    tmem_st_x16(taddr + c * 16, w);
  }
}

// A whole 128-K MXFP4 record for weight row r into TMEM (as dequant_block).
// The single-multiply path runs when every scale byte of the warp's 32 rows
// is below 128 (a warp-uniform choice; both paths give the same bits).
__device__ __forceinline__ void mx_dequant_block(const uint8_t* rec, int r, uint32_t taddr) {
  uint4 raw[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) raw[c] = *reinterpret_cast<const uint4*>(rec + (c * 128 + r) * 16);
  const uint32_t e4 = *reinterpret_cast<const uint32_t*>(rec + kW4RecCodes + 4 * r);
  if (__all_sync(0xffffffffu, (e4 & 0x80808080u) == 0u))
    mx_dequant_chunks<true>(raw, e4, taddr);
  else
    mx_dequant_chunks<false>(raw, e4, taddr);
}

// ---- INT3 weights (3-bit codes, fp16 scale and uint3 zero point per 128 K)
// A whole 128-K INT3 record for weight row r (as dequant_block): the row's
// 12 code words come in three 16-byte loads.  In each 32-K chunk (words
// 3c .. 3c+2) pairs 0-14 sit at bits 3j / 16 + 3j of their word, so one
// shift and one LOP3 give bf16 (128 + q, 128 + q'); pair 15 gathers code
// bit p from bits 15 / 31 of word p.  Then w = (q - z) * s as for INT4.
__device__ __forceinline__ void w3_dequant_block(const uint8_t* rec, int r, int has_zero, uint32_t taddr) {
  uint4 raw[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) raw[i] = *reinterpret_cast<const uint4*>(rec + (i * 128 + r) * 16);
  const uint32_t wv[12] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w, raw[1].x, raw[1].y,
                           raw[1].z, raw[1].w, raw[2].x, raw[2].y, raw[2].z, raw[2].w};
  const RowQ qp = row_qparams_t<kW3RecCodes, 4u>(rec, r, has_zero);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t out[16];
#pragma unroll
    for (int p = 0; p < 3; ++p) {
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        const uint32_t x2 = lop3_and_or(wv[3 * c + p] >> (3 * j), 0x00070007u, 0x43004300u);
        out[5 * p + j] = rescale(x2, qp);
      }
    }
    uint32_t x2 = lop3_and_or(wv[3 * c] >> 15, 0x00010001u, 0x43004300u);
    x2 = lop3_and_or(wv[3 * c + 1] >> 14, 0x00020002u, x2);
    x2 = lop3_and_or(wv[3 * c + 2] >> 13, 0x00040004u, x2);
    out[15] = rescale(x2, qp);
    tmem_st_x16(taddr + c * 16, out);
  }
}

// ---- INT2 weights (2-bit codes, fp16 scale and uint2 zero point per 128 K)
// A whole 128-K INT2 record for weight row r (as dequant_block): the row's
// 8 code words come in two 16-byte loads; pair i of 32-K chunk c sits at
// bits 2j / 16 + 2j (j = i % 8) of word 2c + i / 8, so one shift and one
// LOP3 give bf16 (128 + q, 128 + q'), then w = (q - z) * s as for INT4.
__device__ __forceinline__ void w2_dequant_block(const uint8_t* rec, int r, int has_zero, uint32_t taddr) {
  uint4 raw[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) raw[i] = *reinterpret_cast<const uint4*>(rec + (i * 128 + r) * 16);
  const uint32_t wv[8] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w, raw[1].x, raw[1].y, raw[1].z, raw[1].w};
  const RowQ qp = row_qparams_t<kW2RecCodes, 2u>(rec, r, has_zero);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t out[16];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t x2 = lop3_and_or(wv[2 * c + p] >> (2 * j), 0x00030003u, 0x43004300u);
        out[8 * p + j] = rescale(x2, qp);
      }
    }
    tmem_st_x16(taddr + c * 16, out);
  }
}

// ---- INT8 weights (8-bit codes, fp16 scale and uint8 zero point per 128 K)
// A whole 128-K INT8 record for weight row r (as dequant_block): eight
// 16-byte chunks of 16 codes; each code becomes q - z exactly in fp32, the
// product with the fp16 scale is exact in fp32 (8 + 11 significant bits),
// and the one rounding is the conversion to bf16.
__device__ __forceinline__ void w8_dequant_block(const uint8_t* rec, int r, int has_zero, uint32_t taddr) {
  const float s = __half2float(reinterpret_cast<const __half*>(rec + kW8RecCodes)[r]);
  const float zf = 8388608.f + (float)(has_zero ? rec[kW8RecCodes + 256 + r] : 128u);
#pragma unroll
  for (int c2 = 0; c2 < 4; ++c2) {
    uint32_t out[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 raw = *reinterpret_cast<const uint4*>(rec + ((2 * c2 + h) * 128 + r) * 16);
      const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        out[8 * h + 2 * w] = pack_bf16x2(u8_minus_zero(wv[w], 0, zf) * s, u8_minus_zero(wv[w], 1, zf) * s);
        out[8 * h + 2 * w + 1] = pack_bf16x2(u8_minus_zero(wv[w], 2, zf) * s, u8_minus_zero(wv[w], 3, zf) * s);
      }
    }
    tmem_st_x16(taddr + c2 * 16, out);
  }
}

// ---- MXINT4 weights (two's-complement 4-bit codes, E8M0 scale per 32 K)
// The INT4 nibble placement: flipping bit 3 of a code (the LOP3 XOR) maps
// the integer c in -8..7 to c + 8, so the bf16 pair is (136 + c, 136 + c');
// subtracting 136 and multiplying by 2^(e - 127) are exact (scale bytes
// <= 251 keep every weight finite; 2^-127 is the bf16 subnormal 0x0040).
__device__ __forceinline__ void mxi4_dequant_block(const uint8_t* rec, int r, uint32_t taddr) {
  uint4 raw[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) raw[c] = *reinterpret_cast<const uint4*>(rec + (c * 128 + r) * 16);
  const uint32_t e4 = *reinterpret_cast<const uint32_t*>(rec + kW4RecCodes + 4 * r);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t e = (e4 >> (8 * c)) & 0xFFu;
    const uint32_t sbits = e ? e << 7 : 0x40u;
    const uint32_t s2 = sbits | (sbits << 16);
    const uint32_t wv[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
    uint32_t out[16];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t x2 = lop3_and_xor(wv[w] >> (4 * j), 0x000F000Fu, 0x43084308u);
        out[w * 4 + j] = bf16x2_mul(bf16x2_sub(x2, 0x43084308u), s2);
      }
    }
    tmem_st_x16(taddr + c * 16, out);
  }
}

template <int NTOK, int FMT, bool SW, int CG>
__global__ void __launch_bounds__(kThreads, 1)
    w4a16_kernel(const __grid_constant__ CUtensorMap tmap_a, const W4Params p) {
  using C = Cfg<NTOK, FMT, CG>;
  constexpr int SS = C::kSmemStages;
  constexpr int TS = C::kTmemStages;
  constexpr int ACC = C::kAccBufs;
  constexpr int NDQ = C::kDqGroups;
  constexpr int kATile = C::kATile;
  constexpr int KPS = C::kKps;
  constexpr int kRecs = C::kRecs;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                               // SS * kATile (activations, 128-byte swizzle)
  uint8_t* sR = smem + SS * kATile;                 // SS * kRecs (packed weight records)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + C::kFullBars;
  uint64_t* aready = empty + SS;
  uint64_t* afree = aready + TS;
  uint64_t* acc_full = afree + TS;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_total = const_cast<int*>(s_abort + 1);
  // expert tables packed at the start of their area: [E + 1] each
  int* s_prefix = reinterpret_cast<int*>(smem + C::kTabOff);
  int* s_off = s_prefix + (p.grouped ? p.num_experts + 1 : kMaxExperts + 1);
  // 16-byte aligned: read back with 16-byte loads
  uint16_t* epi_scratch = reinterpret_cast<uint16_t*>(smem + (C::kEpiScratch ? C::kScrOff : C::kTabOff));
  // 256-token grouped tiles: 16-token transposes in the second half of the
  // table area, free when the tables take at most 4 KB (<= 511 experts)
  uint16_t* grouped_scratch =
      (C::kEpiScratch == 0 && p.grouped && 2 * (p.num_experts + 1) * (int)sizeof(int) <= 4096)
          ? reinterpret_cast<uint16_t*>(smem + C::kTabOff + 4096)
          : nullptr;
  auto full_bar = [&](uint32_t i) { return &full[(i % SS) * NDQ + (i % NDQ)]; };
  auto full_par = [](uint32_t i) { return (i / C::kFullPeriod) & 1; };

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  // CTA pairs: rank 0 issues the pair's MMAs; the dequantizing and epilogue
  // warps of both CTAs report to rank 0's barriers
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SS; ++s) mbar_init(&empty[s], 1);
    for (int f = 0; f < C::kFullBars; ++f) mbar_init(&full[f], 1);
    for (int t = 0; t < TS; ++t) {
      mbar_init(&aready[t], C::kDqWarps * CG);
      mbar_init(&afree[t], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4 * CG);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    *s_total = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_a);
  if (threadIdx.x == 0) pdl_launch_dependents();
  // Everything but the packed weights may be written by the previous kernel
  // on the stream: grouped mode needs the expert offsets at once
  if (p.grouped) {
    pdl_wait();
    grouped_tables<NTOK>(p, s_off, s_prefix, s_total);
  }
  if constexpr (CG == 2) {
    // the pair's TMEM is allocated by both CTAs together; barriers and the
    // allocation are visible to both CTAs after the cluster barrier
    if (warp == 2) {
      tmem_alloc_pair(s_tmem, 512);
      tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
  } else {
    __syncthreads();   // barriers (and the grouped tables) visible to every role
  }
  const int total_grouped = *s_total;

  auto a_col = [](int t) -> uint32_t { return (uint32_t)(t * 64 * KPS); };
  auto acc_col = [](int b) -> uint32_t { return (uint32_t)(64 * KPS * TS + b * NTOK); };

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
          // (pairs: this CTA's half of the token tile)
          const int arow = x.row0 + (int)rank * (NTOK / CG);
          for (int r = 0; r < nrec; ++r) {
            uint8_t* a_dst = sA + s * kATile + r * C::kABlock;
            tma_load_2d(a_dst, &tmap_a, (kb + r) * kBlockK, arow, fb);
            tma_load_2d(a_dst + NTOK / CG * 128, &tmap_a, (kb + r) * kBlockK + 64, arow, fb);
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
  if (CG == 1 && warp == 2) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  if (!p.grouped) pdl_wait();   // outputs, partials and counters may be in use by the previous kernel
  tc_fence_before();
  named_bar(1, kThreads - 32);
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp, elected lane issues)
    // one lane, fixed for the whole kernel, issues every MMA and commit: a
    // commit tracks the tcgen05 operations of the thread that issues it
    // (pairs: rank 0 only, for both CTAs)
    const bool leader = elect_one();
    uint32_t it = 0, uc = 0;
    bool ok = rank == 0;
    Unit x;
    for (int idx = 0; ok && get_unit<NTOK>(p, s_prefix, s_off, total_grouped, idx, x); ++idx, ++uc) {
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
      const uint32_t d_tmem = tmem_base + acc_col(ab);
      // the MMAs cover the unit's valid tokens, rounded up to 16 (a ragged
      // tile of an expert or of the last token rows costs no more tensor
      // work than it needs); accumulator columns past them are never stored.
      // A pair's MMA takes each CTA's half of the tile at a fixed place, so
      // it always covers the whole tile.
      const uint32_t idesc = CG == 2 ? idesc_bf16_f32(256, (uint32_t)NTOK)
                                     : idesc_bf16_f32(128, (uint32_t)min(NTOK, (x.rows + 15) & ~15));
      for (int kb = x.kb0; kb < x.kb1; kb += KPS, ++it) {
        const int s = it % SS, t = it % TS;
        const uint32_t ph_t = (it / TS) & 1;
        const int nrec = min(KPS, x.kb1 - kb);
        // weights of both CTAs in TMEM (their dequantizing warps waited for
        // their own stage, records and activations alike), this CTA's stage
        const bool ready = CG == 2 ? (hq_wait_warp_cl(&aready[t], ph_t, p.wait_ns, s_abort) &&
                                      hq_wait_warp(full_bar(it), full_par(it), p.wait_ns, s_abort))
                                   : hq_wait_warp_n(2, &aready[t], ph_t, full_bar(it), full_par(it), nullptr, 0,
                                                    p.wait_ns, s_abort);
        if (!ready) {
          if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
          // descriptors advance by constants: 32 B per 16-K step inside a
          // 128-byte swizzle row, one box (NTOK rows) per 64 K.  Only the low
          // word moves (its 14-bit start-address field cannot overflow inside
          // shared memory), so each MMA costs one 32-bit add.
          const uint64_t b0 = smem_desc_sw128(smem_u32(sA + s * kATile));
          const uint32_t blo = (uint32_t)b0, bhi = (uint32_t)(b0 >> 32);
          const uint32_t a0 = tmem_base + a_col(t);
          const uint32_t acc0 = kb > x.kb0 ? 1u : 0u;
#pragma unroll
          for (int r = 0; r < KPS; ++r) {
            if (r < nrec) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const uint32_t off = (uint32_t)((r * C::kABlock + (j >> 2) * (NTOK / CG * 128) + (j & 3) * 32) >> 4);
                const uint64_t bdesc = ((uint64_t)bhi << 32) | (uint64_t)(blo + off);
                if constexpr (CG == 2)
                  mma_bf16_ts_pair(d_tmem, a0 + r * 64 + j * 8, bdesc, idesc, (r > 0 || j > 0) ? 1u : acc0);
                else
                  mma_bf16_ts(d_tmem, a0 + r * 64 + j * 8, bdesc, idesc, (r > 0 || j > 0) ? 1u : acc0);
              }
            }
          }
          // (pairs: both CTAs' stage slots and weight slots)
          if constexpr (CG == 2) {
            tc_commit_pair(&empty[s]);
            tc_commit_pair(&afree[t]);
          } else {
            tc_commit(&empty[s]);
            tc_commit(&afree[t]);
          }
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
    // make sure no MMA is still running when TMEM is released
    if (leader && rank == 0) {
      if constexpr (CG == 2)
        tc_commit_pair_local(drain);
      else
        tc_commit(drain);
      hq_wait(drain, 0, p.wait_ns, nullptr);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dequantize (+ epilogue in warps 4-7)
    const uint32_t q = warp & 3;
    const int r = (int)(q * 32 + lane);              // weight row within the tile
    const uint32_t lane_addr = (q * 32) << 16;
    const bool epi = warp < 8;
    // dequant group index (2: the epilogue warps)
    const int dq = warp >= 12 ? 1 : warp >= 8 ? 0 : 2;
    const bool does_dq = dq < NDQ;
    uint32_t it = 0, uc = 0;
    bool ok = true;
    Unit x, pend;          // pend: the split tile this CTA reduces after its last unit
    bool has_pend = false;
    for (int idx = 0; ok && get_unit<NTOK>(p, s_prefix, s_off, total_grouped, idx, x); ++idx, ++uc) {
      for (int kb = x.kb0; kb < x.kb1; kb += KPS, ++it) {
        if (!does_dq || (int)(it % NDQ) != dq) continue;
        const int nrec = min(KPS, x.kb1 - kb);
        const int s = it % SS, t = it % TS;
        const uint32_t ph_t = (it / TS) & 1;
        // The full barrier of (stage, group) and TMEM stage t (TS % NDQ == 0)
        // only ever serve this group, so it observes every phase of the
        // barriers it waits on, one after the other (a parity wait can only
        // tell adjacent phases apart).
        // (Dequantizing the first half-record into registers before the TMEM
        // stage is known to be free measured slower: the busier dequant warps
        // take issue slots from the MMA warp on the same sub-partition.)
        if (!hq_wait_warp_n(2, full_bar(it), full_par(it), &afree[t], ph_t ^ 1, nullptr, 0, p.wait_ns, s_abort)) {
          if (lane == 0) raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        const uint32_t tbase = tmem_base + lane_addr + a_col(t);
        tc_fence_after();
        for (int rr = 0; rr < nrec; ++rr) {
          if constexpr (FMT == kFmtMx)
            mx_dequant_block(sR + s * kRecs + rr * p.rec_bytes, r, tbase + rr * 64);
          else if constexpr (FMT == kFmtMxi4)
            mxi4_dequant_block(sR + s * kRecs + rr * p.rec_bytes, r, tbase + rr * 64);
          else if constexpr (FMT == kFmtInt8)
            w8_dequant_block(sR + s * kRecs + rr * p.rec_bytes, r, p.has_zero, tbase + rr * 64);
          else if constexpr (FMT == kFmtInt3)
            w3_dequant_block(sR + s * kRecs + rr * p.rec_bytes, r, p.has_zero, tbase + rr * 64);
          else if constexpr (FMT == kFmtInt2)
            w2_dequant_block(sR + s * kRecs + rr * p.rec_bytes, r, p.has_zero, tbase + rr * 64);
          else
            dequant_block(sR + s * kRecs + rr * p.rec_bytes, r, p.has_zero, tbase + rr * 64);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          // (pairs: the MMA issuer is rank 0's)
          if constexpr (CG == 2)
            mbar_arrive_cluster(mapa_u32(&aready[t], 0));
          else
            mbar_arrive(&aready[t]);
        }
      }
      if (!ok || !epi) continue;

      // ---- epilogue of this unit (warps 4-7)
      const int ab = uc % ACC;
      const uint32_t aph = (uc / ACC) & 1;
      if (!hq_wait(&acc_full[ab], aph, p.wait_ns, s_abort)) {
        raise_error(p.err, s_abort, HQ_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      float* part = x.partial ? p.partials + ((size_t)blockIdx.x * 2 + x.slot) * NTOK * kTileN : nullptr;
      // batched TMEM loads (EB columns), then fp32 partials or bf16 stores
      constexpr int EB = NTOK >= 32 ? 32 : 16;
      if (C::kEpiScratch == 0 && p.grouped) {
        // 256-token grouped tiles: 16 tokens per batch through the 1 KB
        // transposes after the expert tables (element by element when the
        // tables leave no room)
        uint16_t* sc = grouped_scratch ? grouped_scratch + q * 512 : nullptr;
#pragma unroll 1
        for (int j0 = 0; j0 < NTOK; j0 += 16) {
          uint32_t v0[16];
          tmem_ld_x16(tmem_base + lane_addr + acc_col(ab) + j0, v0);
          tmem_wait_ld();
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(v0[j]);
          store_chunk<16, SW>(p, x, part, (int)q, (int)lane, j0, v, sc);
        }
      } else {
        uint16_t* sc = epi_scratch + q * 1024;
#pragma unroll 1
        for (int j0 = 0; j0 < NTOK; j0 += EB) {
          uint32_t v0[16], v1[16];
          tmem_ld_x16(tmem_base + lane_addr + acc_col(ab) + j0, v0);
          if (EB == 32) tmem_ld_x16(tmem_base + lane_addr + acc_col(ab) + j0 + 16, v1);
          tmem_wait_ld();
          float v[EB];
#pragma unroll
          for (int j = 0; j < EB; ++j) v[j] = __uint_as_float(j < 16 ? v0[j] : v1[j - 16]);
          store_chunk<EB, SW>(p, x, part, (int)q, (int)lane, j0, v, sc);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (CG == 2)
          mbar_arrive_cluster(mapa_u32(&acc_empty[ab], 0));
        else
          mbar_arrive(&acc_empty[ab]);
      }
      if (sk_is_reducer(p, x)) {
        pend = x;
        has_pend = true;
      } else if (x.partial) {
        sk_signal(p, x, (int)q, (int)lane);
      }
    }
    if (ok && has_pend) sk_reduce<NTOK>(p, pend, (int)q, (int)lane);
  }

  }  // non-producer roles

  tc_fence_before();
  __syncthreads();
  // a pair's CTAs leave together: rank 0's MMAs read the other CTA's shared
  // memory and TMEM until rank 0 has drained them
  if constexpr (CG == 2) cluster_sync();
  tc_fence_after();
  if (warp == 2) {
    if constexpr (CG == 2)
      tmem_dealloc_pair(*s_tmem, 512);
    else
      tmem_dealloc(*s_tmem, 512);
  }
}

template <int NTOK, int FMT, bool SW, int CG>
bool smem_attr() {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && attr_set[dev]) return true;
  if (cudaFuncSetAttribute(w4a16_kernel<NTOK, FMT, SW, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Cfg<NTOK, FMT, CG>::kSmem) != cudaSuccess)
    return false;
  if (dev < 64) attr_set[dev] = true;
  return true;
}

template <int NTOK, int FMT, bool SW, int CG = 1>
hq_status launch_t(const CUtensorMap& map, const W4Params& p, int grid, cudaStream_t stream) {
  auto kern = w4a16_kernel<NTOK, FMT, SW, CG>;
  const size_t smem = Cfg<NTOK, FMT, CG>::kSmem;
  if (!smem_attr<NTOK, FMT, SW, CG>()) return HQ_ERR_CUDA;
  const cudaError_t e = CG == 2 ? launch_pdl_pairs(kern, dim3(grid), dim3(kThreads), smem, stream, map, p)
                                : launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, map, p);
  return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

// Clusters of two of the CTA-pair kernel resident at once (0 when the query
// fails), per device.
template <int FMT>
int pair_slots_t() {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  if (!smem_attr<256, FMT, false, 2>()) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg<256, FMT, 2>::kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, w4a16_kernel<256, FMT, false, 2>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev < 64) cached[dev] = n;
  return n;
}

// One format's launch for a token tile, with or without the SwiGLU epilogue.
template <int FMT, bool SW>
hq_status launch_tiles(int ntok, const CUtensorMap& map, const W4Params& p, int grid, cudaStream_t stream) {
  switch (ntok) {
    case 16: return launch_t<16, FMT, SW>(map, p, grid, stream);
    case 32: return launch_t<32, FMT, SW>(map, p, grid, stream);
    case 64: return launch_t<64, FMT, SW>(map, p, grid, stream);
    case 128: return launch_t<128, FMT, SW>(map, p, grid, stream);
    case 256: return launch_t<256, FMT, SW>(map, p, grid, stream);
    default: return HQ_ERR_UNSUPPORTED;
  }
}
template <int FMT>
hq_status launch_fmt(int ntok, bool swiglu, bool pairs, const CUtensorMap& map, const W4Params& p, int grid,
                     cudaStream_t stream) {
  if (pairs) return ntok == 256 && !swiglu ? launch_t<256, FMT, false, 2>(map, p, grid, stream) : HQ_ERR_UNSUPPORTED;
  return swiglu ? launch_tiles<FMT, true>(ntok, map, p, grid, stream)
                : launch_tiles<FMT, false>(ntok, map, p, grid, stream);
}

int pair_slots(int kfmt) {
  switch (kfmt) {
    case kFmtMx: return pair_slots_t<kFmtMx>();
    case kFmtMxi4: return pair_slots_t<kFmtMxi4>();
    case kFmtInt3: return pair_slots_t<kFmtInt3>();
    case kFmtInt2: return pair_slots_t<kFmtInt2>();
    case kFmtInt8: return pair_slots_t<kFmtInt8>();
    default: return pair_slots_t<kFmtInt4>();
  }
}
int kernel_fmt(const hq_quant_desc& d) {
  return d.fmt == HQ_FMT_MXFP4_A16 ? kFmtMx : d.fmt == HQ_FMT_MXINT4 ? kFmtMxi4 : d.fmt == HQ_FMT_INT3 ? kFmtInt3
         : d.fmt == HQ_FMT_INT2 ? kFmtInt2 : d.fmt == HQ_FMT_INT8 ? kFmtInt8 : kFmtInt4;
}

int dense_tiles(const hq_quant_desc& d, int m, int ntok) {
  return ((d.n + kTileN - 1) / kTileN) * ((m + ntok - 1) / ntok);
}

}  // namespace

namespace {
W4Config w4_plan_rules(const DeviceInfo& dev, const hq_quant_desc& d, int m, bool grouped, const hq_tuning* t) {
  W4Config cfg{};
  // no tuning from the caller: the caller's per-shape table first, then the rules below
  hq_tuning from_table;
  if (!t) t = tuning_from_table(d, m, &from_table);
  int ntok = (t && t->tile_m) ? t->tile_m : 0;
  if (!ntok) {
    if (grouped) {
      // A typical expert's rows should fit one token tile: an expert split
      // over two tiles streams its weights twice, while a larger tile costs
      // little more at these sizes (HBM bound).  Top-k routing gives about
      // Poisson(avg) rows per expert, so the tile covers avg + 2 sd.
      const double avg = (double)m / std::max(1, d.num_experts);
      const double want = avg + 2.0 * std::sqrt(avg);
      // 256-token tiles for long K ranges only, and only where their output
      // transposes fit beside the expert tables (at most 511 experts).
      // Measured on B200, T=8192 top-8 over 256 experts: gate+up (K=7168)
      // with the fused SwiGLU 4571 us at 128 tokens, 4157 at 256; down
      // (K=2048, 16 k-blocks per unit, whose single 256-token accumulator
      // leaves the epilogue unoverlapped) 2337 at 128, 2399 at 256.
      ntok = want <= 16 ? 16 : want <= 32 ? 32 : want <= 64 ? 64
           : (want > 192 && d.k >= 4096 && d.num_experts <= 511) ? 256 : 128;
    } else {
      ntok = m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : m <= 128 ? 128 : 256;
    }
  }
  cfg.stages = t ? t->stages : 0;
  cfg.splits = 1;
  cfg.cta_group = 1;
  cfg.variant = t ? t->variant : 0;
  cfg.early_weights = (t && (t->flags & HQ_TUNE_NO_EARLY_WEIGHTS)) ? 0 : 1;
  // The register-path kernel: dense INT4 at 1..16 tokens, the library's
  // choice there and on request (variant 3); a request that does not apply
  // (more tokens, another format, MoE) gets the library's choice.  Measured
  // on B200 (per launch, back to back): K=7168 N=18432 M <= 8 20.8 us, M=16
  // 24.8, against 24.5 and 25.0 for the exact-weight kernel; K=18432 N=7168
  // M <= 8 22.9, M=16 26.0, against 30.2 and 32.7.
  const bool reg_fits = !grouped && d.fmt == HQ_FMT_INT4 && m <= 16 && ntok <= 16 && !(t && t->cta_group == 2);
  if (cfg.variant == 3 && !reg_fits && !grouped) cfg.variant = 0;
  const bool use_reg = reg_fits && (cfg.variant == 0 || cfg.variant == 3);
  if (use_reg) {
    const long long tiles = (d.n + kTileN - 1) / kTileN;
    cfg.variant = 3;
    cfg.ntok = m <= 8 ? 8 : 16;   // one or two 8-token MMA tiles
    cfg.dp_tiles = 0;
    cfg.splits = (t && t->split_k > 0) ? (int)std::min<long long>(t->split_k, d.k / kBlockK)
                                       : reg_splits(dev.num_sms, d, m);
    cfg.grid = (int)(tiles * cfg.splits);
    // Grids of fewer CTAs than SMs run eight warps of 16 rows per CTA (more
    // warps on each busy SM): M=16 K=N=1024 (64 CTAs) 8.4 -> 6.5 us on B200;
    // full grids keep four warps of 32 rows (the activations read once per
    // 32 rows; eight warps of 16 rows measured 1-40 % slower there).
    cfg.reg_tw = cfg.grid < dev.num_sms ? 1 : 2;
    return cfg;
  }
  if (grouped) {
    // The register path for INT4 experts of a few tokens each, on request
    // (variant 3) or by default when a typical expert's rows fit 8 tokens:
    // 8- or 16-token units over the whole K range on persistent CTAs.
    // Measured on B200 (256 experts, top-8, hidden 7168, intermediate 2048):
    // T=64 gate+up 778 us and down 419 against 868 and 452 for the
    // exact-weight grouped kernel; T=1024 (32 rows per expert) three times
    // slower, so only the few-token case takes it.
    const double avg = (double)m / std::max(1, d.num_experts);
    const double want = avg + 2.0 * std::sqrt(avg);
    const bool reg_ok = d.fmt == HQ_FMT_INT4 && d.num_experts <= kMaxExperts && !(t && t->cta_group == 2) &&
                        !(t && t->tile_m && t->tile_m != 8 && t->tile_m != 16);
    if (reg_ok && (cfg.variant == 3 || (cfg.variant == 0 && kRegGroupedDefault && want <= 8.0))) {
      cfg.variant = 3;
      cfg.ntok = (t && t->tile_m) ? t->tile_m : want <= 8.0 ? 8 : 16;
      cfg.splits = 0;
      cfg.grid = dev.num_sms * reg_grouped_ctas_per_sm(cfg.ntok / 8);
      cfg.reg_tw = 2;
      return cfg;
    }
    if (cfg.variant == 3) cfg.variant = 0;
    cfg.ntok = ntok;
    cfg.grid = dev.num_sms;
    return cfg;
  }
  if (t && t->cta_group == 2) {
    // CTA pairs on request: 256-token whole tiles, one per resident cluster
    // at a time
    cfg.ntok = 256;
    cfg.splits = 0;
    cfg.cta_group = 2;
    const long long pair_tiles = (long long)dense_tiles(d, m, 256) / 2;
    const long long slots = pair_slots(kernel_fmt(d));
    cfg.grid = (int)(2 * std::max<long long>(1, std::min<long long>(slots > 0 ? slots : dev.num_sms / 2, pair_tiles)));
    return cfg;
  }
  // Whole tiles on persistent CTAs (no partial sums) when they fill the SMs
  // well (a 256-token tile may drop to 128 for that).  Otherwise the K range
  // is shared: large token tiles (big partial sums) split every tile into
  // the same number of parts when that fills the SMs; everything else uses
  // stream-K over all SMs (every CTA an equal share of the (tile, k-block)
  // space, >= 4 k-blocks each).
  auto dp_eff = [&](int nt) {
    const long long tl = dense_tiles(d, m, nt);
    const long long waves = (tl + dev.num_sms - 1) / dev.num_sms;
    return (double)tl / (double)(waves * dev.num_sms);
  };
  const long long kbs = d.k / kBlockK;
  if (t && t->split_k > 0) {
    // explicit request: `split_k` CTAs per tile
    const long long tiles = dense_tiles(d, m, ntok);
    cfg.ntok = ntok;
    cfg.splits = t->split_k;
    cfg.grid = (int)std::max<long long>(1, std::min<long long>(tiles * t->split_k, tiles * kbs));
    return cfg;
  }
  // Large tiles keep whole tiles down to 70 % of the SMs busy: their
  // partial sums are big, and measured, whole tiles beat a shared K range
  // there (M=256, K=18432, N=7168: 128-token whole tiles on 112 SMs take
  // 84 us, stream-K over 148 SMs 101 us, a 256-token 2-way split 104 us).
  const bool fixed_tile = t && t->tile_m;
  const double dp_min = ntok >= 128 ? 0.7 : 0.85;
  if (!fixed_tile && ntok == 256 && dp_eff(256) < dp_min && dp_eff(128) >= dp_min) ntok = 128;
  cfg.ntok = ntok;
  const long long tiles = dense_tiles(d, m, ntok);
  if (dp_eff(ntok) >= dp_min) {
    const long long waves = tiles / dev.num_sms, rest = tiles % dev.num_sms;
    // CTA pairs: 256-token whole tiles of 256-row weight tiles, one pair
    // tile per resident cluster at a time
    // (used for 256-token tiles whose single-CTA ring is shallow, below)
    auto use_pairs = [&](long long tiles_) {
      const long long pair_tiles = tiles_ / 2;
      const long long slots = pair_slots(kernel_fmt(d));
      if (slots <= 0) return false;
      cfg.cta_group = 2;
      cfg.splits = 0;
      cfg.dp_tiles = 0;
      cfg.grid = (int)(2 * std::min<long long>(slots, pair_tiles));
      return true;
    };
    // CTA pairs (half the activation tile per CTA, a deeper ring) only where
    // one CTA's ring holds fewer than 3 stages: INT8 records (16.8 KB) leave
    // room for 2 at 256 tokens, pairs hold 4 (M=4096 K=7168 N=18432
    // 1175 -> 1075 us, M=1024 308 -> 272 us on B200).  With 3 stages one CTA
    // per tile wins (INT4 M=4096 815 us against 881 on pairs): each record
    // waits for both CTAs' dequantization and one SM issues both SMs' MMAs.
    if (ntok == 256 && d.n % 256 == 0 && w4_ring_depth(d, cfg) < 3 && !(t && t->cta_group == 1) && use_pairs(tiles))
      return cfg;
    if (waves >= 2 && rest != 0 && dp_eff(ntok) < 0.95) {
      // Whole tiles for all waves but the last full one; that wave and the
      // ragged rest share their K range stream-K style (every CTA one to two
      // tiles' worth, each tile split over at most three CTAs), so no SM
      // idles through a mostly empty last wave.  Measured: M=4096, K=18432,
      // N=7168 (896 tiles = 6 waves + 8) 831 -> 799 us.  Not with a single
      // full wave (M=1024, K=18432: 224 tiles, 232 -> 238 us): under the
      // power cap the SMs of a part-empty last wave run at higher clocks,
      // and the shared K range pays for partial sums.
      cfg.splits = 1;
      cfg.dp_tiles = (int)((waves - 1) * dev.num_sms);
      cfg.grid = dev.num_sms;
      return cfg;
    }
    cfg.splits = 0;  // data parallel
    cfg.grid = (int)std::min<long long>(dev.num_sms, tiles);
    return cfg;
  }
  if (ntok >= 128 && tiles * 2 <= dev.num_sms && tiles * (dev.num_sms / tiles) >= 0.85 * dev.num_sms) {
    cfg.splits = (int)(dev.num_sms / tiles);
    cfg.grid = (int)std::min<long long>(tiles * cfg.splits, tiles * kbs);
    return cfg;
  }
  cfg.splits = 1;
  cfg.grid = (int)std::max<long long>(1, std::min<long long>(dev.num_sms, tiles * kbs / 4));
  return cfg;
}
}  // namespace

W4Config w4_plan(const DeviceInfo& dev, const hq_quant_desc& d, int m, bool grouped, const hq_tuning* t) {
  W4Config cfg = w4_plan_rules(dev, d, m, grouped, t);
  // four tile counters per output tile, in the workspace's fixed counter region
  if (!grouped && cfg.splits != 0 && (size_t)dense_tiles(d, m, cfg.ntok) * 4 * sizeof(int32_t) > kWsCounterBytes &&
      !(cfg.variant == 3 && cfg.splits == 1))
    cfg = w4_whole_tiles(dev, d, m, cfg);
  return cfg;
}

namespace {
template <int FMT>
int rescaled_depth(int ntok, int cta_group) {
  if (cta_group == 2) return Cfg<256, FMT, 2>::kSmemStages;
  switch (ntok) {
    case 16: return Cfg<16, FMT>::kSmemStages;
    case 32: return Cfg<32, FMT>::kSmemStages;
    case 64: return Cfg<64, FMT>::kSmemStages;
    case 128: return Cfg<128, FMT>::kSmemStages;
    default: return Cfg<256, FMT>::kSmemStages;
  }
}
}  // namespace

int w4_ring_depth(const hq_quant_desc& d, const W4Config& cfg) {
  if (cfg.variant == 3) return cfg.ntok == 8 ? kRegRing8 : kRegRing16;   // the register path's ring of whole-record stages
  const bool mx = d.fmt == HQ_FMT_MXFP4_A16, mxi4 = d.fmt == HQ_FMT_MXINT4;
  const int kfmt = d.fmt == HQ_FMT_INT3 ? kFmtInt3 : d.fmt == HQ_FMT_INT2 ? kFmtInt2 : d.fmt == HQ_FMT_INT8 ? kFmtInt8 : kFmtInt4;
  if (!mx && !mxi4 && cfg.ntok <= 64 && cfg.variant != 1) return small_ring_depth(cfg.ntok, kfmt);
  if (mx) return rescaled_depth<kFmtMx>(cfg.ntok, cfg.cta_group);
  if (mxi4) return rescaled_depth<kFmtMxi4>(cfg.ntok, cfg.cta_group);
  switch (kfmt) {
    case kFmtInt3: return rescaled_depth<kFmtInt3>(cfg.ntok, cfg.cta_group);
    case kFmtInt2: return rescaled_depth<kFmtInt2>(cfg.ntok, cfg.cta_group);
    case kFmtInt8: return rescaled_depth<kFmtInt8>(cfg.ntok, cfg.cta_group);
    default: return rescaled_depth<kFmtInt4>(cfg.ntok, cfg.cta_group);
  }
}

W4Config w4_whole_tiles(const DeviceInfo& dev, const hq_quant_desc& d, int m, W4Config cfg) {
  if (cfg.variant == 3) {
    // register path: one CTA per weight tile over the whole K range
    cfg.splits = 1;
    cfg.grid = (d.n + kTileN - 1) / kTileN;
    cfg.reg_tw = cfg.grid < dev.num_sms ? 1 : 2;
    return cfg;
  }
  cfg.splits = 0;
  cfg.dp_tiles = 0;
  cfg.cta_group = 1;
  cfg.grid = (int)std::min<long long>(dev.num_sms, dense_tiles(d, m, cfg.ntok));
  return cfg;
}

size_t w4_workspace_bytes(const hq_quant_desc& d, int m, const W4Config& cfg, bool grouped) {
  if (!grouped && cfg.variant == 3) return reg_workspace_bytes(cfg);
  size_t bytes = sizeof(WsHeader);
  if (grouped) return bytes;
  if (cfg.splits == 0) return bytes;  // data parallel: no partial sums
  bytes += kWsCounterBytes;                                                     // counters, 4 per tile (fixed region)
  bytes += (size_t)cfg.grid * 2 * cfg.ntok * kTileN * sizeof(float);            // partial tiles, 2 per CTA
  return bytes;
}

hq_status w4_launch(const hq_quant_desc& d, const W4Config& cfg, const void* packed, const void* a, int m,
                    void* c, const int32_t* expert_offsets, void* ws, cudaStream_t stream, int swiglu) {
  const bool grouped = expert_offsets != nullptr;
  if (!grouped && cfg.variant == 3) return reg_launch(d, cfg, packed, a, m, c, ws, stream);
  if (grouped && cfg.variant == 3) return reg_launch_grouped(d, cfg, packed, a, m, c, expert_offsets, ws, stream, swiglu);
  W4Params p{};
  p.packed = static_cast<const uint8_t*>(packed);
  p.c = static_cast<__nv_bfloat16*>(c);
  p.expert_offsets = expert_offsets;
  p.err = static_cast<uint32_t*>(ws);
  const bool mx = d.fmt == HQ_FMT_MXFP4_A16;
  const bool mxi4 = d.fmt == HQ_FMT_MXINT4;
  const bool int3 = d.fmt == HQ_FMT_INT3;
  const bool int2 = d.fmt == HQ_FMT_INT2;
  const bool int8 = d.fmt == HQ_FMT_INT8;
  p.has_zero = d.has_zero_point ? 1 : 0;
  p.rec_bytes = mx     ? kMxA16RecBytes
                : mxi4 ? kMxi4RecBytes
                : int3 ? w3_record_bytes(p.has_zero)
                : int2 ? w2_record_bytes(p.has_zero)
                : int8 ? w8_record_bytes(p.has_zero)
                       : w4_record_bytes(p.has_zero);
  p.n_tiles = (d.n + kTileN - 1) / kTileN;
  p.k_blocks = d.k / kBlockK;
  p.expert_bytes = (uint64_t)p.n_tiles * p.k_blocks * p.rec_bytes;
  p.m = m;
  p.n = d.n;
  p.m_tiles = (m + cfg.ntok - 1) / cfg.ntok;
  p.num_experts = grouped ? d.num_experts : 1;
  p.grouped = grouped ? 1 : 0;
  p.wait_ns = kDefaultWaitNs;
  p.early_weights = cfg.early_weights;
  p.stage_limit = cfg.stages;
  p.cta_pairs = cfg.cta_group == 2 ? 1 : 0;
  p.n_pairs = p.n_tiles / 2;
  if (grouped) {
    // an expert's weight tile is re-read by each of its token tiles
    p.weights_once = (long long)m <= (long long)cfg.ntok * d.num_experts ? 1 : 0;
  } else {
    const size_t tiles = (size_t)dense_tiles(d, m, cfg.ntok);
    p.dp_tiles = cfg.splits == 0 ? 0 : cfg.dp_tiles;
    p.total_iters = (long long)(tiles - (size_t)p.dp_tiles) * p.k_blocks;
    p.weights_once = p.m_tiles == 1 ? 1 : 0;
    p.data_parallel = cfg.splits == 0 ? 1 : 0;
    uint8_t* base = static_cast<uint8_t*>(ws) + sizeof(WsHeader);
    p.counters = reinterpret_cast<int32_t*>(base);
    p.partials = reinterpret_cast<float*>(base + kWsCounterBytes);
  }

  // Activations: bf16 [rows][K], boxes of 64 K x NTOK rows, 128-byte swizzle.
  CUtensorMap map;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return HQ_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)d.k, (cuuint64_t)m};
  cuuint64_t strides[1] = {(cuuint64_t)d.k * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)(cfg.cta_group == 2 ? cfg.ntok / 2 : cfg.ntok)};   // pairs: half a tile
  cuuint32_t estr[2] = {1, 1};
  CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return HQ_ERR_CUDA;

  // The exact-weight kernel for tiles of up to 64 tokens (INT4, INT3, INT2
  // and INT8 weights): the library's choice there, and on request; the
  // bf16-rescaled kernel for larger tiles, for the MX formats (exact in
  // bf16 already) and on request (variant 1).
  const int kfmt = int3 ? kFmtInt3 : int2 ? kFmtInt2 : int8 ? kFmtInt8 : kFmtInt4;
  const bool exact = !mx && !mxi4 && cfg.ntok <= 64 && cfg.variant != 1;
  if (exact) return small_launch(cfg.ntok, kfmt, swiglu != 0, map, p, cfg.grid, stream);
  const bool sw = swiglu != 0;
  const bool pr = cfg.cta_group == 2;
  if (mx) return launch_fmt<kFmtMx>(cfg.ntok, sw, pr, map, p, cfg.grid, stream);
  if (mxi4) return launch_fmt<kFmtMxi4>(cfg.ntok, sw, pr, map, p, cfg.grid, stream);
  if (int8) return launch_fmt<kFmtInt8>(cfg.ntok, sw, pr, map, p, cfg.grid, stream);
  if (int3) return launch_fmt<kFmtInt3>(cfg.ntok, sw, pr, map, p, cfg.grid, stream);
  if (int2) return launch_fmt<kFmtInt2>(cfg.ntok, sw, pr, map, p, cfg.grid, stream);
  return launch_fmt<kFmtInt4>(cfg.ntok, sw, pr, map, p, cfg.grid, stream);
}

}  // namespace hq
