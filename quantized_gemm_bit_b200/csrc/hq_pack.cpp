// Offline weight packer: canonical (code, scale, zero point) tensors -> the
// device layout the kernels read.  Host memory in, host memory out.
//
// The method keeps weight, scale and zero point as separately described
// parts of one standard quantization description ("Humming: open-source
// kernel library for quantized inference", summary paragraph 2); this file
// fixes how those parts sit in device memory for the B200 kernels.
//
// Packed layouts, version 1 (NP = N rounded up to a multiple of 128; rows
// >= N are zero-filled):
//
// INT4 (group 128).  One record per (tile nt of 128 rows, block kb of 128 K),
// records in (nt, kb) order, expert after expert.  Record bytes:
//   [0, 8192)      codes: for row r, K-chunk c = kk/32, word w = (kk%32)/8,
//                  element e = kk%8: byte (c*128 + r)*16 + 4*w holds the
//                  32-bit word whose nibble p = (e%2)*4 + e/2 is the code.
//                  (A thread owning row r reads 16 contiguous bytes per
//                  chunk; nibbles k, k+1 share one 16-bit lane pair.)
//   [8192, 8448)   fp16 scale of row r at 8192 + 2r
//   [8448, 8576)   uint4 zero point of row r at 8448 + r (asymmetric only)
//
// MXFP4 (E8M0 scale per 32 K).
//   codes : [NP][K/2] bytes, row major, even k in the low nibble
//   scales: from byte NP*K/2, one 512-byte block per (tile nt, 128-K group
//           g) in (nt, g) order; byte l*16 + 4*c + j holds the scale of row
//           nt*128 + l + 32*c for the 32-K block 4*g + j (l < 32, c < 4,
//           j < 4).  This is the order tcgen05.cp 32x128b.warpx4 expects.
//
// NVFP4 (E4M3 scale per 16 K, fp32 tensor scale).
//   codes : [NP][K/2] bytes as for MXFP4
//   scales: from byte NP*K/2, one 512-byte block per (tile nt, 64-K group g)
//           in (nt, g) order; byte l*16 + 4*c + j = scale of row
//           nt*128 + l + 32*c for the 16-K block 4*g + j
//   tail  : 16 bytes; the fp32 tensor scale in the first 4.
//
// MXFP4 for bf16 activations (MXFP4_A16: the W4A16 kernels dequantize it).
// Records as for INT4 (one per (tile nt, 128-K block kb), experts one after
// another), 8192 + 512 bytes each:
//   [0, 8192)      codes: the 32-bit word at byte (c*128 + r)*16 + 4*w holds
//                  the 8 codes kk = 32c + 8w + 2j + h (pair j < 4, half
//                  h < 2); bit b of a code (0 mantissa, 1-2 exponent, 3
//                  sign) sits at word bit kMxBits[j][h][b].
//   [8192, 8704)   E8M0 scale of row r, 32-K block c at 8192 + 4r + c.
// (The INT3 layout follows below.)
// The bit positions are chosen so that pair j's two codes land, after the
// kernel rotates the word right by 0, 4 or 10 bits (j = 0, 1, 2) or merges
// two rotations (j = 3), on the bits a bf16x2 word gives its sign (15), the
// low two exponent bits (8..7) and the top mantissa bit (6): one mask per
// pair then leaves two bf16 values e2m1 * 2^-126, and one multiply by a
// power of two applies 2^126 times the block scale.
//
// INT3 (group 128).  Records as for INT4, 6144 + 256 (+128) bytes:
//   [0, 6144)      codes: row r's 12 words; word q = 3c + p (32-K chunk c,
//                  part p < 3) at byte (q/4*128 + r)*16 + 4*(q%4), so a
//                  thread reads its row's record in three 16-byte loads.
//                  Pair i < 15 of chunk c (codes 32c + 2i, 32c + 2i + 1)
//                  sits in word 3c + i/5 at bits 3*(i%5) (even k) and
//                  16 + 3*(i%5) (odd k); pair 15 keeps code bit p at bit 15
//                  (even k) and bit 31 (odd k) of word 3c + p.  As for INT4,
//                  one shift and one LOP3 with 0x00070007 / 0x43004300 give
//                  the bf16 pair (128 + q, 128 + q').
//   [6144, 6400)   fp16 scale of row r at 6144 + 2r
//   [6400, 6528)   uint3 zero point of row r at 6400 + r (asymmetric only)
//
// INT2 (group 128).  Records as for INT4, 4096 + 256 (+128) bytes:
//   [0, 4096)      codes: row r's 8 words; word q = 2c + p (32-K chunk c,
//                  part p < 2) at byte (q/4*128 + r)*16 + 4*(q%4).  Pair i
//                  of chunk c (codes 32c + 2i, 32c + 2i + 1) sits in word
//                  2c + i/8 at bits 2*(i%8) (even k) and 16 + 2*(i%8) (odd
//                  k): one shift and one LOP3 with 0x00030003 / 0x43004300
//                  give the bf16 pair (128 + q, 128 + q').
//   [4096, 4352)   fp16 scale of row r at 4096 + 2r
//   [4352, 4480)   uint2 zero point of row r at 4352 + r (asymmetric only)
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "hq_internal.h"

namespace hq {

namespace {


template <class F>
void parallel_for(size_t n, F&& f) {
  unsigned hw = std::max(1u, std::min(32u, std::thread::hardware_concurrency()));
  size_t nt = std::min<size_t>(hw, n);
  if (nt <= 1) {
    for (size_t i = 0; i < n; ++i) f(i);
    return;
  }
  std::vector<std::thread> th;
  th.reserve(nt);
  for (size_t t = 0; t < nt; ++t) {
    th.emplace_back([&, t]() {
      for (size_t i = t; i < n; i += nt) f(i);
    });
  }
  for (auto& x : th) x.join();
}

// Nibble permutation inside one 32-bit word: canonical element e (bits 4e)
// moves to nibble (e%2)*4 + e/2.
inline uint32_t permute_word(uint32_t w) {
  uint32_t out = 0;
  for (int e = 0; e < 8; ++e) {
    uint32_t code = (w >> (4 * e)) & 0xF;
    int p = (e & 1) * 4 + (e >> 1);
    out |= code << (4 * p);
  }
  return out;
}

hq_status pack_int4(const hq_quant_desc& d, const int32_t* codes, const uint16_t* scales, const uint8_t* zeros,
                    uint8_t* out) {
  const int n = d.n, k = d.k;
  const int nt_count = (n + kTileN - 1) / kTileN;
  const int kb_count = k / kBlockK;
  const bool hz = zeros != nullptr;
  const size_t rec = (size_t)w4_record_bytes(hz);
  const size_t expert_bytes = (size_t)nt_count * kb_count * rec;
  const size_t kw = (size_t)k / 8;   // canonical words per row
  const size_t kg = (size_t)k / 128; // groups per row
  // reject zero points outside 0..15 before writing anything
  if (hz) {
    const size_t total = (size_t)d.num_experts * n * kg;
    for (size_t i = 0; i < total; ++i)
      if (zeros[i] > 15) return HQ_ERR_INVALID_ARG;
  }
  const size_t jobs = (size_t)d.num_experts * nt_count;
  parallel_for(jobs, [&](size_t job) {
    const size_t e = job / nt_count;
    const int nt = (int)(job % nt_count);
    uint8_t* ebase = out + e * expert_bytes;
    for (int kb = 0; kb < kb_count; ++kb) {
      uint8_t* r0 = ebase + ((size_t)nt * kb_count + kb) * rec;
      std::memset(r0, 0, rec);
      for (int r = 0; r < kTileN; ++r) {
        const int row = nt * kTileN + r;
        if (row >= n) break;
        const int32_t* src = codes + (e * n + row) * kw + (size_t)kb * 16;
        for (int c = 0; c < 4; ++c) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(r0 + ((size_t)c * 128 + r) * 16);
          for (int w = 0; w < 4; ++w) dst[w] = permute_word((uint32_t)src[c * 4 + w]);
        }
        const uint16_t s = scales[(e * n + row) * kg + kb];
        std::memcpy(r0 + kW4RecCodes + 2 * r, &s, 2);
        if (hz) r0[kW4RecCodes + 256 + r] = zeros[(e * n + row) * kg + kb];
      }
    }
  });
  return HQ_OK;
}

hq_status pack_int3(const hq_quant_desc& d, const int32_t* codes, const uint16_t* scales, const uint8_t* zeros,
                    uint8_t* out) {
  const int n = d.n, k = d.k;
  const int nt_count = (n + kTileN - 1) / kTileN;
  const int kb_count = k / kBlockK;
  const bool hz = zeros != nullptr;
  const size_t rec = (size_t)w3_record_bytes(hz);
  const size_t expert_bytes = (size_t)nt_count * kb_count * rec;
  const size_t kw = (size_t)k * 3 / 32;  // canonical words per row
  const size_t kg = (size_t)k / 128;
  if (hz) {
    const size_t total = (size_t)d.num_experts * n * kg;
    for (size_t i = 0; i < total; ++i)
      if (zeros[i] > 7) return HQ_ERR_INVALID_ARG;
  }
  const size_t jobs = (size_t)d.num_experts * nt_count;
  parallel_for(jobs, [&](size_t job) {
    const size_t e = job / nt_count;
    const int nt = (int)(job % nt_count);
    uint8_t* ebase = out + e * expert_bytes;
    for (int kb = 0; kb < kb_count; ++kb) {
      uint8_t* r0 = ebase + ((size_t)nt * kb_count + kb) * rec;
      std::memset(r0, 0, rec);
      for (int r = 0; r < kTileN; ++r) {
        const int row = nt * kTileN + r;
        if (row >= n) break;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(codes + (e * n + row) * kw);
        // code k of the row: stream bits 3k .. 3k+2
        auto code = [&](int kk) {
          uint32_t v = 0;
          for (int b = 0; b < 3; ++b) {
            const size_t bit = (size_t)3 * ((size_t)kb * 128 + kk) + b;
            v |= ((src[bit / 32] >> (bit % 32)) & 1u) << b;
          }
          return v;
        };
        uint32_t words[12] = {};
        for (int kk = 0; kk < 128; ++kk) {
          const int c = kk / 32, i = (kk % 32) / 2, h = kk % 2;
          const uint32_t v = code(kk);
          if (i < 15) {
            words[3 * c + i / 5] |= v << (3 * (i % 5) + 16 * h);
          } else {
            for (int b = 0; b < 3; ++b) words[3 * c + b] |= ((v >> b) & 1u) << (15 + 16 * h);
          }
        }
        for (int q = 0; q < 12; ++q) std::memcpy(r0 + ((size_t)(q / 4) * 128 + r) * 16 + 4 * (q % 4), &words[q], 4);
        const uint16_t s = scales[(e * n + row) * kg + kb];
        std::memcpy(r0 + kW3RecCodes + 2 * r, &s, 2);
        if (hz) r0[kW3RecCodes + 256 + r] = zeros[(e * n + row) * kg + kb];
      }
    }
  });
  return HQ_OK;
}

hq_status pack_int2(const hq_quant_desc& d, const int32_t* codes, const uint16_t* scales, const uint8_t* zeros,
                    uint8_t* out) {
  const int n = d.n, k = d.k;
  const int nt_count = (n + kTileN - 1) / kTileN;
  const int kb_count = k / kBlockK;
  const bool hz = zeros != nullptr;
  const size_t rec = (size_t)w2_record_bytes(hz);
  const size_t expert_bytes = (size_t)nt_count * kb_count * rec;
  const size_t kw = (size_t)k / 16;  // canonical words per row
  const size_t kg = (size_t)k / 128;
  if (hz) {
    const size_t total = (size_t)d.num_experts * n * kg;
    for (size_t i = 0; i < total; ++i)
      if (zeros[i] > 3) return HQ_ERR_INVALID_ARG;
  }
  const size_t jobs = (size_t)d.num_experts * nt_count;
  parallel_for(jobs, [&](size_t job) {
    const size_t e = job / nt_count;
    const int nt = (int)(job % nt_count);
    uint8_t* ebase = out + e * expert_bytes;
    for (int kb = 0; kb < kb_count; ++kb) {
      uint8_t* r0 = ebase + ((size_t)nt * kb_count + kb) * rec;
      std::memset(r0, 0, rec);
      for (int r = 0; r < kTileN; ++r) {
        const int row = nt * kTileN + r;
        if (row >= n) break;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(codes + (e * n + row) * kw) + (size_t)kb * 8;
        uint32_t words[8] = {};
        for (int kk = 0; kk < 128; ++kk) {
          const uint32_t v = (src[kk / 16] >> (2 * (kk % 16))) & 3u;
          const int c = kk / 32, i = (kk % 32) / 2, h = kk % 2;
          words[2 * c + i / 8] |= v << (2 * (i % 8) + 16 * h);
        }
        for (int q = 0; q < 8; ++q) std::memcpy(r0 + ((size_t)(q / 4) * 128 + r) * 16 + 4 * (q % 4), &words[q], 4);
        const uint16_t s = scales[(e * n + row) * kg + kb];
        std::memcpy(r0 + kW2RecCodes + 2 * r, &s, 2);
        if (hz) r0[kW2RecCodes + 256 + r] = zeros[(e * n + row) * kg + kb];
      }
    }
  });
  return HQ_OK;
}

// [pair j][half h][code bit b] -> bit of the 32-bit word
constexpr int kMxBits[4][2][4] = {
    {{6, 7, 8, 15}, {22, 23, 24, 31}},
    {{10, 11, 12, 19}, {26, 27, 28, 3}},
    {{16, 17, 18, 25}, {0, 1, 2, 9}},
    {{4, 5, 14, 13}, {20, 21, 30, 29}},
};

hq_status pack_mx_a16(const hq_quant_desc& d, const uint8_t* codes, const uint8_t* scales, uint8_t* out) {
  const int n = d.n, k = d.k;
  const int nt_count = (n + kTileN - 1) / kTileN;
  const int kb_count = k / kBlockK;
  const size_t rec = (size_t)kMxA16RecBytes;
  const size_t expert_bytes = (size_t)nt_count * kb_count * rec;
  const size_t row_bytes = (size_t)k / 2, row_scales = (size_t)k / 32;
  // scales above 2^125 would make bf16 weights overflow (255 is NaN)
  const size_t total_scales = (size_t)d.num_experts * n * row_scales;
  for (size_t i = 0; i < total_scales; ++i)
    if (scales[i] > 252) return HQ_ERR_INVALID_ARG;
  const size_t jobs = (size_t)d.num_experts * nt_count;
  parallel_for(jobs, [&](size_t job) {
    const size_t e = job / nt_count;
    const int nt = (int)(job % nt_count);
    uint8_t* ebase = out + e * expert_bytes;
    for (int kb = 0; kb < kb_count; ++kb) {
      uint8_t* r0 = ebase + ((size_t)nt * kb_count + kb) * rec;
      std::memset(r0, 0, rec);
      for (int r = 0; r < kTileN; ++r) {
        const int row = nt * kTileN + r;
        if (row >= n) break;
        const uint8_t* src = codes + (e * n + row) * row_bytes + (size_t)kb * 64;
        for (int c = 0; c < 4; ++c) {
          for (int w = 0; w < 4; ++w) {
            uint32_t word = 0;
            for (int j = 0; j < 4; ++j)
              for (int h = 0; h < 2; ++h) {
                const int kk = 32 * c + 8 * w + 2 * j + h;
                const uint32_t code = (src[kk / 2] >> (4 * (kk % 2))) & 0xF;
                for (int b = 0; b < 4; ++b) word |= ((code >> b) & 1u) << kMxBits[j][h][b];
              }
            std::memcpy(r0 + ((size_t)c * 128 + r) * 16 + 4 * w, &word, 4);
          }
          r0[kW4RecCodes + 4 * r + c] = scales[(e * n + row) * row_scales + (size_t)kb * 4 + c];
        }
      }
    }
  });
  return HQ_OK;
}

// INT8 (group 128): row r's 16-K chunk c of a record is its 16 code bytes
// at (c*128 + r)*16, in K order; scales and zero points as for INT4.
hq_status pack_int8(const hq_quant_desc& d, const int32_t* codes, const uint16_t* scales, const uint8_t* zeros,
                    uint8_t* out) {
  const int n = d.n, k = d.k;
  const int nt_count = (n + kTileN - 1) / kTileN;
  const int kb_count = k / kBlockK;
  const bool hz = zeros != nullptr;
  const size_t rec = (size_t)w8_record_bytes(hz);
  const size_t expert_bytes = (size_t)nt_count * kb_count * rec;
  const size_t row_bytes = (size_t)k;   // canonical: four codes per int32, low byte first
  const size_t kg = (size_t)k / 128;
  const size_t jobs = (size_t)d.num_experts * nt_count;
  parallel_for(jobs, [&](size_t job) {
    const size_t e = job / nt_count;
    const int nt = (int)(job % nt_count);
    uint8_t* ebase = out + e * expert_bytes;
    const uint8_t* cb = reinterpret_cast<const uint8_t*>(codes);
    for (int kb = 0; kb < kb_count; ++kb) {
      uint8_t* r0 = ebase + ((size_t)nt * kb_count + kb) * rec;
      std::memset(r0, 0, rec);
      for (int r = 0; r < kTileN; ++r) {
        const int row = nt * kTileN + r;
        if (row >= n) break;
        // little-endian words: code k is byte k of the row
        const uint8_t* src = cb + (e * n + row) * row_bytes + (size_t)kb * 128;
        for (int c = 0; c < 8; ++c) std::memcpy(r0 + ((size_t)c * 128 + r) * 16, src + 16 * c, 16);
        const uint16_t s = scales[(e * n + row) * kg + kb];
        std::memcpy(r0 + kW8RecCodes + 2 * r, &s, 2);
        if (hz) r0[kW8RecCodes + 256 + r] = zeros[(e * n + row) * kg + kb];
      }
    }
  });
  return HQ_OK;
}

// MXINT4 (E8M0 scale per 32 K): the INT4 nibble layout of the codes, the
// MXFP4_A16 placement of the scales.
hq_status pack_mxi4(const hq_quant_desc& d, const uint8_t* codes, const uint8_t* scales, uint8_t* out) {
  const int n = d.n, k = d.k;
  const int nt_count = (n + kTileN - 1) / kTileN;
  const int kb_count = k / kBlockK;
  const size_t rec = (size_t)kMxi4RecBytes;
  const size_t expert_bytes = (size_t)nt_count * kb_count * rec;
  const size_t row_bytes = (size_t)k / 2, row_scales = (size_t)k / 32;
  // scales above 2^124 would make bf16 weights of magnitude 8 overflow
  const size_t total_scales = (size_t)d.num_experts * n * row_scales;
  for (size_t i = 0; i < total_scales; ++i)
    if (scales[i] > 251) return HQ_ERR_INVALID_ARG;
  const size_t jobs = (size_t)d.num_experts * nt_count;
  parallel_for(jobs, [&](size_t job) {
    const size_t e = job / nt_count;
    const int nt = (int)(job % nt_count);
    uint8_t* ebase = out + e * expert_bytes;
    for (int kb = 0; kb < kb_count; ++kb) {
      uint8_t* r0 = ebase + ((size_t)nt * kb_count + kb) * rec;
      std::memset(r0, 0, rec);
      for (int r = 0; r < kTileN; ++r) {
        const int row = nt * kTileN + r;
        if (row >= n) break;
        const uint8_t* src = codes + (e * n + row) * row_bytes + (size_t)kb * 64;
        for (int c = 0; c < 4; ++c) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(r0 + ((size_t)c * 128 + r) * 16);
          for (int w = 0; w < 4; ++w) {
            uint32_t word;   // eight codes, even k in the low nibble of each byte: the canonical INT4 word
            std::memcpy(&word, src + 16 * c + 4 * w, 4);
            dst[w] = permute_word(word);
          }
          r0[kW4RecCodes + 4 * r + c] = scales[(e * n + row) * row_scales + (size_t)kb * 4 + c];
        }
      }
    }
  });
  return HQ_OK;
}

// Block-scaled formats: copy codes row by row, then lay out scale blocks.
hq_status pack_fp4(const hq_quant_desc& d, const uint8_t* codes, const uint8_t* scales, float g, uint8_t* out) {
  const int n = d.n, k = d.k;
  const int np = (n + kTileN - 1) / kTileN * kTileN;
  const size_t row_bytes = (size_t)k / 2;
  const int blk = d.group_size;                   // 32 (MX) or 16 (NV)
  const int blocks = k / blk;                     // scale entries per row
  const int groups = blocks / 4;                  // 512-byte chunks per tile
  const size_t codes_bytes = (size_t)np * row_bytes;
  std::memset(out, 0, codes_bytes);
  for (int r = 0; r < n; ++r) std::memcpy(out + (size_t)r * row_bytes, codes + (size_t)r * row_bytes, row_bytes);
  uint8_t* sf = out + codes_bytes;
  const int nt_count = np / kTileN;
  parallel_for((size_t)nt_count, [&](size_t nt) {
    for (int g4 = 0; g4 < groups; ++g4) {
      uint8_t* chunk = sf + ((size_t)nt * groups + g4) * 512;
      for (int l = 0; l < 32; ++l)
        for (int c = 0; c < 4; ++c)
          for (int j = 0; j < 4; ++j) {
            const int row = (int)nt * kTileN + l + 32 * c;
            chunk[l * 16 + c * 4 + j] = row < n ? scales[(size_t)row * blocks + 4 * g4 + j] : 0;
          }
    }
  });
  if (d.fmt == HQ_FMT_NVFP4) {
    uint8_t* tail = sf + (size_t)nt_count * groups * 512;
    std::memset(tail, 0, 16);
    std::memcpy(tail, &g, 4);
  }
  return HQ_OK;
}

}  // namespace

size_t packed_size_impl(const hq_quant_desc& d) {
  const size_t nt = (size_t)(d.n + kTileN - 1) / kTileN;
  switch (d.fmt) {
    case HQ_FMT_INT4:
      return (size_t)d.num_experts * nt * (d.k / kBlockK) * w4_record_bytes(d.has_zero_point != 0);
    case HQ_FMT_MXFP4:
      return nt * kTileN * (size_t)d.k / 2 + nt * (d.k / 128) * 512;
    case HQ_FMT_NVFP4:
      return nt * kTileN * (size_t)d.k / 2 + nt * (d.k / 64) * 512 + 16;
    case HQ_FMT_MXFP4_A16:
      return (size_t)d.num_experts * nt * (d.k / kBlockK) * kMxA16RecBytes;
    case HQ_FMT_INT3:
      return (size_t)d.num_experts * nt * (d.k / kBlockK) * w3_record_bytes(d.has_zero_point != 0);
    case HQ_FMT_INT2:
      return (size_t)d.num_experts * nt * (d.k / kBlockK) * w2_record_bytes(d.has_zero_point != 0);
    case HQ_FMT_INT8:
      return (size_t)d.num_experts * nt * (d.k / kBlockK) * w8_record_bytes(d.has_zero_point != 0);
    case HQ_FMT_MXINT4:
      return (size_t)d.num_experts * nt * (d.k / kBlockK) * kMxi4RecBytes;
    default:
      return 0;
  }
}

hq_status pack_impl(const hq_quant_desc& d, const void* codes, const void* scales, const void* zeros, float g,
                    void* out) {
  switch (d.fmt) {
    case HQ_FMT_INT4:
      return pack_int4(d, static_cast<const int32_t*>(codes), static_cast<const uint16_t*>(scales),
                       static_cast<const uint8_t*>(zeros), static_cast<uint8_t*>(out));
    case HQ_FMT_MXFP4:
    case HQ_FMT_NVFP4:
      return pack_fp4(d, static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(scales), g,
                      static_cast<uint8_t*>(out));
    case HQ_FMT_MXFP4_A16:
      return pack_mx_a16(d, static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(scales),
                         static_cast<uint8_t*>(out));
    case HQ_FMT_INT3:
      return pack_int3(d, static_cast<const int32_t*>(codes), static_cast<const uint16_t*>(scales),
                       static_cast<const uint8_t*>(zeros), static_cast<uint8_t*>(out));
    case HQ_FMT_INT2:
      return pack_int2(d, static_cast<const int32_t*>(codes), static_cast<const uint16_t*>(scales),
                       static_cast<const uint8_t*>(zeros), static_cast<uint8_t*>(out));
    case HQ_FMT_INT8:
      return pack_int8(d, static_cast<const int32_t*>(codes), static_cast<const uint16_t*>(scales),
                       static_cast<const uint8_t*>(zeros), static_cast<uint8_t*>(out));
    case HQ_FMT_MXINT4:
      return pack_mxi4(d, static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(scales),
                       static_cast<uint8_t*>(out));
    default:
      return HQ_ERR_INVALID_ARG;
  }
}

// Canonical bytes per weight row of the W4A16-family formats: codes, scales
// and zero points (0 for formats without them).
struct RowBytes {
  size_t codes, scales, zeros;
};
static bool w16_row_bytes(const hq_quant_desc& d, RowBytes* rb) {
  const size_t k = (size_t)d.k;
  switch (d.fmt) {
    case HQ_FMT_INT4: *rb = {k / 2, 2 * (k / 128), k / 128}; return true;
    case HQ_FMT_INT3: *rb = {3 * k / 8, 2 * (k / 128), k / 128}; return true;
    case HQ_FMT_INT2: *rb = {k / 4, 2 * (k / 128), k / 128}; return true;
    case HQ_FMT_MXFP4_A16: *rb = {k / 2, k / 32, 0}; return true;
    case HQ_FMT_INT8: *rb = {k, 2 * (k / 128), k / 128}; return true;
    case HQ_FMT_MXINT4: *rb = {k / 2, k / 32, 0}; return true;
    default: return false;
  }
}

// Canonical row of packed row p in the gated gate+up order (n = 2I rows,
// gate rows [0, I), up rows [I, 2I)): in every 32-row quarter q of tile j,
// rows 0-15 are gate rows 64j + 16q + l and rows 16-31 the up rows of the
// same indices, I + 64j + 16q + (l - 16).
static int gated_source_row(int p, int n) {
  const int j = p / 128, r = p % 128, q = r / 32, l = r % 32;
  return l < 16 ? 64 * j + 16 * q + l : n / 2 + 64 * j + 16 * q + (l - 16);
}

hq_status pack_gated_impl(const hq_quant_desc& d, const void* codes, const void* scales, const void* zeros,
                          void* out) {
  RowBytes rb{};
  if (!w16_row_bytes(d, &rb) || d.n % 128 != 0) return HQ_ERR_UNSUPPORTED;
  const size_t rows = (size_t)d.num_experts * d.n;
  std::vector<uint8_t> c2(rows * rb.codes), s2(rows * rb.scales), z2(zeros ? rows * rb.zeros : 0);
  const uint8_t* c = static_cast<const uint8_t*>(codes);
  const uint8_t* sc = static_cast<const uint8_t*>(scales);
  const uint8_t* z = static_cast<const uint8_t*>(zeros);
  for (size_t e = 0; e < (size_t)d.num_experts; ++e) {
    for (int p = 0; p < d.n; ++p) {
      const size_t dst = e * d.n + p, src = e * d.n + gated_source_row(p, d.n);
      std::memcpy(&c2[dst * rb.codes], c + src * rb.codes, rb.codes);
      std::memcpy(&s2[dst * rb.scales], sc + src * rb.scales, rb.scales);
      if (z) std::memcpy(&z2[dst * rb.zeros], z + src * rb.zeros, rb.zeros);
    }
  }
  return pack_impl(d, c2.data(), s2.data(), z ? z2.data() : nullptr, 0.f, out);
}

}  // namespace hq
