// Output stores shared by the GEMM epilogues.
//
// Every kernel here is swap-AB: an epilogue warp holds, for 32 consecutive
// weight rows (output columns n = n_warp + lane), the values of a run of
// tokens (output rows).  Written directly, token j of such a run is one
// 64-byte store of 2-byte elements; after a warp-local transpose through
// shared memory each lane writes 16 contiguous bytes of an output row.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

namespace hq {

// Tokens j0 .. j0+EB-1 of one warp's 32 output columns: lane holds v[j] for
// output element (row0 + j0 + j, n_warp + lane).
//   part != nullptr : fp32 into a partial tile slot laid out [token][128]
//                     (column r_tile = the row of the weight tile);
//   n_total % 8 == 0 and sc != nullptr: bf16 through the transpose buffer
//                     `sc` (32 x EB uint16, 16-byte aligned), 16-byte stores;
//   otherwise       : one bf16 per (token, column).
// Rows at or past `rows` (tokens beyond the tile's valid rows) and columns
// at or past n_total are not written.  `sc` is reused after the call (the
// warp is synchronized on both sides of the transpose).
template <int EB>
__device__ __forceinline__ void store_rows_chunk(__nv_bfloat16* c, int n_total, int row0, int rows, int n_warp,
                                                 int r_tile, float* part, int lane, int j0, const float (&v)[EB],
                                                 uint16_t* sc) {
  static_assert(EB % 8 == 0, "token runs of 8");
  if (part) {
#pragma unroll
    for (int j = 0; j < EB; ++j) __stcg(part + (size_t)(j0 + j) * 128 + r_tile, v[j]);
  } else if ((n_total % 8) == 0 && sc != nullptr) {
#pragma unroll
    for (int j = 0; j < EB; ++j) sc[j * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
    __syncwarp();
    const int seg = lane & 3;
    const int n0 = n_warp + seg * 8;
#pragma unroll
    for (int i = 0; i < EB / 8; ++i) {
      const int jj = (lane >> 2) + 8 * i;
      if (j0 + jj < rows && n0 < n_total) {
        const uint4 w = *reinterpret_cast<const uint4*>(sc + jj * 32 + seg * 8);
        *reinterpret_cast<uint4*>(c + (size_t)(row0 + j0 + jj) * n_total + n0) = w;
      }
    }
    __syncwarp();
  } else if (n_warp + lane < n_total) {
#pragma unroll
    for (int j = 0; j < EB; ++j) {
      if (j0 + j < rows) c[(size_t)(row0 + j0 + j) * n_total + n_warp + lane] = __float2bfloat16_rn(v[j]);
    }
  }
}

// SwiGLU epilogue of a gate+up GEMM whose weights were packed in the gated
// row order: in every 32-row quarter of a 128-row weight tile, lanes 0-15
// hold 16 gate features and lanes 16-31 the up features of the same 16
// indices.  Lane l holds v[j] for tokens j0 .. j0+EB-1 of its row; lanes l
// and l ^ 16 swap values, so each has gate g and up u of feature
// h_col0 + (l & 15); lane l < 16 computes tokens j0 .. j0+EB/2-1, lane
// l >= 16 the rest: h = silu(g) * u, silu(x) = x / (1 + exp(-x)), fp32, one
// bf16 rounding.  The exponential and the division are the hardware's
// approximate ones (__expf, __fdividef: relative errors of a few 1e-6 at
// most, far below the 2^-9 of the bf16 rounding that follows); the exact
// library forms cost ~13 % of the grouped gate+up GEMM at T=8192, top-8 of
// 256 experts, because the warps that run this epilogue also dequantize.
// Stores as store_rows_chunk (16-byte rows of 8 features
// through the transpose buffer `sc`, 16 x EB uint16; element by element
// when sc is null or h_cols % 8 != 0).  Rows at or past `rows` are not
// written.
template <int EB>
__device__ __forceinline__ void store_swiglu_chunk(__nv_bfloat16* h, int h_cols, int row0, int rows, int h_col0,
                                                   int lane, int j0, const float (&v)[EB], uint16_t* sc) {
  static_assert(EB % 8 == 0, "token runs of 8");
  const bool up_lane = lane >= 16;
  const int f = h_col0 + (lane & 15);
  uint16_t hv[EB / 2];
#pragma unroll
  for (int j = 0; j < EB / 2; ++j) {
    // the gate lane sends its value of token j + EB/2 and receives the up
    // value of token j; the up lane sends token j and receives the gate
    // value of token j + EB/2
    const float mine = up_lane ? v[j + EB / 2] : v[j];
    const float recv = __shfl_xor_sync(0xffffffffu, up_lane ? v[j] : v[j + EB / 2], 16);
    const float g = up_lane ? recv : mine;
    const float u = up_lane ? mine : recv;
    hv[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fdividef(g, 1.f + __expf(-g)) * u));
  }
  const int jbase = up_lane ? EB / 2 : 0;
  if (sc != nullptr && (h_cols % 8) == 0) {
#pragma unroll
    for (int j = 0; j < EB / 2; ++j) sc[(jbase + j) * 16 + (lane & 15)] = hv[j];
    __syncwarp();
#pragma unroll
    for (int i = 0; i < EB / 16; ++i) {
      const int jj = (lane >> 1) + 16 * i;   // token of this lane's 16-byte piece
      const int half = lane & 1;             // features 0-7 or 8-15 of the warp's 16
      const int col = h_col0 + half * 8;
      if (j0 + jj < rows && col < h_cols) {
        const uint4 w = *reinterpret_cast<const uint4*>(sc + jj * 16 + half * 8);
        *reinterpret_cast<uint4*>(h + (size_t)(row0 + j0 + jj) * h_cols + col) = w;
      }
    }
    __syncwarp();
  } else if (f < h_cols) {
#pragma unroll
    for (int j = 0; j < EB / 2; ++j) {
      if (j0 + jbase + j < rows) h[(size_t)(row0 + j0 + jbase + j) * h_cols + f] = __ushort_as_bfloat16(hv[j]);
    }
  }
}

}  // namespace hq
