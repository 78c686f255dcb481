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

}  // namespace hq
