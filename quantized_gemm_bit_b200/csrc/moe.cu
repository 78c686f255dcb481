// MoE routing and expert-sorted permutation kernels, and the bounded-wait
// test kernel.
//
// The grouped MoE path ("Humming: open-source kernel library for quantized
// inference", summary paragraph 5; Humming news page, table row "MoE W4A16")
// runs every expert's GEMM from one launch over tokens sorted by expert.
// These kernels produce that order:
//   topk    : per token, the k experts with the largest router logits
//             (ties to the lower expert index), descending;
//   permute : per-expert counts -> exclusive prefix sum (expert offsets) ->
//             the flattened slot list ordered by (expert, slot), stable, so
//             it is unique and matches a plain counting sort bit for bit;
//   gather  : rows of A copied into expert-sorted order.
// Around the two grouped GEMMs of the layer:
//   softmax : the selected experts' softmax probabilities (the combine
//             weights), from the same pass as top-k;
//   swiglu  : h = silu(gate) * up on the gate+up GEMM's output;
//   combine : the down GEMM's rows un-permuted and summed per token with
//             those weights, in slot order (deterministic, no atomics).
// Nothing here waits on anything, so nothing can hang.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "hq_internal.h"
#include "ptx.cuh"

namespace hq {

namespace {

constexpr int kPermTok = 128;   // tokens per block in the permutation

// One warp per token.  Each lane holds ceil(E/32) logits; k rounds of a
// warp-wide (value desc, index asc) arg-max pick the experts in order.
__global__ void topk_kernel(const float* __restrict__ logits, int t, int e, int k, int32_t* __restrict__ ids,
                            float* __restrict__ weights) {
  const int warps = blockDim.x >> 5;
  const int tok = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= t) return;
  constexpr int kPer = 32;  // up to 1024 experts
  float v[kPer];
  const float* row = logits + (size_t)tok * e;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = i * 32 + lane;
    v[i] = idx < e ? row[idx] : -__int_as_float(0x7f800000);  // -inf
  }
  uint32_t taken = 0;  // bit i: v[i] already selected
  float vmax = 0.f, vsel = 0.f;
  for (int r = 0; r < k; ++r) {
    float best = 0.f;
    int bidx = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int idx = i * 32 + lane;
      if (idx < e && !((taken >> i) & 1u)) {
        if (bidx == 0x7fffffff || v[i] > best) {  // indices ascend with i: ties keep the lower
          best = v[i];
          bidx = idx;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
      const bool take = (oi != 0x7fffffff) && (bidx == 0x7fffffff || ob > best || (ob == best && oi < bidx));
      if (take) {
        best = ob;
        bidx = oi;
      }
    }
    if (lane == 0) ids[(size_t)tok * k + r] = bidx;
    if ((bidx & 31) == lane) taken |= 1u << (bidx >> 5);
    if (r == 0) vmax = best;
    if (lane == r) vsel = best;            // lane r keeps the logit of slot r
  }
  if (weights) {
    // softmax over all e logits in fp32: each lane sums its own logits in
    // index order, then a fixed butterfly adds the lanes (deterministic)
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int idx = i * 32 + lane;
      if (idx < e) sum += expf(v[i] - vmax);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < k) weights[(size_t)tok * k + lane] = expf(vsel - vmax) / sum;
  }
}

// Per-block expert histogram of the slots of kPermTok tokens.
__global__ void perm_count_kernel(const int32_t* __restrict__ ids, int t, int k, int e, int32_t* __restrict__ counts,
                                  uint32_t* err) {
  extern __shared__ int32_t hist[];
  for (int i = threadIdx.x; i < e; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const long long s0 = (long long)blockIdx.x * kPermTok * k;
  const long long s1 = min((long long)t * k, s0 + (long long)kPermTok * k);
  bool bad = false;
  for (long long s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
    const int x = ids[s];
    if (x < 0 || x >= e) bad = true;
    else atomicAdd(&hist[x], 1);
  }
  if (bad) atomicCAS(err, 0u, (uint32_t)HQ_ERR_DEVICE_BAD_OFFSETS);
  __syncthreads();
  for (int i = threadIdx.x; i < e; i += blockDim.x) counts[(size_t)blockIdx.x * e + i] = hist[i];
}

// One block: expert totals, exclusive scan -> offsets, per-(block, expert)
// base positions.
__global__ void perm_scan_kernel(int32_t* __restrict__ counts_base, int nblocks, int e, int total_slots,
                                 int32_t* __restrict__ offsets) {
  __shared__ int32_t tot[1024];
  __shared__ int32_t warp_sums[32];
  const int x = threadIdx.x;  // expert
  int run = 0;
  if (x < e) {
    for (int b = 0; b < nblocks; ++b) {
      int32_t* p = counts_base + (size_t)b * e + x;
      const int c = *p;
      *p = run;  // becomes the base inside expert x for block b
      run += c;
    }
  }
  tot[x] = x < e ? run : 0;
  __syncthreads();
  // exclusive scan of tot[0..1023] (1024 threads)
  const int lane = x & 31, w = x >> 5;
  int v = tot[x];
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    int ws = warp_sums[lane];
    int wi = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    warp_sums[lane] = wi - ws;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = warp_sums[w] + incl - v;
  if (x < e) {
    offsets[x] = excl;
    for (int b = 0; b < nblocks; ++b) counts_base[(size_t)b * e + x] += excl;
  }
  if (x == 0) offsets[e] = total_slots;
}

// One warp per block of kPermTok tokens walks its slots in order, 32 at a
// time; within a group, ranks among equal experts come from match_any.
__global__ void perm_scatter_kernel(const int32_t* __restrict__ ids, int t, int k, int e,
                                    const int32_t* __restrict__ base, int32_t* __restrict__ sorted_src) {
  extern __shared__ int32_t cursor[];
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < e; i += 32) cursor[i] = base[(size_t)blockIdx.x * e + i];
  __syncwarp();
  const int s0 = blockIdx.x * kPermTok * k;
  const int s1 = min(t * k, s0 + kPermTok * k);
  for (int g = s0; g < s1; g += 32) {
    const int s = g + lane;
    const bool valid_slot = s < s1;
    int x = valid_slot ? ids[s] : -1;
    const bool ok = valid_slot && x >= 0 && x < e;
    if (!ok) x = -1 - lane;  // unique per lane: never matches a real expert
    const unsigned peers = __match_any_sync(0xffffffffu, x);
    const unsigned lower = peers & ((1u << lane) - 1u);
    int pos = 0;
    if (ok) pos = cursor[x] + __popc(lower);
    __syncwarp();
    if (ok) {
      sorted_src[pos] = s;
      if (lower == 0) cursor[x] += __popc(peers);  // lowest peer advances the cursor
    }
    __syncwarp();
  }
}

__global__ void gather_rows_kernel(const int4* __restrict__ a, int hidden_vec, int k, const int32_t* __restrict__ src,
                                   int rows, int4* __restrict__ out) {
  for (long long i = blockIdx.x; i < rows; i += gridDim.x) {
    const long long tok = src[i] / k;
    const int4* s = a + tok * hidden_vec;
    int4* d = out + i * hidden_vec;
    for (int j = threadIdx.x; j < hidden_vec; j += blockDim.x) d[j] = s[j];
  }
}

// h[r][c] = silu(g) * u with g = x[r][c], u = x[r][inter + c]; 8 columns
// (16 bytes) per thread and step, fp32 arithmetic, bf16 round to nearest.
__global__ void swiglu_kernel(const uint4* __restrict__ x, long long rows, int inter_vec, uint4* __restrict__ h) {
  const long long total = rows * inter_vec;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / inter_vec;
    const int c = (int)(i - r * inter_vec);
    const uint4 gv = x[r * 2 * inter_vec + c];
    const uint4 uv = x[r * 2 * inter_vec + inter_vec + c];
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float g0 = __uint_as_float(gw[q] << 16), g1 = __uint_as_float(gw[q] & 0xFFFF0000u);
      const float u0 = __uint_as_float(uw[q] << 16), u1 = __uint_as_float(uw[q] & 0xFFFF0000u);
      const float h0 = g0 / (1.f + expf(-g0)) * u0;
      const float h1 = g1 / (1.f + expf(-g1)) * u1;
      o[q] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(h0)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(h1)) << 16);
    }
    h[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// inv[sorted_src[p]] = p for every sorted position p; a slot index outside
// [0, rows) is reported instead of written.
__global__ void inverse_kernel(const int32_t* __restrict__ src, int rows, int32_t* __restrict__ inv,
                               uint32_t* err) {
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < rows; p += gridDim.x * blockDim.x) {
    const int sl = src[p];
    if (sl < 0 || sl >= rows)
      atomicCAS(err, 0u, (uint32_t)HQ_ERR_DEVICE_BAD_OFFSETS);
    else
      inv[sl] = p;
  }
}

// out[t] = sum_j w[t][j] * y[inv[t*k + j]] over 8 columns per thread and
// step, in slot order j = 0..k-1 (fp32 fused multiply-add), bf16 round to
// nearest.  A slot that no sorted position names (sorted_src was not a
// permutation) is reported and left out.
__global__ void combine_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ inv,
                               const float* __restrict__ w, int t, int k, int hidden_vec, uint4* __restrict__ out,
                               uint32_t* err) {
  __shared__ int s_pos[16];
  __shared__ float s_w[16];
  for (int tok = blockIdx.x; tok < t; tok += gridDim.x) {
    __syncthreads();   // the previous token's slots are no longer read
    if (threadIdx.x < k) {
      int p = inv[(size_t)tok * k + threadIdx.x];
      if (p < 0 || p >= t * k) {
        atomicCAS(err, 0u, (uint32_t)HQ_ERR_DEVICE_BAD_OFFSETS);
        p = -1;
      }
      s_pos[threadIdx.x] = p;
      s_w[threadIdx.x] = w[(size_t)tok * k + threadIdx.x];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < hidden_vec; c += blockDim.x) {
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = 0.f;
      for (int j = 0; j < k; ++j) {
        const int p = s_pos[j];
        if (p < 0) continue;
        const uint4 v = y[(size_t)p * hidden_vec + c];
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
        const float wj = s_w[j];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] = fmaf(wj, __uint_as_float(vw[q] << 16), acc[2 * q]);
          acc[2 * q + 1] = fmaf(wj, __uint_as_float(vw[q] & 0xFFFF0000u), acc[2 * q + 1]);
        }
      }
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * q])) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * q + 1])) << 16);
      out[(size_t)tok * hidden_vec + c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

__global__ void timeout_probe_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    // nobody arrives: the bounded wait must give up and report it
    if (!hq_wait(&bar, 0, limit_ns, nullptr)) atomicCAS(err, 0u, (uint32_t)HQ_ERR_DEVICE_TIMEOUT);
  }
}

}  // namespace

size_t moe_permute_ws_bytes(int t, int k, int e) {
  (void)k;
  const size_t nb = (size_t)(t + kPermTok - 1) / kPermTok;
  return kWsScratchOff + ((nb * e * sizeof(int32_t) + 255) / 256) * 256;
}

hq_status moe_topk_launch(const float* logits, int t, int e, int k, int32_t* ids, float* weights, cudaStream_t s) {
  const int warps = 8;
  topk_kernel<<<(t + warps - 1) / warps, warps * 32, 0, s>>>(logits, t, e, k, ids, weights);
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

hq_status moe_swiglu_launch(const void* x, long long rows, int inter, void* h, cudaStream_t s) {
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  const long long vecs = rows * (inter / 8);
  const long long want = (vecs + 255) / 256;
  const int grid = (int)std::max<long long>(1, std::min<long long>(want, (long long)dev.num_sms * 8));
  swiglu_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), rows, inter / 8, static_cast<uint4*>(h));
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

size_t moe_combine_ws_bytes(int t, int k) {
  return kWsScratchOff + (((size_t)t * k * sizeof(int32_t) + 255) / 256) * 256;
}

hq_status moe_combine_launch(const void* y_sorted, const int32_t* sorted_src, const float* weights, int t, int k,
                             int hidden, void* out, void* ws, cudaStream_t s) {
  DeviceInfo dev{};
  hq_status st = device_info(&dev);
  if (st != HQ_OK) return st;
  uint32_t* err = static_cast<uint32_t*>(ws);
  int32_t* inv = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kWsScratchOff);
  const int rows = t * k;
  // every slot starts unnamed (-1): a sorted list that is not a permutation
  // is reported by the combine instead of read out of bounds
  if (cudaMemsetAsync(inv, 0xFF, (size_t)rows * sizeof(int32_t), s) != cudaSuccess) return HQ_ERR_CUDA;
  const int g1 = std::max(1, std::min((rows + 255) / 256, dev.num_sms * 4));
  inverse_kernel<<<g1, 256, 0, s>>>(sorted_src, rows, inv, err);
  const int g2 = std::max(1, std::min(t, dev.num_sms * 8));
  combine_kernel<<<g2, 128, 0, s>>>(static_cast<const uint4*>(y_sorted), inv, weights, t, k, hidden / 8,
                                    static_cast<uint4*>(out), err);
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

hq_status moe_permute_launch(const int32_t* ids, int t, int k, int e, int32_t* sorted_src, int32_t* offsets,
                             const void* a, int hidden, void* a_sorted, void* ws, cudaStream_t s) {
  uint32_t* err = static_cast<uint32_t*>(ws);
  int32_t* counts = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kWsScratchOff);
  const int nb = (t + kPermTok - 1) / kPermTok;
  if (nb > 0) {
    perm_count_kernel<<<nb, 256, e * sizeof(int32_t), s>>>(ids, t, k, e, counts, err);
  }
  perm_scan_kernel<<<1, 1024, 0, s>>>(counts, nb, e, t * k, offsets);
  if (nb > 0) {
    perm_scatter_kernel<<<nb, 32, e * sizeof(int32_t), s>>>(ids, t, k, e, counts, sorted_src);
    if (a && a_sorted) {
      DeviceInfo dev{};
      device_info(&dev);
      const int rows = t * k;
      const int grid = std::min(rows, dev.num_sms * 8);
      gather_rows_kernel<<<grid, 256, 0, s>>>(static_cast<const int4*>(a), hidden / 8, k, sorted_src, rows,
                                             static_cast<int4*>(a_sorted));
    }
  }
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

hq_status debug_timeout_launch(void* ws, uint64_t limit_ns, cudaStream_t s) {
  timeout_probe_kernel<<<1, 32, 0, s>>>(static_cast<uint32_t*>(ws), limit_ns);
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

}  // namespace hq
