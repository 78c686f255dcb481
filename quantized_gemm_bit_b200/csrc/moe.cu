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
// All integer work; nothing here waits on anything, so nothing can hang.
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
__global__ void topk_kernel(const float* __restrict__ logits, int t, int e, int k, int32_t* __restrict__ ids) {
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
  return sizeof(WsHeader) + ((nb * e * sizeof(int32_t) + 255) / 256) * 256;
}

hq_status moe_topk_launch(const float* logits, int t, int e, int k, int32_t* ids, cudaStream_t s) {
  const int warps = 8;
  topk_kernel<<<(t + warps - 1) / warps, warps * 32, 0, s>>>(logits, t, e, k, ids);
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

hq_status moe_permute_launch(const int32_t* ids, int t, int k, int e, int32_t* sorted_src, int32_t* offsets,
                             const void* a, int hidden, void* a_sorted, void* ws, cudaStream_t s) {
  uint32_t* err = static_cast<uint32_t*>(ws);
  int32_t* counts = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + sizeof(WsHeader));
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
