// Merge of split-KV partial results (the qsa2 audit page, "implementation and
// review": the merge caches each chunk's maximum and weight and computes the
// denominator once).
//
// Each split s of a row left O_s (already divided by its own row sum), W_s =
// base-2 log of the sum of the weights its P.V product used, and L_s = base-2
// log-sum-exp of its float32 weights (-inf for an empty split).  With
// M = max_s W_s and w_s = 2^(W_s - M):
//     O = sum_s w_s O_s / sum_s w_s,
// and lse = ln 2 * (ML + log2 sum_s 2^(L_s - ML)) with ML = max_s L_s.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace attn {

constexpr int kMergeMaxSplits = 128;
constexpr int kMergeWarps = 4;

// grid: rows, 128 threads; one CTA per output row.  Warp 0 computes every
// split's weight once (cached in shared memory) and the denominator; then warp w
// accumulates splits w, w + 4, ... with all of its loads in flight, and the four
// partial sums are added in shared memory.
template <int D, bool F16>
__global__ void __launch_bounds__(32 * kMergeWarps) splitkv_merge_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part,
    uint16_t* __restrict__ out, float* __restrict__ lse, int rows, int splits) {
  constexpr int kPer = D / 32;  // channels per lane
  __shared__ float wts[kMergeMaxSplits];
  __shared__ float red[kMergeWarps][D];
  __shared__ float inv_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x;
  // Launched as a programmatic dependent of the split kernel: wait until that
  // grid has completed and its partials are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (warp == 0) {
    float M = -INFINITY;
    for (int s = lane; s < splits; s += 32) M = fmaxf(M, lse_part[(size_t)s * rows + row]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float wsum = 0.0f;
    for (int s = lane; s < splits; s += 32) {
      const float L = lse_part[(size_t)s * rows + row];
      const float w = (M == -INFINITY) ? 0.0f : ex2(L - M);
      wts[s] = w;
      wsum += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    if (lane == 0) inv_s = (wsum > 0.0f) ? 1.0f / wsum : 0.0f;
    if (lse != nullptr) {
      const float* lf = lse_part + (size_t)splits * rows;
      float ML = -INFINITY;
      for (int s = lane; s < splits; s += 32) ML = fmaxf(ML, lf[(size_t)s * rows + row]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ML = fmaxf(ML, __shfl_xor_sync(0xffffffffu, ML, o));
      float ls = 0.0f;
      for (int s = lane; s < splits; s += 32)
        ls += (ML == -INFINITY) ? 0.0f : ex2(lf[(size_t)s * rows + row] - ML);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
      if (lane == 0)
        lse[row] = (ls > 0.0f) ? (ML + lg2(ls)) * 0.69314718055994531f : -INFINITY;
    }
  }
  __syncthreads();
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.0f;
#pragma unroll 8
  for (int s = warp; s < splits; s += kMergeWarps) {
    const float w = wts[s];
    if (w == 0.0f) continue;  // empty or negligible split: its partials are never read
    const float* src = o_part + ((size_t)s * rows + row) * D + lane * kPer;
    if constexpr (kPer == 4) {
      const float4 v = *reinterpret_cast<const float4*>(src);
      acc[0] += w * v.x;
      acc[1] += w * v.y;
      acc[2] += w * v.z;
      acc[3] += w * v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(src);
      acc[0] += w * v.x;
      acc[1] += w * v.y;
    }
  }
#pragma unroll
  for (int e = 0; e < kPer; ++e) red[warp][lane * kPer + e] = acc[e];
  __syncthreads();
  if (warp == 0) {
    const float inv = inv_s;
    uint16_t h[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      float val = 0.0f;
#pragma unroll
      for (int w = 0; w < kMergeWarps; ++w) val += red[w][lane * kPer + e];
      val *= inv;
      if constexpr (F16) {
        const __half b = __float2half_rn(val);
        h[e] = *reinterpret_cast<const uint16_t*>(&b);
      } else {
        const __nv_bfloat16 b = __float2bfloat16_rn(val);
        h[e] = *reinterpret_cast<const uint16_t*>(&b);
      }
    }
    uint16_t* dst = out + (size_t)row * D + lane * kPer;
    if constexpr (kPer == 4) {
      *reinterpret_cast<uint2*>(dst) =
          make_uint2(h[0] | (uint32_t(h[1]) << 16), h[2] | (uint32_t(h[3]) << 16));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = h[0] | (uint32_t(h[1]) << 16);
    }
  }
}

// O = 0 and lse = -inf for every row (a problem whose rows see no key at all).
__global__ void fill_lse_kernel(float* lse, size_t rows) {
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < rows) lse[i] = -INFINITY;
}

// y = 2^x through poly_ex2 (test hook for the FMA-pipe exponential).
__global__ void poly_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, size_t n) {
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < n) y[i] = poly_ex2(x[i]);
}

}  // namespace attn
