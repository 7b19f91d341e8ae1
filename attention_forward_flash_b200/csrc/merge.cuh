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

// grid: rows, 128 threads; one CTA per output row.  The partials of split sp and
// row r are at sp * stride + r (stride >= rows: a window of a larger partial
// buffer).  Every warp loads all
// splits' weight exponents (one per lane) together with the partial outputs of
// its own splits w, w + 4, ..., so that both arrive in one memory round trip;
// each warp then forms the maximum, its splits' weights and the denominator
// itself, and the four partial sums are added in shared memory.
template <int D, bool F16>
__global__ void __launch_bounds__(32 * kMergeWarps) splitkv_merge_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part,
    uint16_t* __restrict__ out, float* __restrict__ lse, int stride, int splits) {
  constexpr int kPer = D / 32;                    // channels per lane
  constexpr int kMaxPerWarp = kMergeMaxSplits / kMergeWarps;
  __shared__ float red[kMergeWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x;
  // Launched as a programmatic dependent of the split kernel: wait until that
  // grid has completed and its partials are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // this lane's share of the weight exponents (splits lane, lane + 32, ...)
  float W[kMergeMaxSplits / 32];
#pragma unroll
  for (int k = 0; k < kMergeMaxSplits / 32; ++k) {
    const int sp = lane + 32 * k;
    W[k] = sp < splits ? lse_part[(size_t)sp * stride + row] : -INFINITY;
  }
  // this warp's partial outputs, all loads in flight
  float part[kMaxPerWarp / 4][kPer];  // splits warp + 4 i, in groups processed below
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.0f;
  float M = -INFINITY, wsum = 0.0f;
  // splits warp + 4 i in groups of kMaxPerWarp / 4; the first group's loads are
  // issued before the weight exponents are used, so both are in flight together
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    const int i0 = g * (kMaxPerWarp / 4);
    if (g > 0 && warp + 4 * i0 >= splits) break;
#pragma unroll
    for (int i = 0; i < kMaxPerWarp / 4; ++i) {
      const int sp = warp + 4 * (i0 + i);
      const float* src = o_part + ((size_t)sp * stride + row) * D + lane * kPer;
      if (sp < splits) {
        if constexpr (kPer == 4) {
          const float4 v = *reinterpret_cast<const float4*>(src);
          part[i][0] = v.x; part[i][1] = v.y; part[i][2] = v.z; part[i][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(src);
          part[i][0] = v.x; part[i][1] = v.y;
        }
      }
    }
    if (g == 0) {
#pragma unroll
      for (int k = 0; k < kMergeMaxSplits / 32; ++k) M = fmaxf(M, W[k]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
#pragma unroll
      for (int k = 0; k < kMergeMaxSplits / 32; ++k)
        wsum += (M == -INFINITY || W[k] == -INFINITY) ? 0.0f : ex2(W[k] - M);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    }
#pragma unroll
    for (int i = 0; i < kMaxPerWarp / 4; ++i) {
      const int sp = warp + 4 * (i0 + i);
      // weight of split sp from the lane that holds its exponent (all lanes take part)
      const int k = sp >> 5;
      const float Wk = k == 0 ? W[0] : k == 1 ? W[1] : k == 2 ? W[2] : W[3];
      const float Ws = __shfl_sync(0xffffffffu, Wk, sp & 31);
      if (sp < splits) {
        const float w = (M == -INFINITY || Ws == -INFINITY) ? 0.0f : ex2(Ws - M);
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] += w * part[i][e];
      }
    }
  }
#pragma unroll
  for (int e = 0; e < kPer; ++e) red[warp][lane * kPer + e] = acc[e];
  if (warp == 1 && lse != nullptr) {
    const float* lf = lse_part + (size_t)splits * stride;
    float ML = -INFINITY, F[kMergeMaxSplits / 32];
#pragma unroll
    for (int k = 0; k < kMergeMaxSplits / 32; ++k) {
      const int sp = lane + 32 * k;
      F[k] = sp < splits ? lf[(size_t)sp * stride + row] : -INFINITY;
      ML = fmaxf(ML, F[k]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ML = fmaxf(ML, __shfl_xor_sync(0xffffffffu, ML, o));
    float ls = 0.0f;
#pragma unroll
    for (int k = 0; k < kMergeMaxSplits / 32; ++k)
      ls += (ML == -INFINITY || F[k] == -INFINITY) ? 0.0f : ex2(F[k] - ML);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    if (lane == 0) lse[row] = (ls > 0.0f) ? (ML + lg2(ls)) * 0.69314718055994531f : -INFINITY;
  }
  __syncthreads();
  if (warp == 0) {
    const float inv = (wsum > 0.0f) ? 1.0f / wsum : 0.0f;
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

// The same merge with one warp per row, for few splits (at most 32; the host takes
// it up to 16, e.g. the short last wave of the single-pass grid): grid
// ceil(rows / 4), 128 threads.
// Lane s holds split s's two weight exponents; each lane owns D / 32 channels and
// sums them over the splits, all partial loads of a split issued together.
template <int D, bool F16>
__global__ void __launch_bounds__(128) splitkv_merge_rows_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part,
    uint16_t* __restrict__ out, float* __restrict__ lse, int rows, int stride, int splits) {
  constexpr int kPer = D / 32;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float W = lane < splits ? lse_part[(size_t)lane * stride + row] : -INFINITY;
  const float F = lane < splits ? lse_part[(size_t)(splits + lane) * stride + row] : -INFINITY;
  float M = W, ML = F;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    ML = fmaxf(ML, __shfl_xor_sync(0xffffffffu, ML, o));
  }
  const float w = (M == -INFINITY || W == -INFINITY) ? 0.0f : ex2(W - M);
  const float f = (ML == -INFINITY || F == -INFINITY) ? 0.0f : ex2(F - ML);
  float wsum = w, fsum = f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    fsum += __shfl_xor_sync(0xffffffffu, fsum, o);
  }
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.0f;
  for (int sp = 0; sp < splits; ++sp) {
    const float ws = __shfl_sync(0xffffffffu, w, sp);
    const float* src = o_part + ((size_t)sp * stride + row) * D + lane * kPer;
    float v[kPer];
    if constexpr (kPer == 4) {
      const float4 t = *reinterpret_cast<const float4*>(src);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
      const float2 t = *reinterpret_cast<const float2*>(src);
      v[0] = t.x; v[1] = t.y;
    }
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] += ws * v[e];
  }
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  uint16_t h[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const float val = acc[e] * inv;
    if constexpr (F16) {
      const __half b = __float2half_rn(val);
      h[e] = *reinterpret_cast<const uint16_t*>(&b);
    } else {
      const __nv_bfloat16 b = __float2bfloat16_rn(val);
      h[e] = *reinterpret_cast<const uint16_t*>(&b);
    }
  }
  uint16_t* dst = out + (size_t)row * D + lane * kPer;
  if constexpr (kPer == 4)
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(h[0] | (uint32_t(h[1]) << 16), h[2] | (uint32_t(h[3]) << 16));
  else
    *reinterpret_cast<uint32_t*>(dst) = h[0] | (uint32_t(h[1]) << 16);
  if (lane == 0 && lse != nullptr)
    lse[row] = fsum > 0.0f ? (ML + lg2(fsum)) * 0.69314718055994531f : -INFINITY;
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
