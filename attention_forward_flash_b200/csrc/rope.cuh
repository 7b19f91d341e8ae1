// Rotary position embedding (RoPE) for the attention path.
//
// The page "Ядра attention на домашней RTX 5080" (section "Планы · Rigsy
// Kernel") plans RoPE with NTK / YaRN scaling inside the attention kernel
// instead of a separate pass.  Here the rotation runs where Q and K are already
// being read: the quantiser rotates each block before taking its maximum, and
// the exact-mode attention kernel rotates its staged Q tile in shared memory.
// rope_apply_kernel is the one stand-alone pass: keys written once into a cache,
// or the exact mode's keys before the kernel (each key tile is read by every
// query tile, so rotating it once beats rotating it in every CTA).
//
// Rotation of channel pair i at position p: with c = table[p][0][i] and
// s = table[p][1][i] (float32, the YaRN factor folded in),
//     a' = RN(RN(a c) - RN(b s)),   b' = RN(RN(a s) + RN(b c)),
// each product and sum one correctly rounded float32 operation (never fused),
// so every caller gets the same bits.  Pairs: (i, i + R/2) ("half" layout) or
// (2i, 2i + 1) (interleaved) over the first R channels; channels R .. D-1 are
// left as they are.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace attn {

__device__ __forceinline__ void rope_rotate(float& a, float& b, float c, float s) {
  const float na = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
  const float nb = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
  a = na;
  b = nb;
}

// 8 consecutive 16-bit values <-> floats (exact widening; RN narrowing).
template <bool F16>
__device__ __forceinline__ void rope_unpack8(const uint4& w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if constexpr (F16) {
      const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
      f[2 * k] = t.x;
      f[2 * k + 1] = t.y;
    } else {
      f[2 * k] = __uint_as_float(u[k] << 16);
      f[2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
    }
  }
}

template <bool F16>
__device__ __forceinline__ uint4 rope_pack8(const float (&f)[8]) {
  uint32_t u[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if constexpr (F16) {
      __half2 h = __floats2half2_rn(f[2 * k], f[2 * k + 1]);
      u[k] = *reinterpret_cast<uint32_t*>(&h);
    } else {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
      u[k] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

// cos and sin of pairs i .. i + N - 1 at position `pos` (N = 8 or 4; 16-byte
// aligned: R is a multiple of 16 and i a multiple of N).
template <int N>
__device__ __forceinline__ void rope_load(const float* __restrict__ table, int R, int pos, int i,
                                          float (&c)[N], float (&s)[N]) {
  const float4* pc = reinterpret_cast<const float4*>(table + (size_t)pos * R + i);
  const float4* ps = reinterpret_cast<const float4*>(table + (size_t)pos * R + R / 2 + i);
#pragma unroll
  for (int k = 0; k < N / 4; ++k) {
    const float4 a = __ldg(pc + k), b = __ldg(ps + k);
    c[4 * k] = a.x, c[4 * k + 1] = a.y, c[4 * k + 2] = a.z, c[4 * k + 3] = a.w;
    s[4 * k] = b.x, s[4 * k + 1] = b.y, s[4 * k + 2] = b.z, s[4 * k + 3] = b.w;
  }
}

// Rotates the 16-byte chunk `cj` (channels 8 cj .. 8 cj + 7) of one row, given the
// row's chunk and, in the half layout, its partner chunk (the other half of the
// pairs); writes the rotated floats of chunk cj to `out`.  Chunks at or past R
// are copied.  `mine` and `partner` are the raw 16-bit chunks.
template <bool F16>
__device__ __forceinline__ void rope_chunk(const uint4& mine, const uint4& partner, int cj,
                                           const float* __restrict__ table, int R, bool inter,
                                           int pos, float (&out)[8]) {
  rope_unpack8<F16>(mine, out);
  if (cj * 8 >= R) return;
  if (inter) {
    float c[4], s[4];
    rope_load<4>(table, R, pos, 4 * cj, c, s);
#pragma unroll
    for (int m = 0; m < 4; ++m) rope_rotate(out[2 * m], out[2 * m + 1], c[m], s[m]);
    return;
  }
  float other[8], c[8], s[8];
  rope_unpack8<F16>(partner, other);
  const bool lo = cj * 16 < R;  // first half: channel i pairs with i + R/2
  rope_load<8>(table, R, pos, lo ? 8 * cj : 8 * cj - R / 2, c, s);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float a = lo ? out[e] : other[e];
    float b = lo ? other[e] : out[e];
    rope_rotate(a, b, c[e], s[e]);
    out[e] = lo ? a : b;
  }
}

// Partner chunk of chunk cj in the half layout (itself in the interleaved one or
// past R).
__device__ __forceinline__ int rope_partner(int cj, int R, bool inter) {
  if (inter || cj * 8 >= R) return cj;
  return cj * 16 < R ? cj + R / 16 : cj - R / 16;
}

// y = RoPE(x) for `rows` rows of D channels ([..., len, D], row t of a head at
// position pos0 + t % len).  One thread per 16-byte chunk; in the half layout the
// thread of the first-half chunk writes both chunks of its pairs.
template <bool F16>
__global__ void __launch_bounds__(256) rope_apply_kernel(const uint16_t* __restrict__ x,
                                                         uint16_t* __restrict__ y,
                                                         const float* __restrict__ table,
                                                         long long rows, int len, int D, int R,
                                                         int inter, int pos0) {
  const int cpr = D / 8;  // chunks per row
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * cpr) return;
  const long long row = idx / cpr;
  const int cj = static_cast<int>(idx % cpr);
  const int pos = pos0 + static_cast<int>(row % len);
  const uint4* src = reinterpret_cast<const uint4*>(x + row * D);
  uint4* dst = reinterpret_cast<uint4*>(y + row * D);
  if (cj * 8 >= R) {  // not rotated: copied (nothing to do in place)
    if (x != y) dst[cj] = src[cj];
    return;
  }
  if (!inter && cj * 16 >= R) return;  // second-half chunk: written with its partner
  const int pj = rope_partner(cj, R, inter != 0);
  const uint4 a = src[cj];
  const uint4 b = src[pj];
  float fa[8];
  rope_chunk<F16>(a, b, cj, table, R, inter != 0, pos, fa);
  if (!inter) {
    float fb[8];
    rope_chunk<F16>(b, a, pj, table, R, false, pos, fb);
    dst[pj] = rope_pack8<F16>(fb);
  }
  dst[cj] = rope_pack8<F16>(fa);
}

}  // namespace attn
