// Per-block quantisers of the opt-in reduced-precision mode ("SageAttention 2
// INT8 QK · FP8 PV" row of the table in section "1 · Только ядро" of the page
// "Ядра attention на домашней RTX 5080"; its ~14 ms of data preparation next to
// a 42 ms kernel is why these kernels must run at HBM speed).
//
//  * Q and K: one float32 scale per (b, h, 128-token block):
//      s = amax / 127,  code = clamp(rint_half_even(x / s), -127, 127).
//  * V: one float32 scale per (b, hkv, channel) over all tokens:
//      s = amax / 448,  code = E4M3(v / s), nearest-even, saturating,
//    written transposed [b, hkv, channel, token] (zero padded to 128 tokens)
//    so that it is the K-major operand of the P.V MMA.
// Every arithmetic step is one correctly rounded float32 operation, so the
// codes are reproducible bit for bit.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "rope.cuh"

namespace attn {

template <bool F16>
__device__ __forceinline__ void unpack8(const uint4& w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if constexpr (F16) {
      const __half2 h = *reinterpret_cast<const __half2*>(&u[k]);
      f[2 * k] = __low2float(h);
      f[2 * k + 1] = __high2float(h);
    } else {
      const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&u[k]);
      f[2 * k] = __low2float(h);
      f[2 * k + 1] = __high2float(h);
    }
  }
}

template <bool F16>
__device__ __forceinline__ void unpack_16x2_v(uint32_t w, float& lo, float& hi) {
  if constexpr (F16) {
    const __half2 h = *reinterpret_cast<const __half2*>(&w);
    lo = __low2float(h);
    hi = __high2float(h);
  } else {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
  }
}

// x / s correctly rounded (the float32 division) from the block's reciprocal:
// y = RN(x * r) with r = RN(1/s) is within an ulp of x / s, the residual
// x - y * s is exact under one fused multiply-add, and RN(y + residual * r) is
// the correctly rounded quotient (Markstein's theorem on division through a
// correctly rounded reciprocal; Markstein, IBM J. Res. Dev. 34(1), 1990).
// Valid while s, 1/s and the quotient stay normal, which the callers check
// block-wide (else they use the plain division).
// The sign is copied from x (s > 0): the correction step would turn -0 into +0.
__device__ __forceinline__ float div_by_recip(float x, float s, float r) {
  const float y = x * r;
  const float e = fmaf(-y, s, x);
  return copysignf(fmaf(e, r, y), x);
}

// True when div_by_recip(x, s, r) is exact for every |x| <= 127.5 * s (and for
// x = 0): s and 1/s comfortably inside the normal range.
__device__ __forceinline__ bool recip_ok(float s) {
  return s >= 1.0e-30f && s <= 1.0e30f;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Persistent: grid of a few CTAs per SM, 256 threads, each CTA walking the
// 128-token blocks b = blockIdx.x, blockIdx.x + gridDim.x, ...  A block of one
// (b, h) is contiguous (128 tokens x D, 16-bit), so one bulk copy brings it into
// shared memory; two buffers let the next block stream in while this one is
// reduced and quantised, keeping HBM busy.  Waits are bounded: on a timeout the
// CTA records kErrTimeout in `err` and stops.
//
// With ROPE the block is rotated first (rope.cuh: float32 operations on the
// table, token t of block b at position pos0 + 128 b + t): each thread rotates
// its chunks (reading the partner chunk of the pairs from shared memory), keeps
// the rotated floats in registers, and the maximum and the codes are those of
// the rotated values.  The extra registers leave room for fewer CTAs per SM.
// Where the 128-token blocks of a key or value tensor live: dense [units][S][D]
// (table == nullptr), or a paged pool [num_blocks][n_kv_heads][128][D] in which block
// table[b * bt_stride + t] holds tokens 128 t .. 128 t + 127 of batch entry b (unit
// u = b * n_kv_heads + h).  A block is contiguous either way.  A table entry outside
// [0, num_blocks) is read as block 0 and flagged (kErrBadBlock in *err): nothing is
// read outside the pool.
constexpr int kErrBadBlock = 2;  // error word bit (beside kErrTimeout)
struct KvBlocks {
  const int* table;
  int bt_stride;
  int n_kv_heads;
  int num_blocks;
  unsigned* err;
  template <int D>
  __device__ __forceinline__ const uint16_t* block(const uint16_t* base, size_t u, int t,
                                                   int S) const {
    if (table == nullptr) return base + (u * S + static_cast<size_t>(t) * 128) * D;
    const int b = static_cast<int>(u / n_kv_heads), h = static_cast<int>(u % n_kv_heads);
    int blk = __ldg(table + static_cast<size_t>(b) * bt_stride + t);
    if (blk < 0 || blk >= num_blocks) {
      atomicOr(err, (unsigned)kErrBadBlock);
      blk = 0;
    }
    return base + (static_cast<size_t>(blk) * n_kv_heads + h) * 128 * D;
  }
};

template <int D, bool ROPE = false>
struct QuantQkCfg {
  static constexpr int kBlockBytes = 128 * D * 2;
  static constexpr int kSmemBytes = 2 * kBlockBytes + 64 + 128;  // buffers, barriers, reduction
  static constexpr int kCtasPerSm = D == 128 ? (ROPE ? 2 : 3) : (ROPE ? 3 : 6);
};

// RoPE arguments of the quantiser (unused without ROPE).
struct QuantRope {
  const float* table;  // [n_pos][2][R/2] float32
  int R;               // rotated channels
  int inter;           // interleaved pairs
  int pos0;            // position of token 0
};

template <int D, bool F16, bool ROPE = false>
__global__ void __launch_bounds__(256, QuantQkCfg<D, ROPE>::kCtasPerSm) quant_qk_kernel(
    const uint16_t* __restrict__ x, int8_t* __restrict__ codes, float* __restrict__ scales, int S,
    int nblk, int total, unsigned* err, unsigned debug, QuantRope rope, KvBlocks src) {
  using C = QuantQkCfg<D, ROPE>;
  constexpr int kChunks = 128 * D / 8;  // 16-byte chunks of a full block
  constexpr int kPer = kChunks / 256;
  extern __shared__ __align__(128) uint8_t qsm[];
  const uint32_t sbase = smem_u32(qsm);
  const uint32_t bar0 = sbase + 2 * C::kBlockBytes;
  float* red = reinterpret_cast<float*>(qsm + 2 * C::kBlockBytes + 64);
  volatile int* stop = reinterpret_cast<volatile int*>(qsm + 2 * C::kBlockBytes + 32);
  if (threadIdx.x == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    *stop = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto block_bytes = [&](int b) {
    const int t = b % nblk;
    return (uint32_t)(min(128, S - t * 128) * D * 2);
  };
  auto issue = [&](int b, int stage) {  // thread 0
    const size_t bh = b / nblk;
    const int t = b % nblk;
    const uint32_t bytes = block_bytes(b);
    mbar_arrive_expect_tx(bar0 + 8 * stage, bytes);
    bulk_load(sbase + stage * C::kBlockBytes, src.block<D>(x, bh, t, S), bytes, bar0 + 8 * stage);
  };
  if (threadIdx.x == 0) {
    if (blockIdx.x < total) issue(blockIdx.x, 0);
    // timeout test (bit 1): CTA 0 never loads its second block
    if (blockIdx.x + gridDim.x < total && !((debug & 2u) && blockIdx.x == 0))
      issue(blockIdx.x + gridDim.x, 1);
  }
  int it = 0;
  for (int b = blockIdx.x; b < total; b += gridDim.x, ++it) {
    const int stage = it & 1;
    const uint32_t bar = bar0 + 8 * stage;
    if (!__all_sync(0xffffffffu, mbar_wait(bar, (it >> 1) & 1, stop))) {
      if ((threadIdx.x & 31) == 0) {
        *stop = 1;
        atomicOr(err, 1u);
      }
      break;
    }
    const size_t bh = b / nblk;
    const int t = b % nblk;
    const int nelem = min(128, S - t * 128) * D;
    const uint4* src = reinterpret_cast<const uint4*>(qsm + stage * C::kBlockBytes);
    uint4 w[kPer];
    float rv[ROPE ? kPer : 1][8];  // rotated values (ROPE)
    float amax = 0.0f;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int c = threadIdx.x + k * 256;
      if (c * 8 < nelem) {
        w[k] = src[c];
        if constexpr (ROPE) {
          constexpr int kCpr = D / 8;  // chunks per token
          const int tok = c / kCpr, cj = c % kCpr;
          const int pj = rope_partner(cj, rope.R, rope.inter != 0);
          const uint4 pw = src[tok * kCpr + pj];
          rope_chunk<F16>(w[k], pw, cj, rope.table, rope.R, rope.inter != 0,
                          rope.pos0 + t * 128 + tok, rv[k]);
#pragma unroll
          for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(rv[k][e]));
        } else {
          float f[8];
          unpack8<F16>(w[k], f);
#pragma unroll
          for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
        }
      } else {
        w[k] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();  // every thread holds its data: the buffer may be refilled
    if (threadIdx.x == 0 && b + 2 * gridDim.x < total) {
      fence_proxy_async_smem();  // the generic reads above come before the async refill
      issue(b + 2 * gridDim.x, stage);
    }
    amax = red[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) amax = fmaxf(amax, red[k]);

    const float s = __fdiv_rn(amax, 127.0f);
    if (threadIdx.x == 0) scales[bh * nblk + t] = s;
    const float r = __frcp_rn(s);
    const bool fast = recip_ok(s);
    const size_t base = (bh * S + (size_t)t * 128) * D;
    // code = rint_half_even(x / s).  |x| <= amax, so |x / s| <= 127 (1 + 2^-24) < 127.5
    // and the clamp to +-127 never acts; -0 and +0 both give code 0.  Fast path:
    // the correctly rounded quotient through the reciprocal (packed pairs), then
    // round-half-even by adding 1.5 * 2^23 (the integer lands in the low bits:
    // its low byte is the code).
    const f32x2 rr{r, r}, ns{-s, -s}, big{12582912.0f, 12582912.0f};
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int c = threadIdx.x + k * 256;
      if (c * 8 < nelem) {
        float f[8];
        if constexpr (ROPE) {
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = rv[k][e];
        } else {
          unpack8<F16>(w[k], f);
        }
        uint32_t bits[8];
        if (fast) {
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const f32x2 xv{f[e], f[e + 1]};
            const f32x2 y = fmul2(xv, rr);
            const f32x2 q = ffma2(ffma2(y, ns, xv), rr, y);  // Markstein correction
            const f32x2 m = fadd2(q, big);
            bits[e] = __float_as_uint(m.x);
            bits[e + 1] = __float_as_uint(m.y);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int qv = (s > 0.0f) ? max(-127, min(127, __float2int_rn(__fdiv_rn(f[e], s)))) : 0;
            bits[e] = static_cast<uint32_t>(qv);
          }
        }
        const uint32_t w0 = __byte_perm(__byte_perm(bits[0], bits[1], 0x0040),
                                        __byte_perm(bits[2], bits[3], 0x0040), 0x5410);
        const uint32_t w1 = __byte_perm(__byte_perm(bits[4], bits[5], 0x0040),
                                        __byte_perm(bits[6], bits[7], 0x0040), 0x5410);
        *reinterpret_cast<uint2*>(codes + base + (size_t)c * 8) = make_uint2(w0, w1);
      }
    }
    __syncthreads();  // red[] is rewritten by the next block
  }
  // Never leave with a copy in flight into this CTA's shared memory.
  if (threadIdx.x == 0) {
    for (int k = 0; k < 2; ++k) {
      const int b = blockIdx.x + (it + k) * gridDim.x;
      if (b < total) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(bar0 + 8 * ((it + k) & 1), ((it + k) >> 1) & 1) &&
               globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
    }
  }
}

// MXFP4 quantiser of the FP4 mode (head_dim 64), after the OCP Microscaling
// Formats conversion: per row and block of 32 channels, the E8M0 scale 2^e with
// e = floor(log2(amax)) - 2 (2 is the largest E2M1 exponent; clamped to
// [-127, 127]; amax = 0 gives e = -127), and codes E2M1(x * 2^-e) rounded to
// nearest-even and saturated to +-6 (cvt.rn.satfinite.e2m1x2).  x * 2^-e is an
// exact power-of-two scaling (a result that would be subnormal is far below
// E2M1's resolution and rounds to zero either way).
//
// Rows come as `nseq` sequences of L rows (Q: the G * Sq stacked rows of a unit;
// K: the keys of a (batch, kv head)); each sequence has `tiles` 128-row tiles
// (at least ceil(L / 128); rows past L are padding).  Block = one tile, thread =
// (row, channel block): codes [row][32 B] (channel 2i in the low nibble), scales
// in the tensor core's 512-byte chunk per tile: row r, block b at byte
// (r % 32) * 16 + (r / 32) * 4 + b; padding rows and the unused bytes b = 2, 3
// hold 127 (scale 1).
template <bool F16>
__global__ void __launch_bounds__(256) mxfp4_qk_kernel(const uint16_t* __restrict__ x,
                                                       uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ sf, int L, int tiles) {
  const int seq = blockIdx.y, t = blockIdx.x;
  const int r = threadIdx.x >> 1, b = threadIdx.x & 1;
  const int row = t * 128 + r;
  uint8_t* chunk = sf + ((size_t)seq * tiles + t) * 512 + (r & 31) * 16 + (r >> 5) * 4;
  if (row >= L) {
    chunk[b] = 127;
    chunk[2 + b] = 127;
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)seq * L + row) * 64 + 32 * b);
  float f[32];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float g[8];
    unpack8<F16>(ld_nc_v4(src + k), g);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[8 * k + e] = g[e];
  }
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(f[e]));
  int ex = amax > 0.0f ? ilogbf(amax) - 2 : -127;
  ex = max(-127, min(127, ex));
  chunk[b] = static_cast<uint8_t>(ex + 127);
  chunk[2 + b] = 127;
  const float inv = __int_as_float((127 - ex) << 23);  // 2^-ex, a normal float for ex <= 126
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 8 * k + 2 * i;
      uint16_t pair;
      // the first source lands in the high nibble: channel e + 1 high, e low
      asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
          : "=h"(pair)
          : "f"(__fmul_rn(f[e + 1], inv)), "f"(__fmul_rn(f[e], inv)));
      word |= static_cast<uint32_t>(pair & 0xFF) << (8 * i);
    }
    w[k] = word;
  }
  *reinterpret_cast<uint4*>(codes + ((size_t)seq * L + row) * 32 + 16 * b) =
      make_uint4(w[0], w[1], w[2], w[3]);
}

// grid: (ceil(S/kVTok), B*Hkv), 256 threads.  Channel maxima of |V| as float
// bit patterns (non-negative floats order like unsigned integers).
constexpr int kVTok = 256;

template <int D, bool F16>
__global__ void __launch_bounds__(256) v_amax_kernel(const uint16_t* __restrict__ v,
                                                     unsigned* __restrict__ amax_bits, int S,
                                                     KvBlocks src) {
  constexpr int kCC = D / 8;            // 16-byte chunks per token
  constexpr int kRows = 256 / kCC;      // tokens covered per pass
  __shared__ unsigned smax[D];
  for (int c = threadIdx.x; c < D; c += 256) smax[c] = 0u;
  __syncthreads();
  const size_t u = blockIdx.y;
  const int tok0 = blockIdx.x * kVTok;
  const int cc = threadIdx.x % kCC;
  float m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int tk = threadIdx.x / kCC; tk < kVTok; tk += kRows) {
    const int tok = tok0 + tk;
    if (tok < S) {
      float f[8];
      unpack8<F16>(ld_nc_v4(src.block<D>(v, u, tok / 128, S) + (tok % 128) * D + cc * 8), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) atomicMax(&smax[cc * 8 + e], __float_as_uint(m[e]));
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 256) atomicMax(&amax_bits[u * D + c], smax[c]);
}

// Quantise 128-token tiles of V and write them transposed.  Persistent, like
// quant_qk_kernel: tiles (unit u, tile t) in turn, each brought into shared
// memory by one bulk copy (a tile of one unit is contiguous) while the previous
// one is converted.  Thread (channel pair cp, token group tg) converts channels
// 2cp, 2cp + 1 for a run of tokens: each 32-bit shared load gives both channels
// of one token (a warp reads one token row without bank conflicts), divisions
// are paired along tokens, and each channel's codes leave as 16-byte stores of
// consecutive tokens.  s = amax / 448 per (u, channel); the code is the E4M3
// value of x / s (correctly rounded quotient, nearest even, saturating), with
// the sign of a zero following x; tokens past S and all-zero channels give 0.
template <int D>
struct VQuantCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kSmemBytes = 2 * kTileBytes + 64;
  static constexpr int kPairs = D / 2;              // channel pairs
  static constexpr int kGroups = 256 / kPairs;      // token groups
  static constexpr int kRun = 128 / kGroups;        // tokens per thread
  static constexpr int kCtasPerSm = D == 128 ? 3 : 6;
};

template <int D, bool F16>
__global__ void __launch_bounds__(256, VQuantCfg<D>::kCtasPerSm)
    v_quant_kernel(const uint16_t* __restrict__ v, const unsigned* __restrict__ amax_bits,
                   uint8_t* __restrict__ vt, float* __restrict__ v_scale, int S, int S_pad,
                   int nbk, int total, unsigned* err, KvBlocks src) {
  using C = VQuantCfg<D>;
  extern __shared__ __align__(128) uint8_t vsm[];
  const uint32_t sbase = smem_u32(vsm);
  const uint32_t bar0 = sbase + 2 * C::kTileBytes;
  volatile int* stop = reinterpret_cast<volatile int*>(vsm + 2 * C::kTileBytes + 32);
  if (threadIdx.x == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    *stop = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int b, int stage) {  // thread 0
    const size_t u = b / nbk;
    const int t = b % nbk;
    const uint32_t bytes = (uint32_t)(min(128, S - t * 128) * D * 2);
    mbar_arrive_expect_tx(bar0 + 8 * stage, bytes);
    bulk_load(sbase + stage * C::kTileBytes, src.block<D>(v, u, t, S), bytes,
              bar0 + 8 * stage);
  };
  if (threadIdx.x == 0) {
    if (blockIdx.x < total) issue(blockIdx.x, 0);
    if (blockIdx.x + gridDim.x < total) issue(blockIdx.x + gridDim.x, 1);
  }
  const int cp = threadIdx.x % C::kPairs;
  const int tg = threadIdx.x / C::kPairs;
  const int c0 = 2 * cp;
  int it = 0;
  for (int b = blockIdx.x; b < total; b += gridDim.x, ++it) {
    const int stage = it & 1;
    const size_t u = b / nbk;
    const int t = b % nbk;
    // scales of this thread's two channels
    const float s0 = __fdiv_rn(__uint_as_float(amax_bits[u * D + c0]), 448.0f);
    const float s1 = __fdiv_rn(__uint_as_float(amax_bits[u * D + c0 + 1]), 448.0f);
    if (t == 0 && tg == 0) {
      v_scale[u * D + c0] = s0;
      v_scale[u * D + c0 + 1] = s1;
    }
    const bool fast = recip_ok(s0) && recip_ok(s1);
    const float r0 = __frcp_rn(s0), r1 = __frcp_rn(s1);
    if (!__all_sync(0xffffffffu, mbar_wait(bar0 + 8 * stage, (it >> 1) & 1, stop))) {
      if ((threadIdx.x & 31) == 0) {
        *stop = 1;
        atomicOr(err, 1u);
      }
      break;
    }
    const int ntok = min(128, S - t * 128);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(vsm + stage * C::kTileBytes) + cp;
    const int tk0 = tg * C::kRun;
    uint32_t out0[C::kRun / 4], out1[C::kRun / 4];  // codes of channel c0, c0 + 1
#pragma unroll
    for (int i = 0; i < C::kRun; i += 2) {
      const int ta = tk0 + i, tb = tk0 + i + 1;
      const uint32_t wa = ta < ntok ? src[ta * (D / 2)] : 0u;
      const uint32_t wb = tb < ntok ? src[tb * (D / 2)] : 0u;
      float xa0, xa1, xb0, xb1;  // token a / b, channel c0 / c0 + 1
      unpack_16x2_v<F16>(wa, xa0, xa1);
      unpack_16x2_v<F16>(wb, xb0, xb1);
      float q0a = 0.0f, q0b = 0.0f, q1a = 0.0f, q1b = 0.0f;
      if (fast) {
        const f32x2 x0{xa0, xb0}, x1{xa1, xb1};
        const f32x2 y0 = fmul2(x0, f32x2{r0, r0}), y1 = fmul2(x1, f32x2{r1, r1});
        const f32x2 z0 = ffma2(ffma2(y0, f32x2{-s0, -s0}, x0), f32x2{r0, r0}, y0);
        const f32x2 z1 = ffma2(ffma2(y1, f32x2{-s1, -s1}, x1), f32x2{r1, r1}, y1);
        q0a = copysignf(z0.x, xa0);
        q0b = copysignf(z0.y, xb0);
        q1a = copysignf(z1.x, xa1);
        q1b = copysignf(z1.y, xb1);
      } else {
        if (s0 > 0.0f) {
          q0a = __fdiv_rn(xa0, s0);
          q0b = __fdiv_rn(xb0, s0);
        }
        if (s1 > 0.0f) {
          q1a = __fdiv_rn(xa1, s1);
          q1b = __fdiv_rn(xb1, s1);
        }
      }
      if (s0 <= 0.0f) q0a = q0b = 0.0f;
      if (s1 <= 0.0f) q1a = q1b = 0.0f;
      if (ta >= ntok) q0a = q1a = 0.0f;  // padding tokens: code 0x00
      if (tb >= ntok) q0b = q1b = 0.0f;
      const uint32_t h0 = f32x2_to_e4m3x2(q0a, q0b), h1 = f32x2_to_e4m3x2(q1a, q1b);
      if (i % 4 == 0) {
        out0[i / 4] = h0;
        out1[i / 4] = h1;
      } else {
        out0[i / 4] |= h0 << 16;
        out1[i / 4] |= h1 << 16;
      }
    }
    __syncthreads();  // every thread has read the tile: the buffer may be refilled
    if (threadIdx.x == 0 && b + 2 * gridDim.x < total) {
      fence_proxy_async_smem();
      issue(b + 2 * gridDim.x, stage);
    }
    uint8_t* d0 = vt + (u * D + c0) * (size_t)S_pad + (size_t)t * 128 + tk0;
    uint8_t* d1 = d0 + S_pad;
#pragma unroll
    for (int k = 0; k < C::kRun / 16; ++k) {
      reinterpret_cast<uint4*>(d0)[k] =
          make_uint4(out0[4 * k], out0[4 * k + 1], out0[4 * k + 2], out0[4 * k + 3]);
      reinterpret_cast<uint4*>(d1)[k] =
          make_uint4(out1[4 * k], out1[4 * k + 1], out1[4 * k + 2], out1[4 * k + 3]);
    }
  }
  // Never leave with a copy in flight into this CTA's shared memory.
  if (threadIdx.x == 0) {
    for (int k = 0; k < 2; ++k) {
      const int b = blockIdx.x + (it + k) * gridDim.x;
      if (b < total) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(bar0 + 8 * ((it + k) & 1), ((it + k) >> 1) & 1) &&
               globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
    }
  }
}

}  // namespace attn
