// Fused attention forward for sm_100a: O = softmax(scale * Q K^T + mask) V.
//
// The method is the one all the source pages turn on (flash attention over
// key/value tiles with an online softmax; "perf(metal): widen four-row flash
// KV tiles - #89", "Summary"), laid out for Blackwell:
//
//  * one CTA owns NQT query tiles of 128 rows of one (batch, kv-head) "unit";
//    the rows of the query heads that share a kv head (GQA) are stacked, so a
//    unit has R = (Hq/Hkv) * Sq rows and row r is query head g = r / Sq,
//    position start_pos + r % Sq;
//  * warp 0 streams Q once and K/V tiles of 128 keys through a ring of
//    shared-memory slots with TMA (128-byte swizzle, no multicast);
//  * one thread of warp 1 issues the tcgen05 MMAs: S = Q K^T into tensor
//    memory (TMEM), then O += P V with P read from TMEM, O accumulated in TMEM;
//  * one warpgroup per query tile runs the softmax: each thread owns one row
//    (tcgen05.ld 32x32b), applies the causal / window / length masks on
//    boundary tiles only, keeps the running max and sum in base 2, writes P
//    back over S in TMEM, and rescales O in TMEM only when the row max grew by
//    more than a threshold (the final division uses the same stale max, so the
//    result is unchanged);
//  * the epilogue divides O by the row sum and stores it with TMA (or, in the
//    split-KV variant, writes float32 partials and base-2 log-sum-exp for the
//    merge kernel; qsa2 audit, "implementation and review").
//
// Quantised variant (QUANT): Q/K are INT8 codes with one float32 scale per
// 128-token block (kind::i8 MMA, s32 accumulators), P is E4M3 scaled by 2^7,
// V^T is E4M3 with per-channel scales (kind::f8f6f4 MMA); this is the
// "INT8 QK · FP8 PV" form of the table in section "1 · Только ядро" of the page
// "Ядра attention на домашней RTX 5080".
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "ptx.cuh"
#include "rope.cuh"

namespace attn {

struct FwdArgs {
  int R;           // stacked query rows per unit: (Hq/Hkv) * Sq
  int Sq;          // query rows per head
  int Skv;         // keys
  int G;           // query heads per kv head
  int units;       // batch * Hkv
  int row_tiles;   // ceil(R / (NQT*128))
  int splits;      // key splits per row tile (split variant)
  int tiles_per_split;
  int start_pos;
  int causal;
  int window_lo;
  int window_size;  // sliding window W (0: none): row at position p sees keys >= p - W + 1
  // Paged K/V (exact mode): if block_table is set, key tile t of batch entry b is
  // block block_table[b * bt_stride + t] of a pool [blocks][n_kv_heads][128][D],
  // and the K/V tensor maps are 4-D over that pool.
  const int* block_table;
  int bt_stride;
  int n_kv_heads;
  // Causal, single-pass kernel, whole row tiles per head (q_len a multiple of 256):
  // row tiles per head.  The grid then runs all row tiles of one position band
  // (the band nearest the end of the sequence first) before the next band, across
  // every unit and head, so the heaviest CTAs start first.  0: unit-major order.
  int tph;
  float scale_log2;  // scale * log2(e)
  float* lse;        // [units * R] natural-log lse or nullptr (non-split variant)
  // Split variant: CTA b works on 128-row tile tile0 + b / splits (tiles numbered
  // unit-major over the whole problem) and key split b % splits.  Its partial rows are
  // the rows part_row0 .. part_row0 + part_rows - 1 of the problem (unit-major).
  int tile0;
  int part_row0;
  int part_rows;
  float* o_part;     // [splits, part_rows, D] float32 (split variant)
  float* lse_part;   // [2, splits, part_rows] base-2 lse of the P.V weights, then of the
                     // float32 weights (split variant)
  const float* q_scale;  // quantised variant
  const float* k_scale;
  const float* v_scale;
  int nblk_q;
  int nblk_k;
  unsigned* err;     // device error word
  unsigned debug;    // bit 0: skip the second key tile (timeout test)
  // RoPE (exact mode, ROPE variant): the staged Q tile is rotated in shared
  // memory before the first Q K^T; row r of a unit at position start_pos + r % Sq.
  const float* rope_table;  // [n_pos][2][rope_R/2] float32
  int rope_R;               // rotated channels (multiple of 16)
  int rope_inter;           // interleaved pairs
  // FP4 mode: E8M0 scale chunks (512 bytes per 128-row tile) of Q, per unit
  // [units][q_tiles], and of K, per unit [units][nblk_k]
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  int q_tiles;
};

// DIAG (quantised mode only): the key tiles of the causal diagonal band get
// Q K^T from the 16-bit inputs; 16-bit Q tiles sit next to the INT8 ones and one
// 16-bit K tile buffer serves the band tiles (the ring carries the rest).
// FP4 (quantised mode, head_dim 64): Q and K are packed E2M1 (half a byte per
// element) with E8M0 scale chunks (512 bytes per 128-row tile) that the MMA warp
// copies into tensor memory; a K slot holds the tile and, after it, its chunk.
template <int D, int NQT, bool QUANT, bool SPLIT, bool DIAG = false, bool FP4 = false>
struct FwdCfg {
  static_assert(!DIAG || (QUANT && !SPLIT), "the diagonal band mode is a single-pass quantised kernel");
  static_assert(!FP4 || (QUANT && !SPLIT && !DIAG && D == 64), "the FP4 mode: single pass, head_dim 64");
  static constexpr int kThreads = 128 * (1 + NQT);
  static constexpr int kElem = QUANT ? 1 : 2;                 // bytes per Q/K element
  static constexpr int kQTile = FP4 ? 128 * D / 2 : 128 * D * kElem;  // one 128-row Q tile
  static constexpr int kKTile = FP4 ? 128 * D / 2 : 128 * D * kElem;
  static constexpr int kSfChunk = 512;                        // FP4: scales of a 128-row tile
  static constexpr int kKSlotBytes = kKTile + (FP4 ? kSfChunk : 0);
  static constexpr int kVTile = 128 * D * (QUANT ? 1 : 2);
  static constexpr int kSlot = kKSlotBytes > kVTile ? kKSlotBytes : kVTile;
  static constexpr int kOStage = 128 * D * 2;                 // 16-bit output tile
  static constexpr int kQ16Tile = DIAG ? 128 * D * 2 : 0;     // 16-bit Q tile (DIAG)
  static constexpr int kKdBytes = DIAG ? 128 * D * 2 : 0;     // 16-bit K tile (DIAG)
  static constexpr bool kStageInQ = (kQTile >= kOStage);
  static constexpr int kStageBytes = (SPLIT || kStageInQ || DIAG) ? 0 : NQT * kOStage;
  static constexpr int kSfaBytes = FP4 ? NQT * kSfChunk : 0;  // FP4: Q tiles' scale chunks
  static constexpr int kFixed = NQT * (kQTile + kQ16Tile) + kKdBytes + kStageBytes + kSfaBytes;
  // (the band mode's extra 16-bit tiles would leave a 4-slot ring at 200 KB; it takes
  // up to 224 KB of the 227 KB a CTA may use, for 6 slots at head_dim 128)
  static constexpr int kBudget = (DIAG ? 224 : 200) * 1024;
  static constexpr int kNSraw = (kBudget - kFixed) / kSlot;
  // The split-KV variant serves few-row (decode) problems whose CTAs each see a
  // short key range: two K/V slots suffice, so that two CTAs share an SM.
  static constexpr int kNS = SPLIT ? 2 : (kNSraw > 8 ? 8 : kNSraw);
  static constexpr int kCtasPerSm = SPLIT ? 2 : 1;
  static_assert(kNS >= 2, "ring too small");
  static constexpr int kQOff = 0;
  static constexpr int kQ16Off = NQT * kQTile;                // DIAG: 16-bit Q tiles
  static constexpr int kKdOff = kQ16Off + NQT * kQ16Tile;     // DIAG: 16-bit K tile
  // output staging: its own buffers, or the Q tiles (16-bit Q tiles in DIAG)
  static constexpr int kStageOff = DIAG ? kQ16Off : NQT * kQTile;
  static constexpr int kSfaOff = kStageOff + kStageBytes;     // FP4 (after the staging)
  static constexpr int kStageTile = DIAG ? kQ16Tile : (kStageInQ ? kQTile : kOStage);
  static constexpr bool kStageInQBuf = kStageInQ && !DIAG;
  static constexpr int kRingOff = kFixed;
  static constexpr int kBarOff = kRingOff + kNS * kSlot;
  // barriers: q_full, full[NS], empty[NS], s_ready[NQT], p_ready[NQT][2] (one per
  // 64-key half of P), o_final, q_rot (RoPE: the staged Q has been rotated),
  // kd_full, kd_empty (DIAG: the 16-bit K tile buffer)
  static constexpr int kNumBars = 1 + 2 * kNS + 3 * NQT + 4;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;      // tmem base, abort flag
  static constexpr int kSvOff = kMiscOff + 16;                  // v scales (quant)
  static constexpr int kSmemBytes = kSvOff + (QUANT ? D * 4 : 0) + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "more shared memory than a CTA may have");
  // FP4: 4 scale-factor columns per Q tile and two K buffers after S and O
  static constexpr int kSfCols = FP4 ? 4 * NQT + 8 : 0;
  static constexpr int kTmemNeed = NQT * (128 + D) + kSfCols;
  static constexpr int kTmemCols = kTmemNeed <= 256 ? 256 : 512;
  // transaction bytes
  static constexpr uint32_t kQBytes = NQT * (kQTile + kQ16Tile) + kSfaBytes;
  static constexpr uint32_t kKBytes = kKSlotBytes;
  static constexpr uint32_t kVBytes = kVTile;
  // softmax rescale threshold (base-2 units): O and l are rescaled only when a
  // row max grows by more than this, so P <= 2^thresh.  Quantised: P is scaled by
  // 2^kPScale before the E4M3 cast and 2^(kPScale + thresh) = 2^8.8 ~ 445 stays
  // within the largest finite E4M3 value (448).  A larger threshold means fewer
  // rescales; the smaller factor only moves the E4M3 subnormal floor of P from
  // 2^-16 to 2^-14 relative to the running max (video, quantised: 15.41 ms with
  // 2^7 and 1.8, 15.02 ms with 2^5 and 3.8; the outputs' error is unchanged).
  static constexpr float kRescaleThresh = QUANT ? 3.8f : 8.0f;
  static constexpr float kPScale = QUANT ? 5.0f : 0.0f;
  // Registers per thread at launch (65536 / (threads * CTAs per SM), rounded
  // down to a multiple of 8) and their split between warpgroups: the
  // loader/MMA warpgroup needs few, the softmax warpgroups many.
  static constexpr int kRegsLaunch = (65536 / (kThreads * kCtasPerSm)) / 8 * 8;
  static constexpr int kRegsLow = NQT == 2 ? 88 : 56;
  static constexpr int kRegsHigh = NQT == 2 ? 208 : 200;
};

template <bool F16>
__device__ __forceinline__ uint32_t pack_16x2(float lo, float hi) {
  if constexpr (F16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

template <bool F16>
__device__ __forceinline__ void unpack_16x2(uint32_t v, float& lo, float& hi) {
  if constexpr (F16) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&v));
    lo = f.x;
    hi = f.y;
  } else {
    lo = __uint_as_float(v << 16);
    hi = __uint_as_float(v & 0xFFFF0000u);
  }
}

// Share of the exponentials that run on the FMA pipe (poly_ex2x2) instead of the
// MUFU, on key tiles without masked scores: one pair in this many (0: none).
// Measured on the video workload, every share tried (1/4, 1/8, 1/16) was slower
// than none in both modes: the polynomial's extra instructions cost more issue
// slots than the MUFU time they free.
constexpr int kPolyEvery = 0;   // exact mode
constexpr int kPolyEveryQ = 0;  // quantised mode

// Per-tile row-sum accumulators of one softmax thread: r[] adds the 16-bit P
// values that P.V multiplies (exact mode), f0/f1 the float32 P values.
struct RowSums {
  float r[4];
  f32x2 f0, f1;
};

// P = 2^(x * c - m) for one half (64 keys) of a 128-key row, written over S in
// tensor memory as 16-bit pairs (exact) or E4M3 quads (quantised), and added to
// the row sums.  `cm` = {c, c}, `mm` = {-m, -m}; in the quantised mode x holds
// the int32 scores' bits (offset by 1.5 * 2^23 into a float here), and mm
// already subtracts that offset times c.  POLY: one pair in POLY takes the FMA
// pipe exponential (0: all on the MUFU).  LF: keep the float32 sum (exact mode;
// the quantised mode always keeps it, it is its only sum).  `mid` runs in the
// second half once its first 32 keys are computed and before they are stored:
// the hand-off of the first half waits for that half's stores to complete, and
// by then they have.
// FS (quantised mode, diagonal band tiles): x holds float32 scores already.
template <bool F16, bool QUANT, int POLY, bool LF, int H, bool FS = false, typename Mid>
__device__ __forceinline__ void softmax_emit_half(const float (&x)[128], f32x2 cm, f32x2 mm,
                                                  uint32_t tS, RowSums& rs, Mid&& mid) {
#pragma unroll
  for (int ch = 2 * H; ch < 2 * H + 2; ++ch) {
    if constexpr (QUANT) {
      // x holds the int32 scores' bits; adding 0x4B400000 gives 1.5 * 2^23 + s exactly
      auto sc = [](float v) {
        return FS ? v : __uint_as_float(__float_as_uint(v) + 0x4B400000u);
      };
      uint32_t pk[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int e = 32 * ch + 4 * c;
        const f32x2 t0 = ffma2(f32x2{sc(x[e]), sc(x[e + 1])}, cm, mm);
        const f32x2 t1 = ffma2(f32x2{sc(x[e + 2]), sc(x[e + 3])}, cm, mm);
        f32x2 p01, p23;
        if (POLY > 0 && ((2 * c) % (POLY > 0 ? POLY : 1)) == 0) {
          p01 = poly_ex2x2(t0);
        } else {
          p01.x = ex2(t0.x);
          p01.y = ex2(t0.y);
        }
        p23.x = ex2(t1.x);
        p23.y = ex2(t1.y);
        pk[c] = uint32_t(f32x2_to_e4m3x2(p01.x, p01.y)) |
                (uint32_t(f32x2_to_e4m3x2(p23.x, p23.y)) << 16);
        rs.f0 = fadd2(rs.f0, p01);
        rs.f1 = fadd2(rs.f1, p23);
      }
      if (ch == 2) mid();
      tmem_st8(tS + 8 * ch, pk);
    } else {
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int e = 32 * ch + 2 * c;
        const f32x2 t = ffma2(f32x2{x[e], x[e + 1]}, cm, mm);
        f32x2 p;
        if (POLY > 0 && (c % (POLY > 0 ? POLY : 1)) == 0) {
          p = poly_ex2x2(t);
        } else {
          p.x = ex2(t.x);
          p.y = ex2(t.y);
        }
        pk[c] = pack_16x2<F16>(p.x, p.y);
        if (c & 1)
          add_16x2<F16>(pk[c], rs.r[2], rs.r[3]);
        else
          add_16x2<F16>(pk[c], rs.r[0], rs.r[1]);
        if constexpr (LF) {
          if (c & 1)
            rs.f1 = fadd2(rs.f1, p);
          else
            rs.f0 = fadd2(rs.f0, p);
        }
      }
      if (ch == 2) mid();
      tmem_st16(tS + 16 * ch, pk);
    }
  }
}

// Rotates one row of a staged 16-bit Q tile in shared memory (RoPE): the tile is
// 128 rows in boxes of 64 channels, 128-byte rows with 16-byte chunk k of row r
// at chunk position k ^ (r & 7) (the TMA 128-byte swizzle).  Each chunk of the
// first R channels is rotated with its partner chunk (rope.cuh); the half layout
// handles both chunks of a pair at once.
template <int D, bool F16>
__device__ __forceinline__ void rope_q_row(uint32_t tile, int row, const float* table, int R,
                                           bool inter, int pos) {
  auto addr = [&](int cj) {  // chunk cj (channels 8 cj .. 8 cj + 7) of this row
    return tile + (cj >> 3) * (128 * 128) + row * 128 + (((cj & 7) ^ (row & 7)) << 4);
  };
  auto ld = [](uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
  };
  // (no memory clobber: the table loads of later chunks may be issued early; the
  // caller's proxy fence orders these stores before the tensor core reads them)
  auto st = [](uint32_t a, const uint4& v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w));
  };
  const int n = inter ? R / 8 : R / 16;
  // unrolled over the most chunks a row can have, so that the table loads of
  // several chunks are in flight together
  constexpr int kMaxChunks = D / 8;
#pragma unroll
  for (int cj = 0; cj < kMaxChunks; ++cj) {
    if (cj >= n) break;
    const int pj = rope_partner(cj, R, inter);
    const uint4 a = ld(addr(cj));
    const uint4 b = inter ? a : ld(addr(pj));
    float fa[8];
    rope_chunk<F16>(a, b, cj, table, R, inter, pos, fa);
    if (!inter) {
      float fb[8];
      rope_chunk<F16>(b, a, pj, table, R, false, pos, fb);
      st(addr(pj), rope_pack8<F16>(fb));
    }
    st(addr(cj), rope_pack8<F16>(fa));
  }
}

// LF: the kernel also keeps the float32 row sum for the log-sum-exp (exact mode;
// needed by the split variant and when the caller asks for lse).  WIN: the
// per-row sliding window (window_size) is applied; the kernels without it keep
// the bounds they need in fewer registers.  ROPE (exact mode): the softmax
// warpgroups rotate the staged Q tile before the first Q K^T (the keys arrive
// rotated).
template <int D, int NQT, bool QUANT, bool F16, bool SPLIT, bool LF, bool WIN, bool ROPE,
          bool DIAG = false, bool FP4 = false>
__global__ void __launch_bounds__(FwdCfg<D, NQT, QUANT, SPLIT, DIAG, FP4>::kThreads,
                                  FwdCfg<D, NQT, QUANT, SPLIT, DIAG, FP4>::kCtasPerSm)
    flash_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_o,
                     const __grid_constant__ CUtensorMap tm_q16,
                     const __grid_constant__ CUtensorMap tm_k16, const FwdArgs a) {
  using C = FwdCfg<D, NQT, QUANT, SPLIT, DIAG, FP4>;
  static_assert(!SPLIT || LF, "the split variant always needs the float32 row sum");
  static_assert(!(ROPE && QUANT), "the quantised mode rotates Q and K in its quantiser");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---------------------------------------------------------- work decode
  int u, t, split = 0;
  {
    int lin = blockIdx.x;
    if constexpr (SPLIT) {
      split = lin % a.splits;
      lin = lin / a.splits + a.tile0;
    }
    if (!SPLIT && a.causal && a.tph > 0) {
      const int per_band = a.units * a.G;  // row tiles of one position band
      const int band = lin / per_band, rem = lin % per_band;
      const int g = rem % a.G;             // heads of a unit adjacent: they share K/V
      u = rem / a.G;
      t = g * a.tph + (a.tph - 1 - band);
    } else {
      u = lin / a.row_tiles;
      t = lin % a.row_tiles;
      if (!SPLIT && a.causal) t = a.row_tiles - 1 - t;  // heaviest tiles of a unit first
    }
  }
  const int BM = NQT * 128;
  const int r0 = t * BM;
  const int r_last = min(r0 + BM, a.R) - 1;
  int pos_min, pos_max;
  if (r0 / a.Sq != r_last / a.Sq) {
    pos_min = a.start_pos;
    pos_max = a.start_pos + a.Sq - 1;
  } else {
    pos_min = a.start_pos + r0 % a.Sq;
    pos_max = a.start_pos + r_last % a.Sq;
  }
  // Lowest key any row of the CTA sees, and the highest of the rows' lower bounds
  // (key tiles below it hold masked keys for some row).
  const int W = WIN ? a.window_size : 0;  // folded away in the kernels without a window
  const int kv_lo = W > 0 ? max(a.window_lo, pos_min - W + 1) : a.window_lo;
  const int kv_lo_max = W > 0 ? max(a.window_lo, pos_max - W + 1) : a.window_lo;
  const int kv_hi = a.causal ? min(a.Skv - 1, pos_max) : a.Skv - 1;
  int jt0 = 0, jt1 = 0;  // absolute key-tile range [jt0, jt1)
  if (kv_hi >= kv_lo) {
    jt0 = kv_lo / 128;
    jt1 = kv_hi / 128 + 1;
    if constexpr (SPLIT) {
      const int b0 = jt0 + split * a.tiles_per_split;
      jt1 = min(jt1, b0 + a.tiles_per_split);
      jt0 = b0;
      if (jt0 > jt1) jt0 = jt1;
    }
  }
  const int n = jt1 - jt0;

  // ------------------------------------------------------------ set-up
  auto bar = [&](int i) { return sbase + C::kBarOff + 8 * i; };
  const uint32_t q_full = bar(0);
  auto full_bar = [&](int s) { return bar(1 + s); };
  auto empty_bar = [&](int s) { return bar(1 + C::kNS + s); };
  auto s_ready = [&](int q) { return bar(1 + 2 * C::kNS + q); };
  auto p_ready = [&](int q, int h) { return bar(1 + 2 * C::kNS + NQT + 2 * q + h); };
  const uint32_t o_final = bar(1 + 2 * C::kNS + 3 * NQT);
  const uint32_t q_rot = bar(2 + 2 * C::kNS + 3 * NQT);
  const uint32_t kd_full = bar(3 + 2 * C::kNS + 3 * NQT);
  const uint32_t kd_empty = bar(4 + 2 * C::kNS + 3 * NQT);
  // DIAG: key tile j (absolute tile index jt) lies in the causal diagonal band of
  // this CTA when some of its rows must mask part of it for causality; its Q K^T
  // uses the 16-bit inputs.  The loader, the MMA warp and the softmax evaluate the
  // same predicate.
  auto in_band = [&](int jt) { return DIAG && a.causal && (jt * 128 + 127 > pos_min); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  float* sv_smem = reinterpret_cast<float*>(smem + C::kSvOff);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kNS; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int q = 0; q < NQT; ++q) {
      mbar_init(s_ready(q), 1);
      mbar_init(p_ready(q, 0), 4);  // one arrive per softmax warp
      mbar_init(p_ready(q, 1), 4);
    }
    mbar_init(o_final, 1);
    mbar_init(q_rot, 4 * NQT);  // one arrive per softmax warp
    mbar_init(kd_full, 1);
    mbar_init(kd_empty, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (QUANT) {
    if (warp == 2)
      for (int c = lane; c < D; c += 32) sv_smem[c] = a.v_scale[(size_t)u * D + c];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // Split variant: the merge kernel may be scheduled now; it waits for this
  // grid's completion (and memory flush) before reading the partials.
  if constexpr (SPLIT) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Two-tile variant: 384 threads launched at 168 registers each (64512).  The
  // loader/MMA warpgroup needs few, the softmax warpgroups many:
  // 128 x 88 + 256 x 208 = 64512, exactly the launch budget.
  static_assert(128 * C::kRegsLow + (C::kThreads - 128) * C::kRegsHigh <=
                    C::kThreads * C::kRegsLaunch,
                "register split exceeds the launch allocation");

  auto raise = [&]() {
    *abort_flag = 1;
    atomicOr(a.err, (unsigned)kErrTimeout);
  };

  if (warp < 4) {
  regs_dec<C::kRegsLow>();
  if (warp == 0) {
    // ======================================================== TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      constexpr int kBoxCols = FP4 ? D / 2 : (QUANT ? D : 64);  // box row (elements, FP4 bytes)
      constexpr int kQBoxes = QUANT ? 1 : D / 64;
      constexpr int kQBox = FP4 ? C::kQTile : 128 * kBoxCols * C::kElem;
      mbar_arrive_expect_tx(q_full, C::kQBytes);
      for (int q = 0; q < NQT; ++q)
        for (int bx = 0; bx < kQBoxes; ++bx)
          tma_load_3d(&tm_q, sbase + C::kQOff + q * C::kQTile + bx * kQBox, q_full,
                      bx * kBoxCols, r0 + q * 128, u);
      if constexpr (FP4) {  // the Q tiles' scale chunks (every unit has an even count)
        for (int q = 0; q < NQT; ++q)
          bulk_load(sbase + C::kSfaOff + q * C::kSfChunk,
                    a.q_sf + ((size_t)u * a.q_tiles + r0 / 128 + q) * C::kSfChunk, C::kSfChunk,
                    q_full);
      }
      if constexpr (DIAG) {  // the 16-bit Q tiles, for the band's Q K^T
        prefetch_tmap(&tm_q16);
        prefetch_tmap(&tm_k16);
        for (int q = 0; q < NQT; ++q)
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_3d(&tm_q16, sbase + C::kQ16Off + q * C::kQ16Tile + bx * 128 * 64 * 2,
                        q_full, bx * 64, r0 + q * 128, u);
      }
      int last_issue[C::kNS];
      for (int s = 0; s < C::kNS; ++s) last_issue[s] = -1;
      int it = 0;
      int kd_it = 0;  // DIAG: 16-bit K tiles loaded
      bool ok = true;
      // Paged K/V: this unit's row of the block table; each tile's block id is read
      // one tile ahead, so the read does not delay the tile's copies.
      const bool paged = !QUANT && a.block_table != nullptr;
      const int* bt_row =
          paged ? a.block_table + (size_t)(u / a.n_kv_heads) * a.bt_stride + jt0 : nullptr;
      int blk_next = (paged && n > 0) ? __ldg(bt_row) : 0;
      for (int j = 0; j < n && ok; ++j) {
        const int kv0 = (jt0 + j) * 128;
        const int blk = blk_next;
        if (paged && j + 1 < n) blk_next = __ldg(bt_row + j + 1);
        for (int part = 0; part < 2 && ok; ++part, ++it) {  // 0: K tile, 1: V tile
          if (part == 0 && in_band(jt0 + j)) {
            // DIAG: the band's K tile in 16 bits, into its own buffer (no ring slot)
            if (!mbar_wait(kd_empty, (kd_it & 1) ^ 1, abort_flag)) { raise(); ok = false; break; }
            mbar_arrive_expect_tx(kd_full, C::kKdBytes);
            for (int bx = 0; bx < D / 64; ++bx)
              tma_load_3d(&tm_k16, sbase + C::kKdOff + bx * 128 * 64 * 2, kd_full, bx * 64, kv0,
                          u);
            ++kd_it;
            --it;  // undone by the loop's increment: the ring was not used
            continue;
          }
          const int s = it % C::kNS;
          const uint32_t ph = (it / C::kNS) & 1;
          if (!mbar_wait(empty_bar(s), ph ^ 1, abort_flag)) { raise(); ok = false; break; }
          if ((a.debug & 1u) && j == 1 && part == 0) continue;  // timeout test: never load
          const uint32_t dst = sbase + C::kRingOff + s * C::kSlot;
          if (paged) {
            // the tile is one whole block of the pool (an id outside the pool reads
            // TMA's zero fill, never memory outside it)
            const int hk = u % a.n_kv_heads;
            const CUtensorMap* m = part == 0 ? &tm_k : &tm_v;
            mbar_arrive_expect_tx(full_bar(s), part == 0 ? C::kKBytes : C::kVBytes);
            for (int bx = 0; bx < D / 64; ++bx)
              tma_load_4d(m, dst + bx * 128 * 64 * 2, full_bar(s), bx * 64, 0, hk, blk);
          } else if (part == 0) {
            mbar_arrive_expect_tx(full_bar(s), C::kKBytes);
            if constexpr (FP4) {  // the packed tile, then its scale chunk after it
              tma_load_3d(&tm_k, dst, full_bar(s), 0, kv0, u);
              bulk_load(dst + C::kKTile, a.k_sf + ((size_t)u * a.nblk_k + jt0 + j) * C::kSfChunk,
                        C::kSfChunk, full_bar(s));
            } else if constexpr (QUANT) {
              tma_load_3d(&tm_k, dst, full_bar(s), 0, kv0, u);
            } else {
              for (int bx = 0; bx < D / 64; ++bx)
                tma_load_3d(&tm_k, dst + bx * 128 * 64 * 2, full_bar(s), bx * 64, kv0, u);
            }
          } else {
            mbar_arrive_expect_tx(full_bar(s), C::kVBytes);
            if constexpr (QUANT) {
              tma_load_3d(&tm_v, dst, full_bar(s), kv0, 0, u);   // V^T: [D rows, 128 keys]
            } else {
              for (int bx = 0; bx < D / 64; ++bx)
                tma_load_3d(&tm_v, dst + bx * 128 * 64 * 2, full_bar(s), bx * 64, kv0, u);
            }
          }
          last_issue[s] = it;
        }
      }
      // Never leave with copies in flight into this CTA's shared memory.
      {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(q_full, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
      for (int s = 0; s < C::kNS; ++s)
        if (last_issue[s] >= 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait_sleep(full_bar(s), (last_issue[s] / C::kNS) & 1) &&
                 globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      if (kd_it > 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_sleep(kd_full, (kd_it - 1) & 1) &&
               globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ========================================================= MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t fmt = F16 ? 0u : 1u;
      constexpr uint32_t idesc_qk =
          QUANT ? instr_desc(2, 1, 1, 0, 0, 128, 128) : instr_desc(1, fmt, fmt, 0, 0, 128, 128);
      constexpr uint32_t idesc_pv =
          QUANT ? instr_desc(1, 0, 0, 0, 0, 128, D) : instr_desc(1, fmt, fmt, 0, 1, 128, D);
      bool ok = mbar_wait(ROPE ? q_rot : q_full, 0, abort_flag);
      if (!ok) raise();
      int it = 0;
      if constexpr (FP4) {  // the Q tiles' scale factors, once
        if (ok) {
          tc_fence_after();
          for (int q = 0; q < NQT; ++q)
            tmem_cp_32x128b_x4(tmem + NQT * (128 + D) + 4 * q,
                               desc_pack(desc_lo(sbase + C::kSfaOff + q * C::kSfChunk, 16),
                                         desc_hi(128u, 0u)));
        }
      }

      // Descriptor words: the high word is fixed per operand kind; the low word
      // is the start address (>> 4) plus a compile-time offset per K step.
      constexpr uint32_t hi_qk =
          QUANT ? desc_hi(D == 128 ? 1024u : 512u, D == 128 ? 2u : 4u) : desc_hi(1024u, 2u);
      constexpr uint32_t hi_v = desc_hi(1024u, 2u);
      constexpr uint32_t lbo_v = QUANT ? 16u : 128u * 128u;  // exact: 64-column halves of V
      const uint32_t q_lo0 = desc_lo(sbase + C::kQOff, 16);
      const uint32_t ring_lo = desc_lo(sbase + C::kRingOff, 16);
      const uint32_t ring_lo_v = desc_lo(sbase + C::kRingOff, lbo_v);
      // DIAG: Q K^T of a band tile from the 16-bit Q tile and K buffer (f32 scores)
      constexpr uint32_t idesc_qk16 = instr_desc(1, fmt, fmt, 0, 0, 128, 128);
      constexpr uint32_t hi_16 = desc_hi(1024u, 2u);
      const uint32_t q16_lo0 = desc_lo(sbase + C::kQ16Off, 16);
      const uint32_t kd_lo = desc_lo(sbase + C::kKdOff, 16);
      auto issue_qk16 = [&](int q) {
        const uint32_t q_lo = q16_lo0 + q * (C::kQ16Tile >> 4);
        const uint32_t d = tmem + q * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 2;  // (64-col box, 32 B) >> 4
          mma_f16_ss(d, desc_pack(q_lo + off, hi_16), desc_pack(kd_lo + off, hi_16), idesc_qk16,
                     kk > 0);
        }
      };
      int kd_it = 0;  // band K tiles consumed
      // FP4: block-scaled MXFP4 Q K^T (K = 64 = the whole row of 32 bytes, 32-byte
      // swizzle, SBO 256).  Scale factors in tensor memory after S and O: the Q tiles'
      // (copied once) and two K buffers (copied per tile, alternating).
      constexpr uint32_t idesc_qk4 = instr_desc_mx(1, 1, 128, 128);
      constexpr uint32_t hi_4 = desc_hi(256u, 6u);
      const uint32_t sf_col = tmem + NQT * (128 + D);
      int k_sf_it = 0;
      auto copy_k_sf = [&](int slot) {  // the K tile's chunk, behind the tile in its slot
        const uint32_t src = sbase + C::kRingOff + slot * C::kSlot + C::kKTile;
        tmem_cp_32x128b_x4(sf_col + 4 * NQT + 4 * (k_sf_it & 1),
                           desc_pack(desc_lo(src, 16), desc_hi(128u, 0u)));
      };
      auto issue_qk = [&](int q, uint32_t k_lo) {
        const uint32_t q_lo = q_lo0 + q * (C::kQTile >> 4);
        const uint32_t d = tmem + q * 128;
        if constexpr (FP4) {
          mma_mxf4_ss(d, desc_pack(q_lo, hi_4), desc_pack(k_lo, hi_4), idesc_qk4, sf_col + 4 * q,
                      sf_col + 4 * NQT + 4 * (k_sf_it & 1), 0u);
        } else if constexpr (QUANT) {
          // int8, K = D bytes per row: one swizzle atom column (128 B, or 64 B at D = 64)
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8_ss(d, desc_pack(q_lo + kk * 2, hi_qk), desc_pack(k_lo + kk * 2, hi_qk),
                      idesc_qk, kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 2;  // (64-col box, 32 B) >> 4
            mma_f16_ss(d, desc_pack(q_lo + off, hi_qk), desc_pack(k_lo + off, hi_qk), idesc_qk,
                       kk > 0);
          }
        }
      };
      // O += P V over one 64-key half h of the tile (P columns of that half).
      auto issue_pv = [&](int q, int h, uint32_t v_lo, uint32_t accum) {
        const uint32_t d = tmem + NQT * 128 + q * D;
        const uint32_t p = tmem + q * 128;
        if constexpr (QUANT) {
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {  // 32 keys (8 columns of 4 e4m3) per step
            const int kk = 2 * h + k2;
            mma_f8_ts(d, p + kk * 8, desc_pack(v_lo + kk * 2, hi_v), idesc_pv, (accum | kk) != 0);
          }
        } else {
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {  // 16 keys (8 columns of 2 x 16-bit) per step
            const int kk = 4 * h + k2;
            mma_f16_ts(d, p + kk * 8, desc_pack(v_lo + kk * 128, hi_v), idesc_pv,
                       (accum | kk) != 0);
          }
        }
      };

      // S_0 for every query tile
      if (ok && in_band(jt0)) {
        ok = mbar_wait(kd_full, 0, abort_flag);
        if (!ok) raise();
        else {
          tc_fence_after();
          for (int q = 0; q < NQT; ++q) {
            issue_qk16(q);
            tc_commit(s_ready(q));
          }
          tc_commit(kd_empty);
          ++kd_it;
        }
      } else if (ok) {
        const int s = it % C::kNS;
        ok = mbar_wait(full_bar(s), (it / C::kNS) & 1, abort_flag);
        if (!ok) raise();
        else {
          tc_fence_after();
          const uint32_t k_lo = ring_lo + s * (C::kSlot >> 4);
          if constexpr (FP4) copy_k_sf(s);
          for (int q = 0; q < NQT; ++q) {
            issue_qk(q, k_lo);
            tc_commit(s_ready(q));
          }
          tc_commit(empty_bar(s));
          ++it;
          ++k_sf_it;
        }
      }
      for (int j = 0; j < n && ok; ++j) {
        const int sv = it % C::kNS;
        if (!mbar_wait(full_bar(sv), (it / C::kNS) & 1, abort_flag)) { raise(); ok = false; break; }
        ++it;
        const bool has_next = (j + 1 < n);
        const bool next_band = has_next && in_band(jt0 + j + 1);
        int sk = 0;
        if (next_band) {
          if (!mbar_wait(kd_full, kd_it & 1, abort_flag)) { raise(); ok = false; break; }
        } else if (has_next) {
          sk = it % C::kNS;
          if (!mbar_wait(full_bar(sk), (it / C::kNS) & 1, abort_flag)) { raise(); ok = false; break; }
          ++it;
        }
        tc_fence_after();
        const uint32_t v_lo = ring_lo_v + sv * (C::kSlot >> 4);
        const uint32_t k_lo = ring_lo + sk * (C::kSlot >> 4);
        if constexpr (FP4) {
          if (has_next && !next_band) copy_k_sf(sk);
        }
        for (int q = 0; q < NQT && ok; ++q) {
          // The first half of P.V runs while the softmax still writes the second.
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait(p_ready(q, h), j & 1, abort_flag)) { raise(); ok = false; break; }
            tc_fence_after();
            issue_pv(q, h, v_lo, j > 0);
          }
          if (!ok) break;
          if (q == NQT - 1) tc_commit(empty_bar(sv));
          if (next_band) {
            issue_qk16(q);
            tc_commit(s_ready(q));
          } else if (has_next) {
            issue_qk(q, k_lo);
            tc_commit(s_ready(q));
          }
        }
        if (ok && next_band) {
          tc_commit(kd_empty);
          ++kd_it;
        } else if (ok && has_next) {
          tc_commit(empty_bar(sk));
          ++k_sf_it;
        }
      }
      tc_commit(o_final);
      // Leave only once every issued MMA has finished (TMEM is freed at exit).
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait_sleep(o_final, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
  } else {
    regs_inc<C::kRegsHigh>();
    // ============================================================ softmax
    const int q = (warp - 4) >> 2;            // query tile of this warpgroup
    const int wq = warp & 3;                  // TMEM lane quarter
    const int row = wq * 32 + lane;
    const int r = r0 + q * 128 + row;
    const bool rvalid = r < a.R;
    const int ri = rvalid ? r : a.R - 1;
    const int i = ri % a.Sq;
    const int pos = a.start_pos + i;
    const int lo_r = W > 0 ? max(a.window_lo, pos - W + 1) : a.window_lo;
    const int hi_r = a.causal ? min(pos, a.Skv - 1) : a.Skv - 1;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + q * 128;
    const uint32_t tO = tmem + lane_off + NQT * 128 + q * D;
    float qsc = 1.0f;
    if constexpr (QUANT && !FP4) {  // (FP4: the scales are applied inside the MMA)
      const int g = ri / a.Sq;
      qsc = a.q_scale[((size_t)u * a.G + g) * a.nblk_q + i / 128];
    }

    float m_used = -INFINITY;  // running max of the base-2 scaled scores
    float l = 0.0f;            // row sum of the P values P.V uses (relative to m_used)
    float lf = 0.0f;           // row sum of the float32 P values (for lse)
    bool ok = true;
    // Quantised: the K block scale of tile j is loaded one tile ahead (a pinned
    // load, so that its latency hides behind the previous tile's softmax).
    const float* ksrc = (QUANT && !FP4) ? a.k_scale + (size_t)u * a.nblk_k + jt0 : nullptr;
    float ksc_next = 1.0f;
    if constexpr (QUANT && !FP4)
      if (n > 0) ksc_next = ld_global_f32(ksrc);
    constexpr int kPoly = QUANT ? kPolyEveryQ : kPolyEvery;
    if constexpr (ROPE) {
      // Rotate this thread's row of the staged Q tile, then hand the tile to the
      // MMA warp (generic-proxy writes made visible to the tensor core first).
      ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag));
      if (!ok) {
        if (lane == 0) raise();
      } else if (rvalid) {
        constexpr int kQBox = 128 * 64 * 2;
        static_assert(C::kQTile == (D / 64) * kQBox, "16-bit Q tile in 64-channel boxes");
        rope_q_row<D, F16>(sbase + C::kQOff + q * C::kQTile, row, a.rope_table, a.rope_R,
                           a.rope_inter != 0, pos);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_rot);
    }
    // Quantised scores arrive as int32 s; adding 0x4B400000 to the bits gives the
    // float F = 1.5 * 2^23 + s exactly (|s| < 2^22).  The offset is removed in the
    // maximum and folded into the exponent's FMA: 2^(F * c - K) with
    // K = 1.5 * 2^23 * c + m.  K is exact (so the FMA rounds s * c - m once, as a
    // plain conversion would) because c is trimmed to 21 significant bits (the
    // product with 3 * 2^22 then has at most 23) and the running max m is kept on
    // integers in this mode.
    constexpr float kMagic = QUANT ? 12582912.0f : 0.0f;
    auto to_score = [](uint32_t v) {
      return QUANT ? __uint_as_float(v + 0x4B400000u) : __uint_as_float(v);
    };
    // Hands one 64-key half of P to the MMA warp.
    auto p_half_done = [&](int h) {
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready(q, h));
    };
    if constexpr (!DIAG && !FP4) {
    // (the kernels without the band mode keep this straight-line form of the tile loop;
    // the band and FP4 modes below compile the tile body once per kind of score)
    for (int j = 0; j < n && ok; ++j) {
      const float ksc = ksc_next;
      if constexpr (QUANT)
        if (j + 1 < n) ksc_next = ld_global_f32(ksrc + j + 1);
      // raw score -> base-2 scaled score factor (quantised: kept positive so that
      // masked -inf scores stay -inf for an all-zero block); known before S lands
      const float cj =
          QUANT ? __uint_as_float(__float_as_uint(fmaxf(qsc * ksc * a.scale_log2, 1e-30f)) & ~7u)
                : a.scale_log2;
      ok = __all_sync(0xffffffffu, mbar_wait(s_ready(q), j & 1, abort_flag));
      if (!ok) { if (lane == 0) raise(); break; }
      tc_fence_after();
      const int kv0 = (jt0 + j) * 128;
      const bool need_mask =
          (kv0 < kv_lo_max) || (kv0 + 128 > a.Skv) || (a.causal && kv0 + 127 > pos_min);
      // S is read in two 64-column halves: the second half's load overlaps the
      // masking and maximum of the first.  Row max: four chains of three-input maxima.
      // Quantised: x keeps the int32 scores' bits, the row max runs on the integers
      // (eight chains) and the float offset is added in the emit; a masked score is
      // the bit pattern that the offset turns into -inf (below every real score).
      constexpr uint32_t kMaskedBits = 0xFF800000u - 0x4B400000u;
      const float masked = QUANT ? __uint_as_float(kMaskedBits) : -INFINITY;
      float x[128];
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      constexpr int kIntMin = -2147483647 - 1;
      int mi[8] = {kIntMin, kIntMin, kIntMin, kIntMin, kIntMin, kIntMin, kIntMin, kIntMin};
      auto row_max = [&](int c0) {
#pragma unroll
        for (int c = c0; c < c0 + 64; c += 8) {
          if constexpr (QUANT) {
#pragma unroll
            for (int e = 0; e < 8; ++e) mi[e] = max(mi[e], static_cast<int>(__float_as_uint(x[c + e])));
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) m4[e] = fmax3(m4[e], x[c + 2 * e], x[c + 2 * e + 1]);
          }
        }
      };
      {
        uint32_t s0[32], s1[32];
        tmem_ld32(tS + 0, s0);
        tmem_ld32(tS + 32, s1);
        tmem_ld_wait(s0);
        tmem_ld_wait(s1);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = __uint_as_float(s0[c]);
          x[32 + c] = __uint_as_float(s1[c]);
        }
      }
      uint32_t s2[32], s3[32];
      tmem_ld32(tS + 64, s2);
      tmem_ld32(tS + 96, s3);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int kj = kv0 + c;
          if (kj < lo_r || kj > hi_r) x[c] = masked;
        }
      }
      row_max(0);
      tmem_ld_wait(s2);
      tmem_ld_wait(s3);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        x[64 + c] = __uint_as_float(s2[c]);
        x[96 + c] = __uint_as_float(s3[c]);
      }
      if (need_mask) {
#pragma unroll
        for (int c = 64; c < 128; ++c) {
          const int kj = kv0 + c;
          if (kj < lo_r || kj > hi_r) x[c] = masked;
        }
      }
      row_max(64);
      float mx;
      if constexpr (QUANT) {
        int mr = max(max(max(mi[0], mi[1]), max(mi[2], mi[3])),
                     max(max(mi[4], mi[5]), max(mi[6], mi[7])));
        mx = to_score(static_cast<uint32_t>(mr)) - kMagic;  // exact; -inf if all masked
      } else {
        mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
      }
      const float m_tile = mx * cj;  // cj > 0; -inf stays -inf
      const float m_prev = m_used;
      const float m_new = fmaxf(m_prev, m_tile);
      const bool need = (m_prev != -INFINITY) && (m_new > m_prev + C::kRescaleThresh);
      if (m_prev == -INFINITY || need) m_used = QUANT ? ceilf(m_new) : m_new;
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? ex2(m_prev - m_used) : 1.0f;
        l *= f;
        lf *= f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c0, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
          tmem_st32(tO + c0, o);
        }
      }
      // P = 2^(x * cj - m)  (quantised: times 2^7 before the E4M3 cast), written
      // over S in two 64-key halves; the MMA warp starts on the first half while
      // the second is computed.  Exact mode: the row sum l adds the 16-bit values
      // that the P.V product actually uses, so O is a convex combination of V rows;
      // lf adds the float32 values (for lse).  On tiles without masked keys a share
      // of the exponentials run on the FMA pipe (poly_ex2x2).
      const float mb = (m_used == -INFINITY ? 0.0f : m_used) - C::kPScale;
      const float kq = QUANT ? fmaf(kMagic, cj, mb) : mb;  // quantised: offset folded in
      const f32x2 cm{cj, cj}, mm{-kq, -kq};
      RowSums rs{{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f}, {0.0f, 0.0f}};
      auto none = [] {};
      auto first_half_done = [&] { p_half_done(0); };
      if (need_mask) {
        softmax_emit_half<F16, QUANT, 0, LF, 0>(x, cm, mm, tS, rs, none);
        softmax_emit_half<F16, QUANT, 0, LF, 1>(x, cm, mm, tS, rs, first_half_done);
      } else {
        softmax_emit_half<F16, QUANT, kPoly, LF, 0>(x, cm, mm, tS, rs, none);
        softmax_emit_half<F16, QUANT, kPoly, LF, 1>(x, cm, mm, tS, rs, first_half_done);
      }
      p_half_done(1);
      const float fsum = (rs.f0.x + rs.f0.y) + (rs.f1.x + rs.f1.y);
      if constexpr (QUANT) {
        l += fsum;
        lf += fsum;
      } else {
        l += (rs.r[0] + rs.r[1]) + (rs.r[2] + rs.r[3]);
        if constexpr (LF) lf += fsum;
      }
    }
    } else {
    for (int j = 0; j < n && ok; ++j) {
      const float ksc = ksc_next;
      if constexpr (QUANT && !FP4)
        if (j + 1 < n) ksc_next = ld_global_f32(ksrc + j + 1);
      // DIAG: a band tile's scores are float32 products of the 16-bit inputs; FP4:
      // every tile's are (block-scaled MMA)
      const bool band = in_band(jt0 + j);
      // The tile's body, compiled once per kind of score: FS (the diagonal band
      // mode's band tiles) reads float32 scores, otherwise INT8 products (quantised)
      // or float32 (exact).  Separate copies keep each one's registers to itself.
      auto tile = [&](auto fs_tag) -> bool {
        constexpr bool FS = decltype(fs_tag)::value;
        // raw score -> base-2 scaled score factor (quantised: kept positive so that
        // masked -inf scores stay -inf for an all-zero block); known before S lands
        const float cj =
            (QUANT && !FS)
                ? __uint_as_float(__float_as_uint(fmaxf(qsc * ksc * a.scale_log2, 1e-30f)) & ~7u)
                : a.scale_log2;
        bool ok2 = __all_sync(0xffffffffu, mbar_wait(s_ready(q), j & 1, abort_flag));
        if (!ok2) {
          if (lane == 0) raise();
          return false;
        }
        tc_fence_after();
        const int kv0 = (jt0 + j) * 128;
        const bool need_mask =
            (kv0 < kv_lo_max) || (kv0 + 128 > a.Skv) || (a.causal && kv0 + 127 > pos_min);
        // S is read in two 64-column halves: the second half's load overlaps the
        // masking and maximum of the first.  Row max: four chains of three-input maxima.
        // Quantised: x keeps the int32 scores' bits, the row max runs on the integers
        // (eight chains) and the float offset is added in the emit; a masked score is
        // the bit pattern that the offset turns into -inf (below every real score).
        constexpr uint32_t kMaskedBits = 0xFF800000u - 0x4B400000u;
        const float masked = (QUANT && !FS) ? __uint_as_float(kMaskedBits) : -INFINITY;
        float x[128];
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        constexpr int kIntMin = -2147483647 - 1;
        int mi[8] = {kIntMin, kIntMin, kIntMin, kIntMin, kIntMin, kIntMin, kIntMin, kIntMin};
        auto row_max = [&](int c0) {
  #pragma unroll
          for (int c = c0; c < c0 + 64; c += 8) {
            if (QUANT && !FS) {
  #pragma unroll
              for (int e = 0; e < 8; ++e) mi[e] = max(mi[e], static_cast<int>(__float_as_uint(x[c + e])));
            } else {
  #pragma unroll
              for (int e = 0; e < 4; ++e) m4[e] = fmax3(m4[e], x[c + 2 * e], x[c + 2 * e + 1]);
            }
          }
        };
        {
          uint32_t s0[32], s1[32];
          tmem_ld32(tS + 0, s0);
          tmem_ld32(tS + 32, s1);
          tmem_ld_wait(s0);
          tmem_ld_wait(s1);
  #pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = __uint_as_float(s0[c]);
            x[32 + c] = __uint_as_float(s1[c]);
          }
        }
        uint32_t s2[32], s3[32];
        tmem_ld32(tS + 64, s2);
        tmem_ld32(tS + 96, s3);
        if (need_mask) {
  #pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int kj = kv0 + c;
            if (kj < lo_r || kj > hi_r) x[c] = masked;
          }
        }
        row_max(0);
        tmem_ld_wait(s2);
        tmem_ld_wait(s3);
  #pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[64 + c] = __uint_as_float(s2[c]);
          x[96 + c] = __uint_as_float(s3[c]);
        }
        if (need_mask) {
  #pragma unroll
          for (int c = 64; c < 128; ++c) {
            const int kj = kv0 + c;
            if (kj < lo_r || kj > hi_r) x[c] = masked;
          }
        }
        row_max(64);
        float mx;
        if (QUANT && !FS) {
          int mr = max(max(max(mi[0], mi[1]), max(mi[2], mi[3])),
                       max(max(mi[4], mi[5]), max(mi[6], mi[7])));
          mx = to_score(static_cast<uint32_t>(mr)) - kMagic;  // exact; -inf if all masked
        } else {
          mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
        }
        const float m_tile = mx * cj;  // cj > 0; -inf stays -inf
        const float m_prev = m_used;
        const float m_new = fmaxf(m_prev, m_tile);
        const bool need = (m_prev != -INFINITY) && (m_new > m_prev + C::kRescaleThresh);
        if (m_prev == -INFINITY || need) m_used = QUANT ? ceilf(m_new) : m_new;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? ex2(m_prev - m_used) : 1.0f;
          l *= f;
          lf *= f;
  #pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
            tmem_ld_wait(o);
  #pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
            tmem_st32(tO + c0, o);
          }
        }
        // P = 2^(x * cj - m)  (quantised: times 2^7 before the E4M3 cast), written
        // over S in two 64-key halves; the MMA warp starts on the first half while
        // the second is computed.  Exact mode: the row sum l adds the 16-bit values
        // that the P.V product actually uses, so O is a convex combination of V rows;
        // lf adds the float32 values (for lse).  On tiles without masked keys a share
        // of the exponentials run on the FMA pipe (poly_ex2x2).
        const float mb = (m_used == -INFINITY ? 0.0f : m_used) - C::kPScale;
        const float kq = (QUANT && !FS) ? fmaf(kMagic, cj, mb) : mb;  // int scores: offset folded in
        const f32x2 cm{cj, cj}, mm{-kq, -kq};
        RowSums rs{{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f}, {0.0f, 0.0f}};
        auto none = [] {};
        auto first_half_done = [&] { p_half_done(0); };
        if constexpr (FS) {
          softmax_emit_half<F16, QUANT, 0, LF, 0, true>(x, cm, mm, tS, rs, none);
          softmax_emit_half<F16, QUANT, 0, LF, 1, true>(x, cm, mm, tS, rs, first_half_done);
        } else if (need_mask) {
          softmax_emit_half<F16, QUANT, 0, LF, 0>(x, cm, mm, tS, rs, none);
          softmax_emit_half<F16, QUANT, 0, LF, 1>(x, cm, mm, tS, rs, first_half_done);
        } else {
          softmax_emit_half<F16, QUANT, kPoly, LF, 0>(x, cm, mm, tS, rs, none);
          softmax_emit_half<F16, QUANT, kPoly, LF, 1>(x, cm, mm, tS, rs, first_half_done);
        }
        p_half_done(1);
        const float fsum = (rs.f0.x + rs.f0.y) + (rs.f1.x + rs.f1.y);
        if constexpr (QUANT) {
          l += fsum;
          lf += fsum;
        } else {
          l += (rs.r[0] + rs.r[1]) + (rs.r[2] + rs.r[3]);
          if constexpr (LF) lf += fsum;
        }
        return true;
      };
      if constexpr (FP4) {
        ok = tile(std::true_type{});
      } else {
        if (DIAG && band)
          ok = tile(std::true_type{});
        else
          ok = tile(std::false_type{});
      }
    }
    }

    // ----------------------------------------------------------- epilogue
    if (ok && n > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(o_final, 0, abort_flag));
      if (!ok && lane == 0) raise();
      tc_fence_after();
    } else if (n == 0) {
      // No key tile: the Q copy (whose buffer stages the output) must have landed.
      ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag));
      if (!ok && lane == 0) raise();
    }
    const bool have_o = ok && n > 0;
    const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
    // base-2 log-sum-exp: of the weights P.V used (merge weights) and of the
    // float32 weights (the reported lse)
    const float lse2_w = (l > 0.0f) ? m_used + lg2(l) - C::kPScale : -INFINITY;
    const float lse2 = (lf > 0.0f) ? m_used + lg2(lf) - C::kPScale : -INFINITY;
    if constexpr (SPLIT) {
      const size_t prow = (size_t)split * a.part_rows + ((size_t)u * a.R + r - a.part_row0);
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(tO + c0, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        if (rvalid) {
          float4* dst = reinterpret_cast<float4*>(a.o_part + prow * D + c0);
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            float4 v;
            float sv0 = 1.f, sv1 = 1.f, sv2 = 1.f, sv3 = 1.f;
            if constexpr (QUANT) {
              sv0 = sv_smem[c0 + c];
              sv1 = sv_smem[c0 + c + 1];
              sv2 = sv_smem[c0 + c + 2];
              sv3 = sv_smem[c0 + c + 3];
            }
            v.x = __uint_as_float(o[c]) * inv * sv0;
            v.y = __uint_as_float(o[c + 1]) * inv * sv1;
            v.z = __uint_as_float(o[c + 2]) * inv * sv2;
            v.w = __uint_as_float(o[c + 3]) * inv * sv3;
            dst[c / 4] = v;
          }
        }
      }
      if (rvalid) {
        a.lse_part[prow] = lse2_w;
        a.lse_part[(size_t)a.splits * a.part_rows + prow] = lse2;
      }
    } else {
      const uint32_t stage = C::kStageInQBuf ? sbase + C::kQOff + q * C::kQTile
                                             : sbase + C::kStageOff + q * C::kStageTile;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(tO + c0, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float v0 = __uint_as_float(o[2 * c]) * inv;
          float v1 = __uint_as_float(o[2 * c + 1]) * inv;
          if constexpr (QUANT) {
            v0 *= sv_smem[c0 + 2 * c];
            v1 *= sv_smem[c0 + 2 * c + 1];
          }
          pk[c] = pack_16x2<F16>(v0, v1);
        }
        // 128-byte swizzled box of 64 columns: 16-byte chunk k of row r sits at k ^ (r & 7)
        const uint32_t box = stage + (c0 / 64) * (128 * 128);
        const int cb = (c0 % 64) / 8;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t addr = box + row * 128 + (((cb + k) ^ (row & 7)) * 16);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * k]),
                       "r"(pk[4 * k + 1]), "r"(pk[4 * k + 2]), "r"(pk[4 * k + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + q, 128);
      if (row == 0 && !*abort_flag && r0 + q * 128 < a.R) {
        for (int bx = 0; bx < D / 64; ++bx)
          tma_store_3d(&tm_o, stage + bx * (128 * 128), bx * 64, r0 + q * 128, u);
        bulk_commit();
        bulk_wait_all();
      }
      if (rvalid && a.lse != nullptr) a.lse[(size_t)u * a.R + r] = lse2 * 0.69314718055994531f;
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace attn
