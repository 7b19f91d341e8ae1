// Decode-shaped attention: few query rows per kv head (at most 16 stacked rows of
// a unit), exact mode.  The problem statement is that of the page "perf(metal):
// widen four-row flash KV tiles - #89" ("Performance evidence": a handful of
// query rows at a start position against a long key/value cache), and the split
// of the keys across workers with one merge that caches each chunk's maximum and
// weight is the qsa2 audit's ("round 21 track b -- qsa2", "implementation and
// review").
//
// Such a problem reads every key and value once and does 4 * rows * D flops per
// key, so it is bound by HBM and by the latency of getting the whole cache in
// flight, not by the tensor cores.  The layout here:
//
//  * one thread-block cluster per unit (batch entry, kv head); its CTAs split the
//    unit's visible key range into equal runs of 64-key (head_dim 64) or 32-key
//    (head_dim 128) chunks, so each chunk of K and V is 16 KB;
//  * each of a CTA's four warps is an independent flash-decoding worker: it
//    streams its own chunks (every fourth) with TMA into its own ring slots
//    (128-byte swizzle, no multicast), the first ones issued before Q is staged,
//    and computes the two products with warp-level mma.sync (m16n8k16, 16-bit
//    operands, float32 accumulators) and an online softmax in base 2 on the
//    accumulator fragments.  Up to 8 rows the products are transposed (S^T = K Q^T,
//    O^T = V^T P^T: keys and channels on the M = 16 side, the rows on N = 8; P^T
//    reaches the second product's operand by an in-register transpose); from 9 to
//    16 rows the rows are the M side and P goes from the S fragments to the A
//    operand in registers;
//  * each warp's partial result (running maximum m, the sum of the 16-bit P
//    values that entered P V, the float32 sum for the log-sum-exp, and O) is
//    stored straight into the shared memory of the CTA that owns the row (row r:
//    CTA r mod S) through distributed shared memory; after one cluster barrier
//    each owner combines the S * 4 partials of its rows with one denominator and
//    writes them.  No partials go through global memory and there is no second
//    launch.
//
// Masks: row r of a unit is query head r / Sq at position p = start_pos + r % Sq
// and sees the keys lo_r .. hi_r, lo_r = max(window_lo, p - W + 1 if W > 0),
// hi_r = min(kv_len - 1, p if causal); applied by selection on every chunk.  A row
// that sees no key gets O = 0 and lse = -inf.  Keys past kv_len read as zeros
// (dense: the tensor map's bounds) or are cleared in shared memory (a paged
// cache's last block may hold anything there).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "rope.cuh"

namespace attn {

struct DecArgs {
  const uint16_t* q;  // [units][R][D] (the unit's stacked rows)
  uint16_t* o;        // [units][R][D]
  float* lse;         // [units * R] natural-log lse, or nullptr
  int R;              // stacked rows per unit (<= 16)
  int Sq;
  int Skv;
  int start_pos;
  int causal;
  int window_lo;
  int window_size;
  int chunk0;    // first chunk of the union of the rows' visible ranges
  int n_chunks;  // chunks of that union (0: no row sees a key)
  float scale_log2;
  // paged key/value pools: key tile t of batch entry b is block
  // block_table[b * bt_stride + t] of a pool [blocks][n_kv_heads][128][D]
  const int* block_table;
  int bt_stride;
  int n_kv_heads;
  // RoPE on the staged Q rows (keys arrive rotated)
  const float* rope_table;  // [n_pos][2][rope_R/2] float32
  int rope_R;
  int rope_inter;
  unsigned* err;
  unsigned debug;  // bit 0: warp 0 of CTA 0 never loads its second chunk (timeout test)
  int nsw;          // ring slots per warp (2 .. DecCfg::kMaxNsw)
  int owner_slots;  // partial-row slots of the merge area (warps * S * ceil(R / S))
};

template <int D>
struct DecCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int kWarps = 4;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kMaxSplits = 16;                   // cluster size limit (non-portable)
  static constexpr int kChunk = D == 128 ? 32 : 64;       // keys per warp step
  static constexpr int kNT = kChunk / 8;                  // S n-tiles per chunk
  static constexpr int kBox = kChunk * 128;               // one TMA box: kChunk rows x 64 channels
  static constexpr int kHalfBoxes = D / 64;               // boxes per chunk of K (or V)
  static constexpr int kKVBytes = kHalfBoxes * kBox;      // one chunk of K (or V)
  static constexpr int kSlotBytes = 2 * kKVBytes;         // K then V: 16 KB
  static constexpr int kMaxNsw = 4;                       // ring slots per warp, at most
  // (the host takes 2: deeper rings measured slower on the decode workload)
  // Fixed area (compile-time offsets), then the ring, then the merge area, whose
  // sizes the host picks per problem (DecArgs::nsw, owner_slots):
  //   Q rows [16][kQStride] 16-bit | owner weights [16][64] and (M, L, LF) [16][4] |
  //   barriers [kWarps * kMaxNsw] | abort flag | pad | ring [kWarps * nsw][16 KB] |
  //   partial O rows [owner_slots][kMoStride] | partial (m, l, lf, -) [owner_slots]
  // Merge area: every warp of the cluster writes its partial result for each row
  // into the CTA that owns the row (row r: CTA r mod S), partial p = split * kWarps +
  // warp at row slot p * ceil(R/S) + r / S.  With R, S <= 16, S * ceil(R/S) <= 31.
  static constexpr int kQStride = D + 8;                  // staged Q row, 16-bit elements
  static constexpr int kQOff = 0;
  static constexpr int kWtOff = kQOff + 16 * kQStride * 2;
  static constexpr int kBarOff = kWtOff + 16 * 64 * 4 + 16 * 16;
  static constexpr int kMiscOff = kBarOff + 8 * kWarps * kMaxNsw;
  static constexpr int kRingOff = (kMiscOff + 16 + 1023) / 1024 * 1024;
  static constexpr int kMaxOwnerSlots = 31 * kWarps;
  static constexpr int kMoStride = D + 4;                 // floats per partial O row
  static constexpr int kOwnerSlotBytes = kMoStride * 4 + 16;
  static constexpr int kMaxSmem = 227 * 1024;
  // dynamic shared memory of a launch (+ 1 KB to align the base)
  static constexpr int smem_bytes(int nsw, int owner_slots) {
    return kRingOff + kWarps * nsw * kSlotBytes + owner_slots * kOwnerSlotBytes + 1024;
  }
  static_assert((kMoStride * 4) % 16 == 0 && kSlotBytes % 1024 == 0, "merge area alignment");
  static_assert(smem_bytes(2, kMaxOwnerSlots) <= kMaxSmem, "shared memory");
};

// ------------------------------------------------------- warp-level MMA, cluster
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// d += A (16x16, row) * B (16x8, col); 16-bit operands, float32 accumulators.
template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (F16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Split cluster barrier: arrive (no ordering) now, wait later.  Used once at the
// start so that no CTA writes into another's shared memory before that CTA runs.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
// Every thread of every CTA of the cluster arrives; shared-memory writes before
// the barrier are visible to the cluster's reads after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Transpose of an 8x8 16-bit matrix held one 32-bit pair per thread (row lane/4,
// columns 2 (lane%4), +1): afterwards each thread holds the same positions of the
// transpose.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// Stores into (possibly another CTA's) shared memory of the cluster.
__device__ __forceinline__ void st_dsmem(uint32_t addr, float a) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(a) : "memory");
}
__device__ __forceinline__ void st_dsmem_v2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b)
               : "memory");
}
__device__ __forceinline__ void st_dsmem_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

template <bool F16>
__device__ __forceinline__ uint32_t pack16x2(float lo, float hi) {
  if constexpr (F16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

template <bool F16>
__device__ __forceinline__ uint16_t to16(float x) {
  if constexpr (F16) {
    const __half h = __float2half_rn(x);
    return *reinterpret_cast<const uint16_t*>(&h);
  } else {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<const uint16_t*>(&h);
  }
}

template <bool F16>
__device__ __forceinline__ float from16(uint16_t u) {
  if constexpr (F16) return __half2float(*reinterpret_cast<const __half*>(&u));
  else return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

// Shared-memory address of 16-byte column chunk `cc` (0 .. D/8-1) of row `row` of
// a chunk of K or V staged as D/64 boxes of 128-byte rows, 128-byte swizzle.
template <int D>
__device__ __forceinline__ uint32_t swz_addr(uint32_t base, int row, int cc) {
  return base + (cc >> 3) * DecCfg<D>::kBox + row * 128 + (((cc & 7) ^ (row & 7)) << 4);
}

// grid: units * S CTAs in clusters of S (S = splits per unit, <= 16); 128 threads.
// TR (at most 8 rows per unit): the products are taken transposed, S^T = K Q^T and
// O^T = V^T P^T, so that the keys and channels fill the M = 16 side of each MMA and
// the rows the N = 8 side (no padding rows); P^T goes from the S^T accumulators to
// the B operand of the second product by an in-register 8x8 transpose (movmatrix).
template <int D, bool F16, bool PAGED, bool ROPE, bool TR>
__global__ void __launch_bounds__(DecCfg<D>::kThreads, 1)
    flash_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecArgs a) {
  using C = DecCfg<D>;
  constexpr int kNT = C::kNT;
  constexpr int kMS = C::kChunk / 16;          // TR: S^T m-tiles (16 keys) per chunk
  constexpr int kDN = TR ? D / 16 : D / 8;     // O n-tiles of 8 (TR: O^T m-tiles of 16) channels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int S = static_cast<int>(cluster_nctarank());
  const int split = static_cast<int>(cluster_ctarank());
  const int u = blockIdx.x / S;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff);
  const uint32_t bar0 = smem_u32(smem + C::kBarOff);
  const int nsw = a.nsw;
  uint8_t* ring = smem + C::kRingOff;
  uint8_t* mo_base = ring + C::kWarps * nsw * C::kSlotBytes;
  uint8_t* ms_base = mo_base + a.owner_slots * C::kMoStride * 4;
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + C::kQOff);

  // This CTA's chunks: an even share of the union range; warp w's: every
  // kWarps-th of them from the w-th.
  const int base = a.n_chunks / S, rem = a.n_chunks % S;
  const int c_begin = split * base + min(split, rem);
  const int c_count = base + (split < rem ? 1 : 0);
  auto chunks_of = [&](int w) {
    return c_count > w ? (c_count - w + C::kWarps - 1) / C::kWarps : 0;
  };
  const int n_mine = chunks_of(warp);

  // The i-th chunk of warp w into slot nsw * w + i % nsw (one thread).
  auto issue = [&](int w, int i) {
    if ((a.debug & 1u) && i == 1 && w == 0 && blockIdx.x == 0) return;  // timeout test
    const int key0 = (a.chunk0 + c_begin + w + C::kWarps * i) * C::kChunk;
    const int slot = nsw * w + i % nsw;
    const uint32_t dst = smem_u32(ring + slot * C::kSlotBytes);
    const uint32_t bar = bar0 + 8 * slot;
    mbar_arrive_expect_tx(bar, C::kSlotBytes);
    if constexpr (PAGED) {
      const int b = u / a.n_kv_heads, h = u % a.n_kv_heads;
      const int blk = __ldg(a.block_table + static_cast<size_t>(b) * a.bt_stride + key0 / 128);
#pragma unroll
      for (int hf = 0; hf < C::kHalfBoxes; ++hf) {
        tma_load_4d(&tm_k, dst + hf * C::kBox, bar, hf * 64, key0 % 128, h, blk);
        tma_load_4d(&tm_v, dst + C::kKVBytes + hf * C::kBox, bar, hf * 64, key0 % 128, h, blk);
      }
    } else {
#pragma unroll
      for (int hf = 0; hf < C::kHalfBoxes; ++hf) {
        tma_load_3d(&tm_k, dst + hf * C::kBox, bar, hf * 64, key0, u);
        tma_load_3d(&tm_v, dst + C::kKVBytes + hf * C::kBox, bar, hf * 64, key0, u);
      }
    }
  };

  // The barriers first; then every warp starts its first two chunks before anything
  // else, so that the whole CTA's loads are in flight while Q is staged.
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kWarps * nsw; ++i) mbar_init(bar0 + 8 * i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    for (int i = 0; i < n_mine && i < nsw; ++i) issue(warp, i);
  }
  // Stage the unit's rows (zeros past R), 16 bytes per thread and step.
  const uint16_t* qsrc = a.q + static_cast<size_t>(u) * a.R * D;
  for (int e = threadIdx.x; e < 16 * (D / 8); e += C::kThreads) {
    const int r = e / (D / 8), cc = e % (D / 8);
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r < a.R) val = __ldg(reinterpret_cast<const uint4*>(qsrc + static_cast<size_t>(r) * D) + cc);
    *reinterpret_cast<uint4*>(qs + r * C::kQStride + cc * 8) = val;
  }
  __syncthreads();  // Q staged
  cluster_arrive_relaxed();  // this CTA runs (waited for before the first remote store)
  int issued = min(n_mine, nsw);
  if constexpr (ROPE) {
    // rotate each pair of the staged rows: the same float32 operations and 16-bit
    // rounding as every other rotation of the library
    const int half = a.rope_R / 2;
    for (int e = threadIdx.x; e < a.R * half; e += C::kThreads) {
      const int r = e / half, i = e % half;
      const int pos = a.start_pos + r % a.Sq;
      const int ca = a.rope_inter ? 2 * i : i, cb = a.rope_inter ? 2 * i + 1 : i + half;
      float x0 = from16<F16>(qs[r * C::kQStride + ca]);
      float x1 = from16<F16>(qs[r * C::kQStride + cb]);
      const float* tr = a.rope_table + static_cast<size_t>(pos) * a.rope_R;
      rope_rotate(x0, x1, __ldg(tr + i), __ldg(tr + half + i));
      qs[r * C::kQStride + ca] = to16<F16>(x0);
      qs[r * C::kQStride + cb] = to16<F16>(x1);
    }
    __syncthreads();
  }
  // Q fragments: the A operand (rows g and g + 8, channels 16 ks + 2t (+1, +8, +9)),
  // or with TR the B operand of S^T (row g, the same channels; words 0 and 2).
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint16_t* r0 = qs + g * C::kQStride + 16 * ks + 2 * t;
    const uint16_t* r1 = r0 + 8 * C::kQStride;
    qa[ks][0] = *reinterpret_cast<const uint32_t*>(r0);
    qa[ks][1] = TR ? 0u : *reinterpret_cast<const uint32_t*>(r1);
    qa[ks][2] = *reinterpret_cast<const uint32_t*>(r0 + 8);
    qa[ks][3] = TR ? 0u : *reinterpret_cast<const uint32_t*>(r1 + 8);
  }
  // visible key range of this thread's two rows (g and g + 8; TR: 2t and 2t + 1; a
  // padding row sees nothing)
  int lo[2], hi[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = TR ? 2 * t + h : g + 8 * h;
    const int p = a.start_pos + r % a.Sq;
    lo[h] = max(a.window_lo, 0);
    if (a.window_size > 0) lo[h] = max(lo[h], p - a.window_size + 1);
    hi[h] = a.causal ? min(a.Skv - 1, p) : a.Skv - 1;
    if (r >= a.R) lo[h] = 1, hi[h] = 0;
  }

  float m[2] = {-INFINITY, -INFINITY};
  float la[2] = {0.0f, 0.0f}, lb[2] = {0.0f, 0.0f};  // sums of the 16-bit P values
  float lf[2] = {0.0f, 0.0f};                        // float32 sums (log-sum-exp)
  float o[kDN][4];
#pragma unroll
  for (int dn = 0; dn < kDN; ++dn) o[dn][0] = o[dn][1] = o[dn][2] = o[dn][3] = 0.0f;

  int done = 0;
  bool ok = true;
  for (int i = 0; i < n_mine; ++i) {
    const int slot = nsw * warp + i % nsw;
    ok = __all_sync(0xffffffffu, mbar_wait(bar0 + 8 * slot, (i / nsw) & 1, abort_flag));
    if (!ok) {
      if (lane == 0) {
        *abort_flag = 1;
        atomicOr(a.err, (unsigned)kErrTimeout);
      }
      break;
    }
    const int key0 = (a.chunk0 + c_begin + warp + C::kWarps * i) * C::kChunk;
    const uint32_t kb = smem_u32(ring + slot * C::kSlotBytes);
    const uint32_t vb = kb + C::kKVBytes;
    if constexpr (PAGED) {
      // keys past kv_len in the last block: clear V there (P is 0, but 0 * NaN is not)
      if (key0 + C::kChunk > a.Skv) {
        const int from = max(a.Skv - key0, 0);
        uint4* vrow = reinterpret_cast<uint4*>(ring + slot * C::kSlotBytes + C::kKVBytes);
        for (int e = lane; e < (C::kChunk - from) * (D / 8); e += 32) {
          const int row = from + e / (D / 8), cc = e % (D / 8);
          vrow[((cc >> 3) * C::kBox + row * 128) / 16 + (cc & 7)] = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
    }
    if constexpr (TR) {
      // S^T = K Q^T: kMS m-tiles of 16 keys (even and odd k-steps into separate
      // accumulators)
      float st[kMS][4], st2[kMS][4];
#pragma unroll
      for (int ms = 0; ms < kMS; ++ms)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[ms][e] = st2[ms][e] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int ms = 0; ms < kMS; ++ms) {
          uint32_t ka[4];
          ldsm_x4(swz_addr<D>(kb, 16 * ms + (lane & 7) + ((lane >> 3) & 1) * 8,
                              2 * ks + (lane >> 4)),
                  ka[0], ka[1], ka[2], ka[3]);
          mma16816<F16>((ks & 1) ? st2[ms] : st[ms], ka, qa[ks][0], qa[ks][2]);
        }
      }
      // mask, scale, running maximum per row (row 2t + h: elements e with e % 2 == h;
      // keys 16 ms + g and + 8), reduced over the eight lanes of a column
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int ms = 0; ms < kMS; ++ms) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = e & 1;
          const int j = key0 + 16 * ms + g + (e >> 1) * 8;
          const float x =
              (j < lo[h] || j > hi[h]) ? -INFINITY : (st[ms][e] + st2[ms][e]) * a.scale_log2;
          st[ms][e] = x;
          mx[h] = fmaxf(mx[h], x);
        }
      }
      float bse[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 4));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 8));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
        const float mn = fmaxf(m[h], mx[h]);
        bse[h] = mn == -INFINITY ? 0.0f : mn;
        const float alpha = ex2(m[h] - bse[h]);
        m[h] = mn;
        la[h] *= alpha;
        lb[h] *= alpha;
        lf[h] *= alpha;
#pragma unroll
        for (int mt = 0; mt < kDN; ++mt) {
          o[mt][h] *= alpha;
          o[mt][2 + h] *= alpha;
        }
      }
      // P^T (16-bit) by 8x8 blocks, transposed into the B operand of O^T += V^T P^T
      uint32_t pb[kMS][2];
#pragma unroll
      for (int ms = 0; ms < kMS; ++ms) {
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {  // keys g (hk 0) and g + 8 (hk 1)
          const float p0 = ex2(st[ms][2 * hk] - bse[0]), p1 = ex2(st[ms][2 * hk + 1] - bse[1]);
          lf[0] += p0;
          lf[1] += p1;
          const uint32_t w = pack16x2<F16>(p0, p1);  // (row 2t, row 2t + 1) at one key
          if (hk == 0) add_16x2<F16>(w, la[0], la[1]);
          else add_16x2<F16>(w, lb[0], lb[1]);
          pb[ms][hk] = movmatrix_t(w);
        }
      }
      // O^T += V^T P^T: m-tiles of 16 channels, k-steps of 16 keys
#pragma unroll
      for (int kk = 0; kk < kMS; ++kk) {
#pragma unroll
        for (int mt = 0; mt < kDN; ++mt) {
          uint32_t va[4];
          ldsm_x4_t(swz_addr<D>(vb, 16 * kk + (lane & 7) + ((lane >> 4) & 1) * 8,
                                2 * mt + ((lane >> 3) & 1)),
                    va[0], va[1], va[2], va[3]);
          mma16816<F16>(o[mt], va, pb[kk][0], pb[kk][1]);
        }
      }
    } else {
      // S = Q K^T for the chunk's kNT n-tiles of 8 keys (even and odd k-steps into
      // separate accumulators: two dependency chains of D/32 MMAs per n-tile)
      float s[kNT][4], s2[kNT][4];
  #pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
  #pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = s2[nt][e] = 0.0f;
  #pragma unroll
      for (int ks2 = 0; ks2 < D / 32; ++ks2) {
  #pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(swz_addr<D>(kb, nt * 8 + (lane & 7), 4 * ks2 + (lane >> 3)), b0, b1, b2, b3);
          mma16816<F16>(s[nt], qa[2 * ks2], b0, b1);
          mma16816<F16>(s2[nt], qa[2 * ks2 + 1], b2, b3);
        }
      }
  #pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
  #pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];
      // mask, scale to base 2, running maximum per row
      float mx[2] = {-INFINITY, -INFINITY};
  #pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
  #pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = e >> 1;
          const int j = key0 + nt * 8 + 2 * t + (e & 1);
          const float x = (j < lo[h] || j > hi[h]) ? -INFINITY : s[nt][e] * a.scale_log2;
          s[nt][e] = x;
          mx[h] = fmaxf(mx[h], x);
        }
      }
      float bse[2];
  #pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        const float mn = fmaxf(m[h], mx[h]);
        bse[h] = mn == -INFINITY ? 0.0f : mn;
        const float alpha = ex2(m[h] - bse[h]);  // 0 while the row has seen nothing
        m[h] = mn;
        la[h] *= alpha;
        lb[h] *= alpha;
        lf[h] *= alpha;
  #pragma unroll
        for (int dn = 0; dn < kDN; ++dn) {
          o[dn][2 * h] *= alpha;
          o[dn][2 * h + 1] *= alpha;
        }
      }
      // P = 2^(x - m), rounded to the 16-bit type for P V; A fragments of P V
      uint32_t pa[kNT / 2][4];
  #pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float p0 = ex2(s[nt][2 * h] - bse[h]), p1 = ex2(s[nt][2 * h + 1] - bse[h]);
          lf[h] += p0 + p1;
          const uint32_t w = pack16x2<F16>(p0, p1);
          add_16x2<F16>(w, la[h], lb[h]);
          pa[nt >> 1][(nt & 1) * 2 + h] = w;
        }
      }
      // O += P V: k-steps of 16 keys, two n-tiles of 8 channels per transposed load
  #pragma unroll
      for (int kk = 0; kk < kNT / 2; ++kk) {
  #pragma unroll
        for (int dn2 = 0; dn2 < D / 16; ++dn2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(swz_addr<D>(vb, 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8,
                                2 * dn2 + (lane >> 4)),
                    b0, b1, b2, b3);
          mma16816<F16>(o[2 * dn2], pa[kk], b0, b1);
          mma16816<F16>(o[2 * dn2 + 1], pa[kk], b2, b3);
        }
      }
    }
    ++done;
    __syncwarp();
    if (i + nsw < n_mine) {
      if (lane == 0) {
        fence_proxy_async_smem();  // this warp's reads (and clears) before the next copy
        issue(warp, i + nsw);
      }
      ++issued;
    }
  }
  // Never leave with a copy in flight into this CTA's shared memory.
  if (!ok && lane == 0) {
    for (int i = done; i < issued; ++i) {
      const uint32_t bar = bar0 + 8 * (nsw * warp + i % nsw);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait_sleep(bar, (i / nsw) & 1) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
  float l[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] = la[h] + lb[h];
#pragma unroll
    for (int o2 = TR ? 4 : 1; o2 <= (TR ? 16 : 2); o2 <<= 1) {
      l[h] += __shfl_xor_sync(0xffffffffu, l[h], o2);
      lf[h] += __shfl_xor_sync(0xffffffffu, lf[h], o2);
    }
  }

  // ---- merge: each warp writes its partial (m, l, lf, O) of every row into the
  // shared memory of the CTA that owns the row; one cluster barrier; each owner
  // combines its rows' S * kWarps partials with one denominator and writes them.
  const int rpo = (a.R + S - 1) / S;            // rows per owner
  const int np = S * C::kWarps;                 // partials per row
  const uint32_t mo_u = smem_u32(mo_base), ms_u = smem_u32(ms_base);
  const int part = split * C::kWarps + warp;
  cluster_wait();  // every CTA of the cluster has started
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = TR ? 2 * t + h : g + 8 * h;
    if (r < a.R) {
      const uint32_t owner = static_cast<uint32_t>(r % S);
      const int slot = part * rpo + r / S;
      const uint32_t dst = dsmem_addr(mo_u + slot * C::kMoStride * 4, owner);
      if constexpr (TR) {  // channels 16 mt + g and + 8 of row 2t + h
#pragma unroll
        for (int mt = 0; mt < kDN; ++mt) {
          st_dsmem(dst + (16 * mt + g) * 4, o[mt][h]);
          st_dsmem(dst + (16 * mt + g + 8) * 4, o[mt][2 + h]);
        }
        if (g == 0) st_dsmem_v4(dsmem_addr(ms_u + slot * 16, owner), m[h], l[h], lf[h], 0.0f);
      } else {
#pragma unroll
        for (int dn = 0; dn < kDN; ++dn)
          st_dsmem_v2(dst + (8 * dn + 2 * t) * 4, o[dn][2 * h], o[dn][2 * h + 1]);
        if (t == 0) st_dsmem_v4(dsmem_addr(ms_u + slot * 16, owner), m[h], l[h], lf[h], 0.0f);
      }
    }
  }
  cluster_sync();

  // Owner: per owned row, one warp forms the maximum over the row's partials, their
  // weights 2^(m_p - M) (into shared memory) and the two denominators; then every
  // thread sums its channel over the partials.
  const float* mo = reinterpret_cast<const float*>(mo_base);
  const float4* ms = reinterpret_cast<const float4*>(ms_base);
  float* wt = reinterpret_cast<float*>(smem + C::kWtOff);      // [rpo][64] weights
  float* rs = reinterpret_cast<float*>(smem + C::kWtOff + 16 * 64 * 4);  // [rpo][4]: M, L, LF
  const int nown = split < a.R ? (a.R - split + S - 1) / S : 0;  // rows this CTA owns
  for (int i = warp; i < nown; i += C::kWarps) {
    const float4 s0 = lane < np ? ms[lane * rpo + i] : make_float4(-INFINITY, 0.0f, 0.0f, 0.0f);
    const float4 s1 =
        lane + 32 < np ? ms[(lane + 32) * rpo + i] : make_float4(-INFINITY, 0.0f, 0.0f, 0.0f);
    float M = fmaxf(s0.x, s1.x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w0 = s0.x == -INFINITY ? 0.0f : ex2(s0.x - M);
    const float w1 = s1.x == -INFINITY ? 0.0f : ex2(s1.x - M);
    wt[i * 64 + lane] = w0;
    wt[i * 64 + lane + 32] = w1;
    float L = w0 * s0.y + w1 * s1.y, LF = w0 * s0.z + w1 * s1.z;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      L += __shfl_xor_sync(0xffffffffu, L, o);
      LF += __shfl_xor_sync(0xffffffffu, LF, o);
    }
    if (lane == 0) {
      rs[i * 4] = M;
      rs[i * 4 + 1] = L;
      rs[i * 4 + 2] = LF;
    }
  }
  __syncthreads();
  constexpr int kRowsPerPass = C::kThreads / D;  // 1 (head_dim 128) or 2 (64)
  const int d = threadIdx.x % D;
  for (int i = threadIdx.x / D; i < nown; i += kRowsPerPass) {
    const int r = split + S * i;
    float acc0 = 0.0f, acc1 = 0.0f;
    int p = 0;
    for (; p + 1 < np; p += 2) {
      acc0 += wt[i * 64 + p] * mo[(p * rpo + i) * C::kMoStride + d];
      acc1 += wt[i * 64 + p + 1] * mo[((p + 1) * rpo + i) * C::kMoStride + d];
    }
    if (p < np) acc0 += wt[i * 64 + p] * mo[(p * rpo + i) * C::kMoStride + d];
    const float L = rs[i * 4 + 1], LF = rs[i * 4 + 2];
    const size_t row = static_cast<size_t>(u) * a.R + r;
    a.o[row * D + d] = to16<F16>(L > 0.0f ? (acc0 + acc1) / L : 0.0f);
    if (d == 0 && a.lse != nullptr)
      a.lse[row] = LF > 0.0f ? (rs[i * 4] + lg2(LF)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace attn
