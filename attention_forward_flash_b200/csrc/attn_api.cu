// Host side of the C ABI declared in include/attn.h: argument validation, the
// choice of kernel variant and key/value split, workspace ownership, TMA
// tensor-map encoding and the launches.  No computation happens here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "decode.cuh"
#include "device_once.h"
#include "flash_fwd.cuh"
#include "merge.cuh"
#include "quant.cuh"

using namespace attn;

namespace {
constexpr int kMaxHostChunks = 64;  // ranges of units of one attn_forward_host call

// Tensor maps of one launch, kept with the base pointers and unit count they were
// encoded for: a later launch on the same buffers reuses them.
// The tensor maps of one attention launch: Q, K, V (or their INT8 / E4M3 codes),
// O, and in the diagonal band mode the 16-bit Q and K (else unused copies).
struct FwdMaps {
  CUtensorMap q, k, v, o, q16, k16;
};

struct MapCache {
  bool valid;
  const void* key[6];  // the base pointers the maps were encoded for
  int nu;
  FwdMaps m;
};
}  // namespace

struct attn_ctx {
  attn_params p;
  int device;
  int num_sms;
  int G;           // query heads per kv head
  int R;           // stacked rows per unit
  int units;       // batch * n_kv_heads
  int split_path;  // 1: single-query-tile kernel + merge; 0: two-query-tile kernel
  int decode;      // 1: flash_decode_kernel (one cluster of `splits` CTAs per unit)
  int dec_chunk0;  // decode kernel: first key chunk of the rows' visible union
  int dec_nchunks; //   and its number of chunks
  int dec_nsw;     //   ring slots per warp
  int dec_owner_slots;  // partial-row slots of its merge area
  int dec_smem;    //   dynamic shared memory per CTA
  // Single-pass kernel whose grid ends in a short last wave: its last tail_items
  // CTAs run as the split kernel with tail_k key splits (partials in the workspace).
  int tail_items;
  int tail_k;
  float* tail_opart;
  float* tail_lse;
  int splits;
  int tiles_per_split;
  int row_tiles;
  float scale;
  void* ws;         // workspace (one allocation)
  size_t ws_bytes;
  float* o_part;
  float* lse_part;
  unsigned* v_amax;
  unsigned* err;
  unsigned debug;
  // RoPE: the caller's cos/sin table (attn_set_rope_table) and, in the exact mode
  // on unrotated keys, a buffer of K's size that receives the rotated keys.
  const float* rope_table;
  int rope_npos;
  void* ws_k;
  // Recorded on the caller's stream after the work of every call: attn_destroy
  // waits for it (the context's last call) instead of the whole device.
  cudaEvent_t done_ev;
  // attn_forward_host's pipeline, created by its first call: stream 0 carries the
  // host-to-device copies, 1 and 2 the kernels of even and odd ranges, 3 the
  // device-to-host copies.
  bool pipe_ready;
  cudaStream_t pipe[4];
  cudaEvent_t pev_start, pev_join[4];
  cudaEvent_t pev_in[kMaxHostChunks], pev_done[kMaxHostChunks];
  // Encoded tensor maps: slot 0 for attn_forward, slot 1 + i for range i of
  // attn_forward_host.
  MapCache maps[1 + kMaxHostChunks];
};

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D tiled map: dims (d0 fastest, d1, d2), byte strides of d1 and d2, box (b0, b1, 1).
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
              uint64_t d2, uint64_t st1, uint64_t st2, uint32_t b0, uint32_t b1,
              CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {st1, st2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D tiled map of a paged key/value pool [blocks][kv heads][128 positions][D]:
// dims (D, 128, kv heads, blocks), box (64 channels, `rows` positions, 1, 1).
bool make_pool_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t D,
                   uint64_t hkv, uint64_t blocks, uint32_t rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {D, 128, hkv, blocks};
  cuuint64_t strides[3] = {D * 2, 128 * D * 2, hkv * 128 * D * 2};
  cuuint32_t box[4] = {64, rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Raises the dynamic shared-memory limit of kernel `Kern` to `bytes` on the
// current device, once per device: the attribute is per device, so each kernel
// (one template instance of this function, hence one flag set, per kernel) keeps
// a flag per device ordinal.
template <auto Kern>
bool set_smem(int bytes) {
  static PerDeviceOnce<> once;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  return once.ensure(dev, [&] {
    return cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
           cudaSuccess;
  });
}

// The decode kernel's attributes, once per device: its dynamic shared memory, and
// clusters of up to 16 CTAs (above the portable 8).
template <auto Kern>
bool set_decode_attrs(int bytes) {
  static PerDeviceOnce<> once;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  return once.ensure(dev, [&] {
    return cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
               cudaSuccess &&
           cudaFuncSetAttribute(Kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
               cudaSuccess;
  });
}

// Launch configuration of the decode kernel: `units` clusters of `splits` CTAs.
template <int D>
cudaLaunchConfig_t decode_config(int units, int splits, int smem, cudaStream_t st,
                                 cudaLaunchAttribute* at) {
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(splits);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(units * splits));
  cfg.blockDim = dim3(DecCfg<D>::kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cfg;
}

// Clusters of `splits` decode CTAs that the current device holds at once (0 if none
// or on error).
template <int D>
int decode_max_clusters(int units, int splits) {
  constexpr auto kern = flash_decode_kernel<D, false, false, false, false>;
  if (!set_decode_attrs<kern>(DecCfg<D>::kMaxSmem)) return 0;
  cudaLaunchAttribute at[1];
  // every launch takes more than half an SM's shared memory: one CTA per SM
  const cudaLaunchConfig_t cfg = decode_config<D>(units, splits, DecCfg<D>::kMaxSmem, nullptr, at);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int D, bool F16, bool PAGED, bool ROPE, bool TR>
attn_status launch_decode(const attn_ctx* c, const CUtensorMap& mk, const CUtensorMap& mv,
                          const DecArgs& a, int nu, cudaStream_t st) {
  constexpr auto kern = flash_decode_kernel<D, F16, PAGED, ROPE, TR>;
  if (!set_decode_attrs<kern>(DecCfg<D>::kMaxSmem)) return ATTN_ERR_CUDA;
  cudaLaunchAttribute at[1];
  const cudaLaunchConfig_t cfg = decode_config<D>(nu, c->splits, c->dec_smem, st, at);
  return cudaLaunchKernelEx(&cfg, kern, mk, mv, a) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool PAGED, bool TR>
attn_status dispatch_decode_t(const attn_ctx* c, const CUtensorMap& mk, const CUtensorMap& mv,
                              const DecArgs& a, int nu, cudaStream_t st) {
  const bool rope = a.rope_table != nullptr;
  if (c->p.dtype == ATTN_FP16)
    return rope ? launch_decode<D, true, PAGED, true, TR>(c, mk, mv, a, nu, st)
                : launch_decode<D, true, PAGED, false, TR>(c, mk, mv, a, nu, st);
  return rope ? launch_decode<D, false, PAGED, true, TR>(c, mk, mv, a, nu, st)
              : launch_decode<D, false, PAGED, false, TR>(c, mk, mv, a, nu, st);
}

// At most 8 rows per unit: the transposed products (no padding rows in the MMAs).
template <int D, bool PAGED>
attn_status dispatch_decode(const attn_ctx* c, const CUtensorMap& mk, const CUtensorMap& mv,
                            const DecArgs& a, int nu, cudaStream_t st) {
  return c->R <= 8 ? dispatch_decode_t<D, PAGED, true>(c, mk, mv, a, nu, st)
                   : dispatch_decode_t<D, PAGED, false>(c, mk, mv, a, nu, st);
}

// Decode-kernel arguments for the units whose Q, O and lse start at q, o, lse.
DecArgs decode_args(const attn_ctx* c, const void* q, void* o, float* lse) {
  const attn_params& p = c->p;
  DecArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.o = static_cast<uint16_t*>(o);
  a.lse = lse;
  a.R = c->R;
  a.Sq = p.q_len;
  a.Skv = p.kv_len;
  a.start_pos = p.start_pos;
  a.causal = p.causal;
  a.window_lo = p.window_lo;
  a.window_size = p.window_size;
  a.chunk0 = c->dec_chunk0;
  a.n_chunks = c->dec_nchunks;
  a.scale_log2 = c->scale * 1.4426950408889634f;
  if (p.rope_dim > 0) {
    a.rope_table = c->rope_table;
    a.rope_R = p.rope_dim;
    a.rope_inter = p.rope_interleaved;
  }
  a.err = c->err;
  a.debug = c->debug;
  a.nsw = c->dec_nsw;
  a.owner_slots = c->dec_owner_slots;
  return a;
}

inline uint32_t decode_chunk(int head_dim) {
  return head_dim == 128 ? DecCfg<128>::kChunk : DecCfg<64>::kChunk;
}

// The kernel choice for a problem on a GPU with `sms` SMs (attn_create, attn_plan_for).
// `max_clusters(S)`: how many decode clusters of S CTAs the device holds at once.
struct Plan {
  int path = ATTN_PATH_SINGLE_PASS;
  int splits = 1;           // key splits (decode: CTAs per cluster)
  int tiles_per_split = 1;  // split kernel: 128-key tiles per split
  int row_tiles = 1;        // row tiles per unit (256 rows; 128 on the split kernel)
  int tail_items = 0;       // single pass: last-wave CTAs moved to the split kernel
  int tail_splits = 0;
  int dec_chunk0 = 0;       // decode: first chunk of the rows' visible union
  int dec_nchunks = 0;
};

template <typename MaxClusters>
void plan_problem(const attn_params& p, int sms, Plan& pl, MaxClusters&& max_clusters) {
  const int G = p.n_q_heads / p.n_kv_heads;
  const int R = G * p.q_len;
  const int units = p.batch * p.n_kv_heads;
  const int kv_tiles = ceil_div(p.kv_len, 128);
  const int big_ctas = units * ceil_div(R, 256);
  bool split = false, decode = false;
  int splits = 1;
  if (p.precision == ATTN_MIXED_DIAG || p.precision == ATTN_MXFP4QK_FP8PV) {
    // single-pass kernel only (the band and FP4 modes have no split-KV variant)
  } else if (p.precision == ATTN_EXACT && R <= 16 && p.kv_len > 0 &&
             (p.num_splits == 0 ||
              (p.num_splits > 1 && p.num_splits <= DecCfg<128>::kMaxSplits))) {
    // Decode-shaped (at most 16 stacked rows per unit): the cluster kernel.  The
    // union of the rows' visible key ranges: row 0 has the lowest lower bound,
    // the last position the highest upper bound.
    decode = true;
    const int chunk = static_cast<int>(decode_chunk(p.head_dim));
    long long lo = std::max(p.window_lo, 0);
    if (p.window_size > 0)
      lo = std::max<long long>(lo, static_cast<long long>(p.start_pos) - p.window_size + 1);
    long long hi = p.kv_len - 1;
    if (p.causal) hi = std::min<long long>(hi, static_cast<long long>(p.start_pos) + p.q_len - 1);
    pl.dec_chunk0 = lo <= hi ? static_cast<int>(lo / chunk) : 0;
    pl.dec_nchunks = lo <= hi ? static_cast<int>(hi / chunk - lo / chunk + 1) : 0;
    // about one CTA per SM over all units (at most 16 per cluster, at most one chunk
    // each), then as large a cluster as lets every unit's cluster (or as many as
    // the SMs hold) be resident at once
    int S = p.num_splits > 1 ? p.num_splits
                             : std::max(1, std::min(DecCfg<128>::kMaxSplits, sms / units));
    S = std::max(1, std::min(S, std::max(pl.dec_nchunks, 1)));
    while (S > 1 && max_clusters(S) < std::min(units, std::max(1, sms / S))) --S;
    splits = S;
  } else if (p.num_splits > 1) {
    split = true;
    splits = p.num_splits;
  } else if (p.num_splits == 0) {
    // Few rows per kv head or too few CTAs to fill the GPU: one 128-row query tile
    // per CTA, keys split across CTAs, then a merge.
    if (R <= 128 || (big_ctas * 2 < sms && kv_tiles >= 4)) {
      split = true;
      const int base = units * ceil_div(R, 128);
      splits = std::max(1, std::min(kv_tiles, ceil_div(2 * sms, base)));  // two CTAs per SM
    }
  }
  if (!decode) {
    splits = std::min(std::max(splits, 1), std::max(kv_tiles, 1));
    splits = std::min(splits, kMergeMaxSplits);
  }
  pl.tiles_per_split = std::max(1, ceil_div(kv_tiles, splits));
  pl.splits = split ? std::max(1, ceil_div(kv_tiles, pl.tiles_per_split)) : (decode ? splits : 1);
  pl.row_tiles = ceil_div(R, split ? 128 : 256);
  pl.path = decode ? ATTN_PATH_DECODE : (split ? ATTN_PATH_SPLIT_MERGE : ATTN_PATH_SINGLE_PASS);
  // Tail of the single-pass grid (non-causal, whole 256-row tiles, library's split
  // choice; the band and FP4 modes have no split variant): when the CTAs leave a
  // last wave at most half full, its CTAs' keys are split instead.
  if (!split && !decode && !p.causal && p.num_splits == 0 && R % 256 == 0 &&
      (p.precision == ATTN_EXACT || p.precision == ATTN_INT8QK_FP8PV)) {
    const int nctas = units * (R / 256);
    const int T = nctas % sms;
    if (nctas > sms && T > 0 && 2 * T <= sms && kv_tiles >= 2) {
      // the split kernel holds two CTAs per SM: 2 T tiles x k splits <= 2 x #SM
      pl.tail_items = T;
      pl.tail_splits = std::max(2, std::min(std::min(sms / T, kv_tiles), kMergeMaxSplits));
      pl.path = ATTN_PATH_SINGLE_PASS_TAIL;
    }
  }
}

template <int D, int NQT, bool QUANT, bool F16, bool SPLIT, bool LF, bool WIN, bool ROPE,
          bool DIAG = false, bool FP4 = false>
attn_status launch_fwd(const attn_ctx* /*context*/, const FwdMaps& m, const FwdArgs& a, int grid,
                       cudaStream_t st) {
  using Cfg = FwdCfg<D, NQT, QUANT, SPLIT, DIAG, FP4>;
  constexpr auto kern = flash_fwd_kernel<D, NQT, QUANT, F16, SPLIT, LF, WIN, ROPE, DIAG, FP4>;
  if (!set_smem<kern>(Cfg::kSmemBytes)) return ATTN_ERR_CUDA;
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(m.q, m.k, m.v, m.o, m.q16, m.k16, a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool QUANT, bool F16, bool WIN, bool ROPE>
attn_status dispatch_win(const attn_ctx* c, const FwdMaps& m, const FwdArgs& a, int grid,
                         cudaStream_t st, bool split) {
  // the diagonal band mode: single-pass quantised kernel with 16-bit band tiles
  if constexpr (QUANT) {
    if (c->p.precision == ATTN_MIXED_DIAG)
      return launch_fwd<D, 2, true, F16, false, false, WIN, false, true>(c, m, a, grid, st);
  }
  // the FP4 mode (head_dim 64): single-pass kernel with block-scaled MXFP4 Q K^T
  if constexpr (QUANT && D == 64) {
    if (c->p.precision == ATTN_MXFP4QK_FP8PV)
      return launch_fwd<D, 2, true, F16, false, false, WIN, false, false, true>(c, m, a, grid,
                                                                                st);
  }
  if (split) return launch_fwd<D, 1, QUANT, F16, true, true, WIN, ROPE>(c, m, a, grid, st);
  // Exact mode keeps a second (float32) row sum only when the caller asks for lse
  // (the quantised mode's only sum is the float32 one).
  if constexpr (!QUANT) {
    if (a.lse != nullptr)
      return launch_fwd<D, 2, QUANT, F16, false, true, WIN, ROPE>(c, m, a, grid, st);
  }
  return launch_fwd<D, 2, QUANT, F16, false, false, WIN, ROPE>(c, m, a, grid, st);
}

template <int D, bool QUANT, bool F16, bool ROPE>
attn_status dispatch_rope(const attn_ctx* c, const FwdMaps& m, const FwdArgs& a, int grid,
                          cudaStream_t st, bool split) {
  if (a.window_size > 0)
    return dispatch_win<D, QUANT, F16, true, ROPE>(c, m, a, grid, st, split);
  return dispatch_win<D, QUANT, F16, false, ROPE>(c, m, a, grid, st, split);
}

// Exact mode with RoPE: the variant that rotates the staged Q tile (the keys
// arrive rotated); the quantised mode rotates in its quantiser.
template <int D, bool QUANT, bool F16>
attn_status dispatch_fwd(const attn_ctx* c, const FwdMaps& m, const FwdArgs& a, int grid,
                         cudaStream_t st, bool split) {
  if constexpr (!QUANT) {
    if (a.rope_table != nullptr)
      return dispatch_rope<D, QUANT, F16, true>(c, m, a, grid, st, split);
  }
  return dispatch_rope<D, QUANT, F16, false>(c, m, a, grid, st, split);
}

// The merge is a programmatic dependent launch of the split kernel: its launch
// overlaps the split kernel's tail, and it waits on the grid dependency before
// reading the partials.
template <int D, bool F16>
attn_status launch_merge_rows(const float* op, const float* lp, uint16_t* out, float* lse,
                              int rows, int stride, int splits, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows);
  cfg.blockDim = dim3(32 * kMergeWarps);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Few splits: one warp per row.  (The choice depends on the split count alone, so
  // that a range of rows merges exactly as the whole problem does.)
  if (splits <= 16) {
    cfg.gridDim = dim3((rows + 3) / 4);
    if (cudaLaunchKernelEx(&cfg, splitkv_merge_rows_kernel<D, F16>, op, lp, out, lse, rows,
                           stride, splits) != cudaSuccess)
      return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  if (cudaLaunchKernelEx(&cfg, splitkv_merge_kernel<D, F16>, op, lp, out, lse, stride, splits) !=
      cudaSuccess)
    return ATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool F16>
attn_status launch_merge(const attn_ctx* c, void* o, float* lse, cudaStream_t st) {
  const int rows = c->units * c->R;
  return launch_merge_rows<D, F16>(c->o_part, c->lse_part, static_cast<uint16_t*>(o), lse, rows,
                                   rows, c->splits, st);
}

attn_status validate(const attn_params* p) {
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->batch < 1 || p->n_q_heads < 1 || p->n_kv_heads < 1) return ATTN_ERR_INVALID_ARG;
  if (p->n_q_heads % p->n_kv_heads != 0) return ATTN_ERR_INVALID_ARG;
  if (p->q_len < 0 || p->kv_len < 0 || p->start_pos < 0 || p->window_lo < 0 ||
      p->window_size < 0)
    return ATTN_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return ATTN_ERR_INVALID_ARG;
  if (p->dtype != ATTN_BF16 && p->dtype != ATTN_FP16) return ATTN_ERR_INVALID_ARG;
  if (p->precision != ATTN_EXACT && p->precision != ATTN_INT8QK_FP8PV &&
      p->precision != ATTN_MIXED_DIAG && p->precision != ATTN_MXFP4QK_FP8PV)
    return ATTN_ERR_INVALID_ARG;
  const bool single_pass_mode =
      p->precision == ATTN_MIXED_DIAG || p->precision == ATTN_MXFP4QK_FP8PV;
  if (single_pass_mode && p->num_splits > 1) return ATTN_ERR_INVALID_ARG;
  // FP4: the scale factors fit tensor memory beside head_dim-64 scores and outputs only
  if (p->precision == ATTN_MXFP4QK_FP8PV && (p->head_dim != 64 || p->rope_dim > 0))
    return ATTN_ERR_UNSUPPORTED;
  // the band tiles read the caller's 16-bit Q and K, which the quantiser's RoPE never sees
  if (p->precision == ATTN_MIXED_DIAG && p->rope_dim > 0) return ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(p->scale)) return ATTN_ERR_INVALID_ARG;
  if (p->num_splits < 0 || p->num_splits > kMergeMaxSplits) return ATTN_ERR_INVALID_ARG;
  if (p->rope_dim < 0 || p->rope_dim % 16 != 0 || p->rope_dim > p->head_dim ||
      (p->rope_interleaved != 0 && p->rope_interleaved != 1) ||
      (p->rope_keys_rotated != 0 && p->rope_keys_rotated != 1))
    return ATTN_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return ATTN_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(p->n_q_heads / p->n_kv_heads) * p->q_len;
  if (rows > (1ll << 30)) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->start_pos) + p->q_len > (1ll << 30)) return ATTN_ERR_UNSUPPORTED;
  // Grid and block counts are 32-bit: the (batch, kv head) units times their row tiles
  // and splits, and the quantisers' 128-token blocks of all heads.
  const long long units = static_cast<long long>(p->batch) * p->n_kv_heads;
  const long long row_tiles = std::max(1ll, (rows + 127) / 128);
  if (units * row_tiles * std::max(1, p->num_splits) > INT_MAX) return ATTN_ERR_UNSUPPORTED;
  const long long nbq = (p->q_len + 127ll) / 128, nbk = (p->kv_len + 127ll) / 128;
  if (static_cast<long long>(p->batch) * p->n_q_heads * nbq > INT_MAX ||
      units * nbk > INT_MAX)
    return ATTN_ERR_UNSUPPORTED;
  // the quantisers run the units along gridDim.y (at most 65535)
  if (p->precision != ATTN_EXACT && units > 65535) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

// Pointer checks of attn_forward.  Buffers of zero length may be NULL (an empty
// tensor has no storage); every other one must be non-NULL and 16-byte aligned.
bool bad_ptr(const void* ptr, bool needed) {
  return needed ? (ptr == nullptr || !aligned16(ptr)) : (ptr != nullptr && !aligned16(ptr));
}

bool bad_qbufs(const attn_params& p, const attn_qbufs* qb) {
  const bool need_q = p.q_len > 0, need_kv = p.kv_len > 0;
  if (!qb) return true;
  if (p.precision == ATTN_MXFP4QK_FP8PV)  // packed codes and scale chunks; no FP32 scales
    return bad_ptr(qb->q, need_q) || bad_ptr(qb->q_sf, need_q) || bad_ptr(qb->k, need_kv) ||
           bad_ptr(qb->k_sf, need_kv) || bad_ptr(qb->v_t, need_kv) ||
           bad_ptr(qb->v_scale, need_kv);
  return bad_ptr(qb->q, need_q) || bad_ptr(qb->q_scale, need_q) ||
         bad_ptr(qb->k, need_kv) || bad_ptr(qb->k_scale, need_kv) || bad_ptr(qb->v_t, need_kv) ||
         bad_ptr(qb->v_scale, need_kv);
}

// FP4 mode: 128-row scale chunks per unit of Q (an even count: the two-tile CTAs
// always read two) and of K.
int fp4_q_tiles(const attn_params& p) {
  const long long R = static_cast<long long>(p.n_q_heads / p.n_kv_heads) * p.q_len;
  return 2 * static_cast<int>((R + 255) / 256);
}

attn_status check_forward_buffers(const attn_ctx* c, const void* q, const void* k, const void* v,
                                  const attn_qbufs* qb, const void* o, const float* lse) {
  const attn_params& p = c->p;
  const bool need_q = p.q_len > 0, need_kv = p.kv_len > 0;
  if (bad_ptr(o, need_q) || (lse && !aligned16(lse))) return ATTN_ERR_INVALID_ARG;
  if (p.precision == ATTN_MIXED_DIAG) {  // codes and the 16-bit Q and K
    if (bad_qbufs(p, qb) || bad_ptr(q, need_q) || bad_ptr(k, need_kv)) return ATTN_ERR_INVALID_ARG;
  } else if (p.precision != ATTN_EXACT) {  // the quantised and FP4 modes read the codes only
    if (bad_qbufs(p, qb)) return ATTN_ERR_INVALID_ARG;
  } else {
    if (qb) return ATTN_ERR_INVALID_ARG;
    if (bad_ptr(q, need_q) || bad_ptr(k, need_kv) || bad_ptr(v, need_kv))
      return ATTN_ERR_INVALID_ARG;
  }
  return ATTN_OK;
}

// y = RoPE(x) over `rows` rows of head_dim channels (row t of a head at position
// pos0 + t % len), with the context's table and pair layout.
attn_status launch_rope_apply(const attn_ctx* c, const void* x, void* y, long long rows, int len,
                              int pos0, cudaStream_t st) {
  const attn_params& p = c->p;
  if (rows <= 0) return ATTN_OK;
  const long long threads = rows * (p.head_dim / 8);
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  if (p.dtype == ATTN_FP16)
    rope_apply_kernel<true><<<blocks, 256, 0, st>>>(
        static_cast<const uint16_t*>(x), static_cast<uint16_t*>(y), c->rope_table, rows, len,
        p.head_dim, p.rope_dim, p.rope_interleaved, pos0);
  else
    rope_apply_kernel<false><<<blocks, 256, 0, st>>>(
        static_cast<const uint16_t*>(x), static_cast<uint16_t*>(y), c->rope_table, rows, len,
        p.head_dim, p.rope_dim, p.rope_interleaved, pos0);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Row tiles per head for the causal heaviest-band-first order of the single-pass
// kernel (FwdArgs::tph), or 0 where it does not apply.
int causal_band_tiles(const attn_ctx* c) {
  const attn_params& p = c->p;
  if (!p.causal || c->split_path || p.q_len % 256 != 0) return 0;
  return p.q_len / 256;
}

// One Q/K quantiser launch over `tot` 128-token blocks (persistent grid).
template <int D, bool F16, bool ROPE>
attn_status quant_qk_launch(const attn_ctx* c, const uint16_t* x, int8_t* codes, float* scales,
                            int S, int nblk, int tot, unsigned debug, const QuantRope& r,
                            cudaStream_t st, const KvBlocks& src = KvBlocks{}) {
  using Cfg = QuantQkCfg<D, ROPE>;
  if (!set_smem<quant_qk_kernel<D, F16, ROPE>>(Cfg::kSmemBytes)) return ATTN_ERR_CUDA;
  const int ctas = std::min(tot, Cfg::kCtasPerSm * c->num_sms);
  quant_qk_kernel<D, F16, ROPE><<<ctas, 256, Cfg::kSmemBytes, st>>>(x, codes, scales, S, nblk,
                                                                     tot, c->err, debug, r, src);
  return ATTN_OK;
}

// V's channel maxima, then its transposed E4M3 codes (both quantised modes).
template <int D, bool F16>
attn_status v_launch(attn_ctx* c, const uint16_t* vx, unsigned* vamax, uint8_t* vt, float* vs,
                     int nbk, unsigned BHk, cudaStream_t st, const KvBlocks& src = KvBlocks{}) {
  const attn_params& p = c->p;
  const int tot = nbk * static_cast<int>(BHk);
  v_amax_kernel<D, F16><<<dim3(ceil_div(p.kv_len, kVTok), BHk), 256, 0, st>>>(vx, vamax,
                                                                             p.kv_len, src);
  if (!set_smem<v_quant_kernel<D, F16>>(VQuantCfg<D>::kSmemBytes)) return ATTN_ERR_CUDA;
  const int vq_ctas = std::min(tot, VQuantCfg<D>::kCtasPerSm * c->num_sms);
  v_quant_kernel<D, F16><<<vq_ctas, 256, VQuantCfg<D>::kSmemBytes, st>>>(
      vx, vamax, vt, vs, p.kv_len, nbk * 128, nbk, tot, c->err, src);
  return ATTN_OK;
}

// The quantisers of one range of units: Q and K blocks (rotated first with RoPE),
// then V's channel maxima and codes.
template <int D, bool F16>
attn_status quant_launch(attn_ctx* c, const uint16_t* qx, int8_t* qc, float* qs,
                         const uint16_t* kx, int8_t* kc, float* ks, const uint16_t* vx,
                         unsigned* vamax, uint8_t* vt, float* vs, int nbq, int nbk, unsigned BHq,
                         unsigned BHk, bool rope_q, bool rope_k, const QuantRope& rq,
                         const QuantRope& rk, cudaStream_t st, const KvBlocks& kvsrc) {
  const attn_params& p = c->p;
  attn_status s = ATTN_OK;
  if (nbq > 0) {
    const int tot = nbq * static_cast<int>(BHq);
    s = rope_q ? quant_qk_launch<D, F16, true>(c, qx, qc, qs, p.q_len, nbq, tot, c->debug, rq, st)
               : quant_qk_launch<D, F16, false>(c, qx, qc, qs, p.q_len, nbq, tot, c->debug, rq,
                                                st);
    if (s != ATTN_OK) return s;
  }
  if (nbk > 0) {
    const int tot = nbk * static_cast<int>(BHk);
    s = rope_k ? quant_qk_launch<D, F16, true>(c, kx, kc, ks, p.kv_len, nbk, tot, 0u, rk, st,
                                               kvsrc)
               : quant_qk_launch<D, F16, false>(c, kx, kc, ks, p.kv_len, nbk, tot, 0u, rk, st,
                                                kvsrc);
    if (s != ATTN_OK) return s;
    return v_launch<D, F16>(c, vx, vamax, vt, vs, nbk, BHk, st, kvsrc);
  }
  return ATTN_OK;
}

// Launches the quantisers on `st` for the units [u0, u0 + nu) (unit = one
// (batch, kv head) pair with its query heads).  Pointers are those of the whole
// problem, already validated.
// With a paged key/value source (kvsrc.table set), k and v are the pools and the
// range is the whole problem.
attn_status quantize_units(attn_ctx* c, int u0, int nu, const void* q, const void* k,
                           const void* v, const attn_qbufs* qb, cudaStream_t st,
                           const KvBlocks& kvsrc = KvBlocks{}) {
  const attn_params& p = c->p;
  const int D = p.head_dim;
  const bool f16 = p.dtype == ATTN_FP16;
  const int nbq = ceil_div(p.q_len, 128), nbk = ceil_div(p.kv_len, 128);
  const int S_pad = nbk * 128;
  const unsigned BHq = static_cast<unsigned>(nu) * c->G;  // query heads of the range
  const unsigned BHk = static_cast<unsigned>(nu);
  // Every tensor is unit-major, so the range [u0, u0 + nu) is a contiguous slice of each.
  const size_t qe = static_cast<size_t>(u0) * c->R * D;         // Q elements / codes before u0
  const size_t ke = static_cast<size_t>(u0) * p.kv_len * D;     // K, V elements before u0
  const uint16_t* qx = static_cast<const uint16_t*>(q) + (nbq > 0 ? qe : 0);
  const size_t kvoff = (nbk > 0 && kvsrc.table == nullptr) ? ke : 0;
  const uint16_t* kx = static_cast<const uint16_t*>(k) + kvoff;
  const uint16_t* vx = static_cast<const uint16_t*>(v) + kvoff;
  int8_t* qc = nbq > 0 ? qb->q + qe : nullptr;
  float* qs = (nbq > 0 && qb->q_scale) ? qb->q_scale + static_cast<size_t>(u0) * c->G * nbq
                                       : nullptr;
  int8_t* kc = nbk > 0 ? qb->k + ke : nullptr;
  float* ks = (nbk > 0 && qb->k_scale) ? qb->k_scale + static_cast<size_t>(u0) * nbk : nullptr;
  uint8_t* vt = nbk > 0 ? qb->v_t + static_cast<size_t>(u0) * D * S_pad : nullptr;
  float* vs = nbk > 0 ? qb->v_scale + static_cast<size_t>(u0) * D : nullptr;
  unsigned* vamax = nbk > 0 ? c->v_amax + static_cast<size_t>(u0) * D : nullptr;

  if (nbk > 0 &&
      cudaMemsetAsync(vamax, 0, static_cast<size_t>(nu) * D * 4, st) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (p.precision == ATTN_MXFP4QK_FP8PV) {
    // Q and K to MXFP4 (packed E2M1 codes and E8M0 scale chunks; head_dim 64), V as in
    // the quantised mode.  Q's rows are each unit's stacked query rows.
    const int qt = fp4_q_tiles(p);
    uint8_t* qcodes = reinterpret_cast<uint8_t*>(qb->q) + static_cast<size_t>(u0) * c->R * (D / 2);
    uint8_t* kcodes =
        reinterpret_cast<uint8_t*>(qb->k) + static_cast<size_t>(u0) * p.kv_len * (D / 2);
    uint8_t* qsf = qb->q_sf + static_cast<size_t>(u0) * qt * 512;
    uint8_t* ksf = qb->k_sf + static_cast<size_t>(u0) * nbk * 512;
    if (nbq > 0) {
      if (f16) mxfp4_qk_kernel<true><<<dim3(qt, nu), 256, 0, st>>>(qx, qcodes, qsf, c->R, qt);
      else mxfp4_qk_kernel<false><<<dim3(qt, nu), 256, 0, st>>>(qx, qcodes, qsf, c->R, qt);
    }
    if (nbk > 0) {
      if (f16) mxfp4_qk_kernel<true><<<dim3(nbk, nu), 256, 0, st>>>(kx, kcodes, ksf, p.kv_len, nbk);
      else mxfp4_qk_kernel<false><<<dim3(nbk, nu), 256, 0, st>>>(kx, kcodes, ksf, p.kv_len, nbk);
      const attn_status vs_st = f16 ? v_launch<64, true>(c, vx, vamax, vt, vs, nbk, BHk, st)
                                    : v_launch<64, false>(c, vx, vamax, vt, vs, nbk, BHk, st);
      if (vs_st != ATTN_OK) return vs_st;
    }
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  // RoPE: Q rows at start_pos + token, K rows at token (unless already rotated)
  const bool rope = p.rope_dim > 0;
  const QuantRope rq{c->rope_table, p.rope_dim, p.rope_interleaved, p.start_pos};
  const QuantRope rk{c->rope_table, p.rope_dim, p.rope_interleaved, 0};
  const bool rope_k = rope && !p.rope_keys_rotated;
  attn_status s = ATTN_OK;
  if (D == 128) {
    s = f16 ? quant_launch<128, true>(c, qx, qc, qs, kx, kc, ks, vx, vamax, vt, vs, nbq, nbk,
                                      BHq, BHk, rope, rope_k, rq, rk, st, kvsrc)
            : quant_launch<128, false>(c, qx, qc, qs, kx, kc, ks, vx, vamax, vt, vs, nbq, nbk,
                                       BHq, BHk, rope, rope_k, rq, rk, st, kvsrc);
  } else {
    s = f16 ? quant_launch<64, true>(c, qx, qc, qs, kx, kc, ks, vx, vamax, vt, vs, nbq, nbk,
                                     BHq, BHk, rope, rope_k, rq, rk, st, kvsrc)
            : quant_launch<64, false>(c, qx, qc, qs, kx, kc, ks, vx, vamax, vt, vs, nbq, nbk,
                                      BHq, BHk, rope, rope_k, rq, rk, st, kvsrc);
  }
  if (s != ATTN_OK) return s;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Launches the forward on `st` for the units [u0, u0 + nu).  Pointers are those
// of the whole problem, already validated.  The split-KV path keeps its partials
// in the context's workspace, so it only runs on the whole problem at once.
attn_status forward_units(attn_ctx* c, int u0, int nu, const void* q, const void* k,
                          const void* v, const attn_qbufs* qb, void* o, float* lse,
                          cudaStream_t st, int slot) {
  if (c->split_path && (u0 != 0 || nu != c->units)) return ATTN_ERR_INVALID_ARG;
  const attn_params& p = c->p;
  const bool quant = p.precision != ATTN_EXACT;        // INT8/FP8 codes (both quantised modes)
  const bool diag = p.precision == ATTN_MIXED_DIAG;    // plus 16-bit Q, K for the band tiles
  const int D = p.head_dim;
  const bool f16 = p.dtype == ATTN_FP16;
  const size_t rows = static_cast<size_t>(nu) * c->R;
  if (rows == 0) return ATTN_OK;
  // Every tensor is unit-major: move each base to unit u0 (the kernels index
  // from their base, so a range of units is just a smaller problem).
  const size_t qe = static_cast<size_t>(u0) * c->R * D;      // Q, O elements before u0
  const size_t ke = static_cast<size_t>(u0) * p.kv_len * D;  // K, V elements before u0
  o = static_cast<uint16_t*>(o) + qe;
  if (lse) lse += static_cast<size_t>(u0) * c->R;
  if (p.kv_len == 0) {  // every row sees no key
    if (cudaMemsetAsync(o, 0, rows * D * 2, st) != cudaSuccess) return ATTN_ERR_CUDA;
    if (lse) fill_lse_kernel<<<ceil_div(rows, 256), 256, 0, st>>>(lse, rows);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  attn_qbufs qo{};
  const bool fp4 = p.precision == ATTN_MXFP4QK_FP8PV;
  if (quant) {
    const int nbq = ceil_div(p.q_len, 128), nbk = ceil_div(p.kv_len, 128);
    const size_t half = fp4 ? 2 : 1;  // FP4: two codes per byte
    qo.q = qb->q + qe / half;
    qo.k = qb->k + ke / half;
    if (fp4) {
      qo.q_sf = qb->q_sf + static_cast<size_t>(u0) * fp4_q_tiles(p) * 512;
      qo.k_sf = qb->k_sf + static_cast<size_t>(u0) * nbk * 512;
    } else {
      qo.q_scale = qb->q_scale + static_cast<size_t>(u0) * c->G * nbq;
      qo.k_scale = qb->k_scale + static_cast<size_t>(u0) * nbk;
    }
    qo.v_t = qb->v_t + static_cast<size_t>(u0) * D * (static_cast<size_t>(nbk) * 128);
    qo.v_scale = qb->v_scale + static_cast<size_t>(u0) * D;
    qb = &qo;
  }
  if (!quant || diag) {
    q = static_cast<const uint16_t*>(q) + qe;
    k = static_cast<const uint16_t*>(k) + ke;
    if (!quant) v = static_cast<const uint16_t*>(v) + ke;
    if (!quant && p.rope_dim > 0 && !p.rope_keys_rotated) {
      // the range's keys, rotated once into the workspace (positions 0 .. kv_len-1)
      uint16_t* kr = static_cast<uint16_t*>(c->ws_k) + ke;
      const attn_status rs = launch_rope_apply(c, k, kr, static_cast<long long>(nu) * p.kv_len,
                                               p.kv_len, 0, st);
      if (rs != ATTN_OK) return rs;
      k = kr;
    }
  }

  // Tensor maps.  Q, O: [units][R][D]; K, V: [units][Skv][D]; V^T: [units][D][S_pad].
  const CUtensorMapDataType t16 =
      f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t R = c->R, Sk = p.kv_len, U = nu;
  MapCache& mc = c->maps[slot];
  if (c->decode) {  // K and V in boxes of one key chunk; Q and O by plain loads and stores
    const void* key[6] = {k, v, nullptr, nullptr, nullptr, nullptr};
    bool hit = mc.valid && mc.nu == nu;
    for (int i = 0; i < 6; ++i) hit = hit && mc.key[i] == key[i];
    if (!hit) {
      const uint32_t rows = decode_chunk(D);
      bool ok = make_map(&mc.m.k, t16, k, D, Sk, U, D * 2, Sk * D * 2, 64, rows,
                         CU_TENSOR_MAP_SWIZZLE_128B);
      ok &= make_map(&mc.m.v, t16, v, D, Sk, U, D * 2, Sk * D * 2, 64, rows,
                     CU_TENSOR_MAP_SWIZZLE_128B);
      mc.valid = ok;
      mc.nu = nu;
      for (int i = 0; i < 6; ++i) mc.key[i] = key[i];
      if (!ok) return ATTN_ERR_CUDA;
    }
    const DecArgs a = decode_args(c, q, o, lse);
    return D == 128 ? dispatch_decode<128, false>(c, mc.m.k, mc.m.v, a, nu, st)
                    : dispatch_decode<64, false>(c, mc.m.k, mc.m.v, a, nu, st);
  }
  const void* key[6] = {quant ? static_cast<const void*>(qb->q) : q,
                        quant ? static_cast<const void*>(qb->k) : k,
                        quant ? static_cast<const void*>(qb->v_t) : v, o,
                        diag ? q : nullptr, diag ? k : nullptr};
  bool hit = mc.valid && mc.nu == nu;
  for (int i = 0; i < 6; ++i) hit = hit && mc.key[i] == key[i];
  FwdMaps& m = mc.m;
  bool ok = true;
  if (hit) {
  } else if (quant) {
    const CUtensorMapSwizzle sw8 =
        fp4 ? CU_TENSOR_MAP_SWIZZLE_32B
            : (D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
    const uint64_t S_pad = static_cast<uint64_t>(ceil_div(p.kv_len, 128)) * 128;
    const uint64_t W = fp4 ? D / 2 : D;  // bytes per row of the Q/K codes
    ok &= make_map(&m.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, qb->q, W, R, U, W, R * W, W, 128, sw8);
    ok &= make_map(&m.k, CU_TENSOR_MAP_DATA_TYPE_UINT8, qb->k, W, Sk, U, W, Sk * W, W, 128, sw8);
    ok &= make_map(&m.v, CU_TENSOR_MAP_DATA_TYPE_UINT8, qb->v_t, S_pad, D, U, S_pad, S_pad * D,
                   128, D, CU_TENSOR_MAP_SWIZZLE_128B);
    if (diag) {
      ok &= make_map(&m.q16, t16, q, D, R, U, D * 2, R * D * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B);
      ok &= make_map(&m.k16, t16, k, D, Sk, U, D * 2, Sk * D * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
      m.q16 = m.q;
      m.k16 = m.k;
    }
  } else {
    ok &= make_map(&m.q, t16, q, D, R, U, D * 2, R * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&m.k, t16, k, D, Sk, U, D * 2, Sk * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&m.v, t16, v, D, Sk, U, D * 2, Sk * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    m.q16 = m.q;
    m.k16 = m.k;
  }
  if (!hit) {
    ok &= make_map(&m.o, t16, o, D, R, U, D * 2, R * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    mc.valid = ok;
    mc.nu = nu;
    for (int i = 0; i < 6; ++i) mc.key[i] = key[i];
  }
  if (!ok) return ATTN_ERR_CUDA;

  FwdArgs a{};
  a.R = c->R;
  a.Sq = p.q_len;
  a.Skv = p.kv_len;
  a.G = c->G;
  a.units = nu;
  a.row_tiles = c->row_tiles;
  a.splits = c->splits;
  a.tiles_per_split = c->tiles_per_split;
  a.start_pos = p.start_pos;
  a.causal = p.causal;
  a.window_lo = p.window_lo;
  a.window_size = p.window_size;
  a.scale_log2 = c->scale * 1.4426950408889634f;
  a.lse = lse;
  a.o_part = c->o_part;
  a.lse_part = c->lse_part;
  a.part_rows = c->units * c->R;  // split path: every row
  if (quant) {
    a.q_scale = qb->q_scale;
    a.k_scale = qb->k_scale;
    a.v_scale = qb->v_scale;
  }
  a.nblk_q = ceil_div(p.q_len, 128);
  a.nblk_k = ceil_div(p.kv_len, 128);
  a.err = c->err;
  a.debug = c->debug;
  if (!quant && p.rope_dim > 0) {
    a.rope_table = c->rope_table;
    a.rope_R = p.rope_dim;
    a.rope_inter = p.rope_interleaved;
  }
  if (fp4) {
    a.q_sf = qb->q_sf;
    a.k_sf = qb->k_sf;
    a.q_tiles = fp4_q_tiles(p);
  }
  a.tph = causal_band_tiles(c);

  auto run = [&](const FwdArgs& fa, int grid, bool split) -> attn_status {
    if (D == 128) {
      if (quant) return f16 ? dispatch_fwd<128, true, true>(c, m, fa, grid, st, split)
                            : dispatch_fwd<128, true, false>(c, m, fa, grid, st, split);
      return f16 ? dispatch_fwd<128, false, true>(c, m, fa, grid, st, split)
                 : dispatch_fwd<128, false, false>(c, m, fa, grid, st, split);
    }
    if (quant) return f16 ? dispatch_fwd<64, true, true>(c, m, fa, grid, st, split)
                          : dispatch_fwd<64, true, false>(c, m, fa, grid, st, split);
    return f16 ? dispatch_fwd<64, false, true>(c, m, fa, grid, st, split)
               : dispatch_fwd<64, false, false>(c, m, fa, grid, st, split);
  };
  // merge of the partials of rows row0 .. row0 + rows - 1 (of this call's units);
  // split sp of a row is at sp * stride in the partial buffers op, lp
  auto merge = [&](const float* op, const float* lp, size_t row0, int rows, int stride,
                   int splits) -> attn_status {
    uint16_t* out = static_cast<uint16_t*>(o) + row0 * D;
    float* l = lse ? lse + row0 : nullptr;
    if (D == 128)
      return f16 ? launch_merge_rows<128, true>(op, lp, out, l, rows, stride, splits, st)
                 : launch_merge_rows<128, false>(op, lp, out, l, rows, stride, splits, st);
    return f16 ? launch_merge_rows<64, true>(op, lp, out, l, rows, stride, splits, st)
               : launch_merge_rows<64, false>(op, lp, out, l, rows, stride, splits, st);
  };
  if (c->split_path) {
    const attn_status s = run(a, nu * c->row_tiles * c->splits, true);
    if (s != ATTN_OK) return s;
    const int rows = c->units * c->R;
    return merge(c->o_part, c->lse_part, 0, rows, rows, c->splits);
  }
  const int nctas = nu * c->row_tiles;
  if (c->tail_items > 0) {
    // Short last wave: the last tail_items CTAs of the whole problem's single-pass
    // grid (256 rows each) run instead as the split kernel over their 128-row tiles
    // with tail_k key splits, and a merge of those rows; the others fill whole
    // waves.  A range of units takes the same split for the same rows, so every
    // row is computed the same way whatever the range (partials by global row).
    const int main_g = c->units * c->row_tiles - c->tail_items;  // first tail CTA
    const int first = u0 * c->row_tiles;                          // this range's first
    const int n_main = std::max(0, std::min(nctas, main_g - first));
    const int n_tail = nctas - n_main;
    attn_status s = ATTN_OK;
    if (n_main > 0) s = run(a, n_main, false);
    if (s != ATTN_OK || n_tail == 0) return s;
    const int pstride = c->tail_items * 256;                   // partial rows (whole tail)
    FwdArgs at = a;
    at.row_tiles = c->R / 128;
    at.splits = c->tail_k;
    at.tiles_per_split = ceil_div(ceil_div(p.kv_len, 128), c->tail_k);
    at.tile0 = 2 * n_main;
    at.part_row0 = main_g * 256 - u0 * c->R;                   // range-local row of partial 0
    at.part_rows = pstride;
    at.o_part = c->tail_opart;
    at.lse_part = c->tail_lse;
    at.tph = 0;
    s = run(at, 2 * n_tail * c->tail_k, true);
    if (s != ATTN_OK) return s;
    const size_t p0 = static_cast<size_t>(first + n_main - main_g) * 256;  // first partial row
    return merge(c->tail_opart + p0 * D, c->tail_lse + p0, static_cast<size_t>(n_main) * 256,
                 n_tail * 256, pstride, c->tail_k);
  }
  return run(a, nctas, false);
}

// Creates attn_forward_host's streams and events on the current device (all or none).
attn_status ensure_pipeline(attn_ctx* c) {
  if (c->pipe_ready) return ATTN_OK;
  constexpr int kEvents = 1 + 4 + 2 * kMaxHostChunks;
  cudaStream_t st[4] = {};
  cudaEvent_t ev[kEvents] = {};
  int ns = 0, ne = 0;
  while (ns < 4 && cudaStreamCreateWithFlags(&st[ns], cudaStreamNonBlocking) == cudaSuccess) ++ns;
  if (ns == 4)
    while (ne < kEvents && cudaEventCreateWithFlags(&ev[ne], cudaEventDisableTiming) == cudaSuccess)
      ++ne;
  if (ns < 4 || ne < kEvents) {  // release what was created
    for (int i = 0; i < ne; ++i) cudaEventDestroy(ev[i]);
    for (int i = 0; i < ns; ++i) cudaStreamDestroy(st[i]);
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  for (int i = 0; i < 4; ++i) c->pipe[i] = st[i];
  c->pev_start = ev[0];
  for (int i = 0; i < 4; ++i) c->pev_join[i] = ev[1 + i];
  for (int i = 0; i < kMaxHostChunks; ++i) {
    c->pev_in[i] = ev[5 + i];
    c->pev_done[i] = ev[5 + kMaxHostChunks + i];
  }
  c->pipe_ready = true;
  return ATTN_OK;
}

// Number of unit ranges attn_forward_host cuts a problem into when the caller
// leaves it to the library: about 24 MiB of inputs per range, at most
// kMaxHostChunks.  The pipeline's fill and drain (the first range's inputs, the
// last range's kernels and outputs) shrink with the range, but a range's kernel
// cannot finish faster than its longest CTA, which sits on the pipeline's
// critical path once per range.  On a PCIe 5.0 x16 host both the 1 x 40 x
// 32760 x 128 MHA problem (40 ranges) and the 4 x 32/8 x 8192 x 128 causal GQA
// one (16 ranges) ran fastest near this size.
int default_host_chunks(const attn_ctx* c) {
  const attn_params& p = c->p;
  const double in_bytes = static_cast<double>(c->units) *
                          (static_cast<double>(c->R) + 2.0 * p.kv_len) * p.head_dim * 2.0;
  const int n = static_cast<int>(in_bytes / (24.0 * 1024 * 1024) + 0.5);
  return std::max(1, std::min(n, kMaxHostChunks));
}

// Size of the pieces attn_forward_host copies O back in.  Host-to-device and
// device-to-host copies share the PCIe link unevenly: measured on a PCIe 5.0 x16
// host, with the outputs copied back in 1 MiB pieces the inputs kept ~51 GB/s and
// the outputs got ~23 GB/s; in 8 MiB pieces 49 and 40; as one large copy 37 and
// 47.  The inputs are the larger stream, so the pieces are the smallest whose
// rate still keeps up with the inputs at the problem's output/input byte ratio.
size_t d2h_piece_bytes(size_t out_per_unit, size_t in_per_unit) {
  const double ratio = static_cast<double>(out_per_unit) / static_cast<double>(in_per_unit);
  const size_t mib = size_t(1) << 20;
  return ratio <= 0.4 ? mib : ratio <= 0.6 ? 2 * mib : ratio <= 0.8 ? 4 * mib : 8 * mib;
}

// Marks the end of a call's work on `st` (everything it enqueued, errors included).
attn_status mark_done(attn_ctx* c, attn_status s, cudaStream_t st) {
  // A call captured into a CUDA graph runs when the graph is launched: the event
  // cannot mark it (an event last recorded during capture cannot be waited for
  // outside the graph), so it keeps marking the context's last direct call.
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return s == ATTN_OK ? ATTN_ERR_CUDA : s;
  }
  if (cs != cudaStreamCaptureStatusNone) return s;
  if (cudaEventRecord(c->done_ev, st) != cudaSuccess && s == ATTN_OK) return ATTN_ERR_CUDA;
  return s;
}

// With RoPE the context needs its table before anything is launched.
bool rope_ready(const attn_ctx* c) { return c->p.rope_dim == 0 || c->rope_table != nullptr; }

}  // namespace

extern "C" {

const char* attn_status_string(attn_status s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_OOM: return "out of device memory";
    case ATTN_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

attn_status attn_qbufs_sizes(const attn_params* p, size_t sizes[6]) {
  if (!sizes) return ATTN_ERR_INVALID_ARG;
  attn_status v = validate(p);
  if (v != ATTN_OK) return v;
  const size_t B = p->batch, Hq = p->n_q_heads, Hk = p->n_kv_heads, D = p->head_dim;
  const size_t Sq = p->q_len, Sk = p->kv_len;
  const size_t nbq = (Sq + 127) / 128, nbk = (Sk + 127) / 128;
  sizes[0] = B * Hq * Sq * D;
  sizes[1] = B * Hk * Sk * D;
  sizes[2] = B * Hq * nbq * 4;
  sizes[3] = B * Hk * nbk * 4;
  sizes[4] = B * Hk * D * nbk * 128;
  sizes[5] = B * Hk * D * 4;
  if (p->precision == ATTN_MXFP4QK_FP8PV) {  // packed E2M1 codes; no FP32 Q/K scales
    sizes[0] /= 2;
    sizes[1] /= 2;
    sizes[2] = sizes[3] = 0;
  }
  return ATTN_OK;
}

attn_status attn_qbufs_sf_sizes(const attn_params* p, size_t sizes[2]) {
  if (!sizes) return ATTN_ERR_INVALID_ARG;
  attn_status v = validate(p);
  if (v != ATTN_OK) return v;
  sizes[0] = sizes[1] = 0;
  if (p->precision == ATTN_MXFP4QK_FP8PV) {
    const size_t units = static_cast<size_t>(p->batch) * p->n_kv_heads;
    sizes[0] = units * fp4_q_tiles(*p) * 512;
    sizes[1] = units * ((static_cast<size_t>(p->kv_len) + 127) / 128) * 512;
  }
  return ATTN_OK;
}

attn_status attn_create(const attn_params* p, attn_ctx** out) {
  if (!out) return ATTN_ERR_INVALID_ARG;
  *out = nullptr;
  attn_status v = validate(p);
  if (v != ATTN_OK) return v;

  int dev = 0, sms = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (major != 10) return ATTN_ERR_UNSUPPORTED;  // built for sm_100a only

  attn_ctx* c = new attn_ctx();
  c->p = *p;
  c->device = dev;
  c->num_sms = sms;
  c->G = p->n_q_heads / p->n_kv_heads;
  c->R = c->G * p->q_len;
  c->units = p->batch * p->n_kv_heads;
  c->scale = p->scale > 0.0f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->head_dim));
  const int kv_tiles = ceil_div(p->kv_len, 128);

  Plan pl;
  plan_problem(*p, sms, pl, [&](int S) {
    return p->head_dim == 128 ? decode_max_clusters<128>(c->units, S)
                              : decode_max_clusters<64>(c->units, S);
  });
  const bool split = pl.path == ATTN_PATH_SPLIT_MERGE;
  c->decode = pl.path == ATTN_PATH_DECODE ? 1 : 0;
  c->split_path = split ? 1 : 0;
  c->splits = pl.splits;
  c->tiles_per_split = pl.tiles_per_split;
  c->row_tiles = pl.row_tiles;
  c->dec_chunk0 = pl.dec_chunk0;
  c->dec_nchunks = pl.dec_nchunks;
  if (c->decode) {
    // the merge area for this S, and two ring slots per warp: the K/V stream is
    // bound by the bytes the whole GPU has in flight, and a third slot per warp
    // measured slower (decode workload: 9.3 against 8.2 us per call back to back)
    const int S = pl.splits;
    const int rpo = (c->R + S - 1) / S;
    const bool d128 = p->head_dim == 128;
    c->dec_owner_slots = DecCfg<128>::kWarps * S * rpo;
    const int nsw = 2;
    c->dec_nsw = nsw;
    c->dec_smem = d128 ? DecCfg<128>::smem_bytes(nsw, c->dec_owner_slots)
                       : DecCfg<64>::smem_bytes(nsw, c->dec_owner_slots);
  }

  // workspace: error word | V channel maxima | split partials
  size_t off = 256;
  size_t vamax_off = 0, opart_off = 0, lpart_off = 0;
  if (p->precision != ATTN_EXACT) {
    vamax_off = off;
    off += (static_cast<size_t>(c->units) * p->head_dim * 4 + 255) / 256 * 256;
  }
  if (split) {
    const size_t rows = static_cast<size_t>(c->units) * c->R;
    opart_off = off;
    off += (static_cast<size_t>(c->splits) * rows * p->head_dim * 4 + 255) / 256 * 256;
    lpart_off = off;
    off += (2 * static_cast<size_t>(c->splits) * rows * 4 + 255) / 256 * 256;
  }
  // Tail of the single-pass grid (non-causal, whole 256-row tiles, library's split
  // choice; the band and FP4 modes have no split variant): when the CTAs leave a
  // last wave at most half full, its CTAs' keys are split instead.
  size_t topart_off = 0, tlse_off = 0;
  if (pl.path == ATTN_PATH_SINGLE_PASS_TAIL) {
    const int T = pl.tail_items, k = pl.tail_splits;
    c->tail_items = T;
    c->tail_k = k;
    const size_t rows = static_cast<size_t>(T) * 256;
    topart_off = off;
    off += (static_cast<size_t>(k) * rows * p->head_dim * 4 + 255) / 256 * 256;
    tlse_off = off;
    off += (2 * static_cast<size_t>(k) * rows * 4 + 255) / 256 * 256;
  }
  if (cudaEventCreateWithFlags(&c->done_ev, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    delete c;
    return ATTN_ERR_CUDA;
  }
  if (cudaMalloc(&c->ws, off) != cudaSuccess) {
    cudaGetLastError();
    cudaEventDestroy(c->done_ev);
    delete c;
    return ATTN_ERR_OOM;
  }
  c->ws_bytes = off;
  if (p->rope_dim > 0 && !p->rope_keys_rotated && p->precision == ATTN_EXACT) {
    const size_t kbytes = static_cast<size_t>(c->units) * p->kv_len * p->head_dim * 2;
    if (kbytes > 0 && cudaMalloc(&c->ws_k, kbytes) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(c->ws);
      cudaEventDestroy(c->done_ev);
      delete c;
      return ATTN_ERR_OOM;
    }
  }
  uint8_t* base = static_cast<uint8_t*>(c->ws);
  c->err = reinterpret_cast<unsigned*>(base);
  c->v_amax = vamax_off ? reinterpret_cast<unsigned*>(base + vamax_off) : nullptr;
  c->o_part = split ? reinterpret_cast<float*>(base + opart_off) : nullptr;
  c->lse_part = split ? reinterpret_cast<float*>(base + lpart_off) : nullptr;
  c->tail_opart = c->tail_items ? reinterpret_cast<float*>(base + topart_off) : nullptr;
  c->tail_lse = c->tail_items ? reinterpret_cast<float*>(base + tlse_off) : nullptr;
  if (cudaMemset(c->err, 0, 256) != cudaSuccess) {
    cudaFree(c->ws);
    if (c->ws_k) cudaFree(c->ws_k);
    cudaEventDestroy(c->done_ev);
    delete c;
    return ATTN_ERR_CUDA;
  }
  *out = c;
  return ATTN_OK;
}

void attn_destroy(attn_ctx* c) {
  if (!c) return;
  // Wait for the context's own work only: its last call, and the streams of the
  // host pipeline.  (Other work on the device is not waited for here.)
  cudaEventSynchronize(c->done_ev);
  if (c->pipe_ready)
    for (int i = 0; i < 4; ++i) cudaStreamSynchronize(c->pipe[i]);
  cudaFree(c->ws);
  if (c->ws_k) cudaFree(c->ws_k);
  cudaEventDestroy(c->done_ev);
  if (c->pipe_ready) {
    for (int i = 0; i < 4; ++i) {
      cudaStreamDestroy(c->pipe[i]);
      cudaEventDestroy(c->pev_join[i]);
    }
    for (int i = 0; i < kMaxHostChunks; ++i) {
      cudaEventDestroy(c->pev_in[i]);
      cudaEventDestroy(c->pev_done[i]);
    }
    cudaEventDestroy(c->pev_start);
  }
  delete c;
  cudaGetLastError();  // these calls report nothing: leave no error for the next launch check
}

int attn_num_splits(const attn_ctx* c) {
  return c ? ((c->split_path || c->decode) ? c->splits : 1) : 0;
}

attn_status attn_plan_for(const attn_params* p, int num_sms, attn_plan* out) {
  if (!out || num_sms < 1) return ATTN_ERR_INVALID_ARG;
  const attn_status v = validate(p);
  if (v != ATTN_OK) return v;
  Plan pl;
  plan_problem(*p, num_sms, pl, [](int) { return 1 << 30; });
  const int units = p->batch * p->n_kv_heads;
  out->path = pl.path;
  out->splits = pl.splits;
  out->tiles_per_split = pl.path == ATTN_PATH_SPLIT_MERGE ? pl.tiles_per_split : 0;
  out->ctas = pl.path == ATTN_PATH_DECODE
                  ? units * pl.splits
                  : units * pl.row_tiles * (pl.path == ATTN_PATH_SPLIT_MERGE ? pl.splits : 1) -
                        pl.tail_items;
  out->tail_items = pl.tail_items;
  out->tail_splits = pl.tail_splits;
  out->decode_chunk = pl.path == ATTN_PATH_DECODE ? static_cast<int>(decode_chunk(p->head_dim)) : 0;
  out->decode_chunks = pl.dec_nchunks;
  return ATTN_OK;
}

int attn_kernel_path(const attn_ctx* c) {
  if (!c) return 0;
  if (c->decode) return ATTN_PATH_DECODE;
  if (c->split_path) return ATTN_PATH_SPLIT_MERGE;
  return c->tail_items > 0 ? ATTN_PATH_SINGLE_PASS_TAIL : ATTN_PATH_SINGLE_PASS;
}

attn_status attn_debug_set(attn_ctx* c, unsigned flags) {
  if (!c) return ATTN_ERR_INVALID_ARG;
  c->debug = flags;
  return ATTN_OK;
}

attn_status attn_debug_exp2(const float* x, float* y, size_t n, void* stream) {
  if ((!x || !y) && n > 0) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  poly_exp2_kernel<<<ceil_div(static_cast<long long>(n), 256), 256, 0,
                     static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status attn_get_error(attn_ctx* c, void* stream) {
  if (!c) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned h = 0;
  if (cudaMemcpy(&h, c->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  if (h != 0) {
    if (cudaMemset(c->err, 0, 4) != cudaSuccess) return ATTN_ERR_CUDA;
    // a paged quantiser met a block-table entry outside the pool; else a wait ran out
    return (h & kErrBadBlock) ? ATTN_ERR_INVALID_ARG : ATTN_ERR_TIMEOUT;
  }
  return ATTN_OK;
}

attn_status attn_quantize_qk(attn_ctx* c, const void* q, const void* k, const void* v,
                             const attn_qbufs* qb, void* stream) {
  if (!c || !qb) return ATTN_ERR_INVALID_ARG;
  if (c->p.precision == ATTN_EXACT || !rope_ready(c)) return ATTN_ERR_INVALID_ARG;
  const bool need_q = c->p.q_len > 0, need_kv = c->p.kv_len > 0;
  if (bad_ptr(q, need_q) || bad_ptr(k, need_kv) || bad_ptr(v, need_kv) || bad_qbufs(c->p, qb))
    return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return mark_done(c, quantize_units(c, 0, c->units, q, k, v, qb, st), st);
}

attn_status attn_quantize_qk_paged(attn_ctx* c, const void* q, const void* k_pool,
                                   const void* v_pool, const int32_t* block_table,
                                   int num_blocks, const attn_qbufs* qb, void* stream) {
  if (!c || !qb) return ATTN_ERR_INVALID_ARG;
  const attn_params& p = c->p;
  if (p.precision != ATTN_INT8QK_FP8PV) return ATTN_ERR_UNSUPPORTED;
  if (p.rope_dim > 0 && !p.rope_keys_rotated) return ATTN_ERR_UNSUPPORTED;  // pool keys rotated
  if (!rope_ready(c)) return ATTN_ERR_INVALID_ARG;
  const bool need_q = p.q_len > 0, need_kv = p.kv_len > 0;
  if (bad_ptr(q, need_q) || bad_ptr(k_pool, need_kv) || bad_ptr(v_pool, need_kv) ||
      bad_qbufs(p, qb) ||
      (need_kv && (block_table == nullptr || (reinterpret_cast<uintptr_t>(block_table) & 3u))) ||
      (need_kv && num_blocks < 1))
    return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const KvBlocks src{block_table, ceil_div(p.kv_len, 128), p.n_kv_heads, num_blocks, c->err};
  return mark_done(c, quantize_units(c, 0, c->units, q, k_pool, v_pool, qb, st, src), st);
}

attn_status attn_forward(attn_ctx* c, const void* q, const void* k, const void* v,
                         const attn_qbufs* qb, void* o, float* lse, void* stream) {
  if (!c || !rope_ready(c)) return ATTN_ERR_INVALID_ARG;
  const attn_status s = check_forward_buffers(c, q, k, v, qb, o, lse);
  if (s != ATTN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return mark_done(c, forward_units(c, 0, c->units, q, k, v, qb, o, lse, st, 0), st);
}

static attn_status forward_paged_impl(attn_ctx* c, const void* q, const void* k_pool,
                                      const void* v_pool, const int32_t* block_table,
                                      int num_blocks, void* o, float* lse, void* stream) {
  const attn_params& p = c->p;
  if (p.precision != ATTN_EXACT) return ATTN_ERR_UNSUPPORTED;
  if (p.rope_dim > 0 && !p.rope_keys_rotated) return ATTN_ERR_UNSUPPORTED;  // pool keys rotated
  if (!rope_ready(c)) return ATTN_ERR_INVALID_ARG;
  const bool need_q = p.q_len > 0, need_kv = p.kv_len > 0;
  if (bad_ptr(q, need_q) || bad_ptr(o, need_q) || (lse && !aligned16(lse)) ||
      bad_ptr(k_pool, need_kv) || bad_ptr(v_pool, need_kv) ||
      (need_kv && (block_table == nullptr || (reinterpret_cast<uintptr_t>(block_table) & 3u))) ||
      (need_kv && num_blocks < 1))
    return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = p.head_dim;
  const bool f16 = p.dtype == ATTN_FP16;
  const size_t rows = static_cast<size_t>(c->units) * c->R;
  if (rows == 0) return ATTN_OK;
  if (p.kv_len == 0) {  // every row sees no key
    if (cudaMemsetAsync(o, 0, rows * D * 2, st) != cudaSuccess) return ATTN_ERR_CUDA;
    if (lse) fill_lse_kernel<<<ceil_div(rows, 256), 256, 0, st>>>(lse, rows);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  const CUtensorMapDataType t16 =
      f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (c->decode) {
    CUtensorMap mk, mv;
    const uint32_t crow = decode_chunk(D);
    bool ok = make_pool_map(&mk, t16, k_pool, D, p.n_kv_heads, num_blocks, crow);
    ok &= make_pool_map(&mv, t16, v_pool, D, p.n_kv_heads, num_blocks, crow);
    if (!ok) return ATTN_ERR_CUDA;
    DecArgs a = decode_args(c, q, o, lse);
    a.block_table = block_table;
    a.bt_stride = ceil_div(p.kv_len, 128);
    a.n_kv_heads = p.n_kv_heads;
    return D == 128 ? dispatch_decode<128, true>(c, mk, mv, a, c->units, st)
                    : dispatch_decode<64, true>(c, mk, mv, a, c->units, st);
  }
  const uint64_t R = c->R, U = c->units;
  FwdMaps m;
  bool ok = make_map(&m.q, t16, q, D, R, U, D * 2, R * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_pool_map(&m.k, t16, k_pool, D, p.n_kv_heads, num_blocks);
  ok &= make_pool_map(&m.v, t16, v_pool, D, p.n_kv_heads, num_blocks);
  ok &= make_map(&m.o, t16, o, D, R, U, D * 2, R * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  m.q16 = m.q;
  m.k16 = m.k;
  if (!ok) return ATTN_ERR_CUDA;
  FwdArgs a{};
  a.R = c->R;
  a.Sq = p.q_len;
  a.Skv = p.kv_len;
  a.G = c->G;
  a.units = c->units;
  a.row_tiles = c->row_tiles;
  a.splits = c->splits;
  a.tiles_per_split = c->tiles_per_split;
  a.start_pos = p.start_pos;
  a.causal = p.causal;
  a.window_lo = p.window_lo;
  a.window_size = p.window_size;
  a.block_table = block_table;
  a.bt_stride = ceil_div(p.kv_len, 128);
  a.tph = causal_band_tiles(c);
  if (p.rope_dim > 0) {
    a.rope_table = c->rope_table;
    a.rope_R = p.rope_dim;
    a.rope_inter = p.rope_interleaved;
  }
  a.n_kv_heads = p.n_kv_heads;
  a.scale_log2 = c->scale * 1.4426950408889634f;
  a.lse = lse;
  a.o_part = c->o_part;
  a.lse_part = c->lse_part;
  a.part_rows = c->units * c->R;  // split path: every row
  a.nblk_q = ceil_div(p.q_len, 128);
  a.nblk_k = ceil_div(p.kv_len, 128);
  a.err = c->err;
  a.debug = c->debug;
  const int grid = c->units * c->row_tiles * (c->split_path ? c->splits : 1);
  attn_status s;
  if (D == 128)
    s = f16 ? dispatch_fwd<128, false, true>(c, m, a, grid, st, c->split_path)
            : dispatch_fwd<128, false, false>(c, m, a, grid, st, c->split_path);
  else
    s = f16 ? dispatch_fwd<64, false, true>(c, m, a, grid, st, c->split_path)
            : dispatch_fwd<64, false, false>(c, m, a, grid, st, c->split_path);
  if (s != ATTN_OK || !c->split_path) return s;
  if (D == 128)
    return f16 ? launch_merge<128, true>(c, o, lse, st) : launch_merge<128, false>(c, o, lse, st);
  return f16 ? launch_merge<64, true>(c, o, lse, st) : launch_merge<64, false>(c, o, lse, st);
}

attn_status attn_forward_paged(attn_ctx* c, const void* q, const void* k_pool,
                               const void* v_pool, const int32_t* block_table, int num_blocks,
                               void* o, float* lse, void* stream) {
  if (!c) return ATTN_ERR_INVALID_ARG;
  return mark_done(c,
                   forward_paged_impl(c, q, k_pool, v_pool, block_table, num_blocks, o, lse,
                                      stream),
                   static_cast<cudaStream_t>(stream));
}

static attn_status forward_host_impl(attn_ctx* c, const void* q_host, const void* k_host,
                                     const void* v_host, void* o_host, float* lse_host,
                                     void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                                     float* lse_dev, const attn_qbufs* qb, int chunks,
                                     void* stream) {
  if (chunks < 0 || chunks > kMaxHostChunks || !rope_ready(c)) return ATTN_ERR_INVALID_ARG;
  const attn_params& p = c->p;
  const bool quant = p.precision != ATTN_EXACT;
  const bool need_q = p.q_len > 0, need_kv = p.kv_len > 0;
  if ((need_q && (!q_host || !o_host)) || (need_kv && (!k_host || !v_host)))
    return ATTN_ERR_INVALID_ARG;
  if ((lse_host == nullptr) != (lse_dev == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (bad_ptr(q_dev, need_q) || bad_ptr(k_dev, need_kv) || bad_ptr(v_dev, need_kv) ||
      bad_ptr(o_dev, need_q) || (lse_dev && !aligned16(lse_dev)))
    return ATTN_ERR_INVALID_ARG;
  if (quant ? bad_qbufs(p, qb) : qb != nullptr) return ATTN_ERR_INVALID_ARG;
  if (static_cast<size_t>(c->units) * c->R == 0) return ATTN_OK;
  attn_status s = ensure_pipeline(c);
  if (s != ATTN_OK) return s;

  const int U = c->units;
  int n = chunks > 0 ? chunks : default_host_chunks(c);
  n = c->split_path ? 1 : std::min(n, U);
  const size_t qU = static_cast<size_t>(c->R) * p.head_dim * 2;   // Q or O bytes per unit
  const size_t kU = static_cast<size_t>(p.kv_len) * p.head_dim * 2;  // K or V bytes per unit
  const size_t lU = static_cast<size_t>(c->R) * 4;                // lse bytes per unit
  auto copy = [](void* dst, const void* src, size_t off, size_t bytes, cudaMemcpyKind kind,
                 cudaStream_t cs) {
    if (bytes == 0) return true;
    return cudaMemcpyAsync(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off,
                           bytes, kind, cs) == cudaSuccess;
  };
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t h2d = c->pipe[0], d2h = c->pipe[3];
  const size_t piece = d2h_piece_bytes(qU, qU + 2 * kU);
  auto bounds = [&](int i, int* u0, int* nu) {
    *u0 = static_cast<int>(static_cast<long long>(i) * U / n);
    *nu = static_cast<int>(static_cast<long long>(i + 1) * U / n) - *u0;
  };
  // Range j's outputs go back once its kernels are done and range j+1's inputs
  // are in, so that they never split the link with the input copy that the next
  // kernels wait on.
  auto copy_out = [&](int j) {
    int u0, nu;
    bounds(j, &u0, &nu);
    if (cudaStreamWaitEvent(d2h, c->pev_done[j], 0) != cudaSuccess) return false;
    if (j + 1 < n && cudaStreamWaitEvent(d2h, c->pev_in[j + 1], 0) != cudaSuccess) return false;
    for (size_t off = 0; off < nu * qU; off += piece)
      if (!copy(o_host, o_dev, u0 * qU + off, std::min(piece, nu * qU - off),
                cudaMemcpyDeviceToHost, d2h))
        return false;
    return !lse_dev || copy(lse_host, lse_dev, u0 * lU, nu * lU, cudaMemcpyDeviceToHost, d2h);
  };
  bool ok = cudaEventRecord(c->pev_start, st) == cudaSuccess;
  for (int i = 0; i < 4 && ok; ++i)
    ok = cudaStreamWaitEvent(c->pipe[i], c->pev_start, 0) == cudaSuccess;
  int issued = 0;  // ranges whose kernels are queued
  for (int i = 0; i < n && ok; ++i) {
    int u0, nu;
    bounds(i, &u0, &nu);
    cudaStream_t cs = c->pipe[1 + (i & 1)];
    const cudaMemcpyKind in = cudaMemcpyHostToDevice;
    ok = copy(q_dev, q_host, u0 * qU, nu * qU, in, h2d) &&
         copy(k_dev, k_host, u0 * kU, nu * kU, in, h2d) &&
         copy(v_dev, v_host, u0 * kU, nu * kU, in, h2d) &&
         cudaEventRecord(c->pev_in[i], h2d) == cudaSuccess &&
         cudaStreamWaitEvent(cs, c->pev_in[i], 0) == cudaSuccess;
    if (!ok) break;
    if (quant) {
      s = quantize_units(c, u0, nu, q_dev, k_dev, v_dev, qb, cs);
      // the band mode also reads the 16-bit Q and K of its diagonal tiles
      const bool diag = p.precision == ATTN_MIXED_DIAG;
      if (s == ATTN_OK)
        s = forward_units(c, u0, nu, diag ? q_dev : nullptr, diag ? k_dev : nullptr, nullptr, qb,
                          o_dev, lse_dev, cs, 1 + i);
    } else {
      s = forward_units(c, u0, nu, q_dev, k_dev, v_dev, nullptr, o_dev, lse_dev, cs, 1 + i);
    }
    if (s != ATTN_OK) break;
    ok = cudaEventRecord(c->pev_done[i], cs) == cudaSuccess;
    issued = i + 1;
    if (ok && i > 0) ok = copy_out(i - 1);
  }
  if (ok && s == ATTN_OK && issued == n) ok = copy_out(n - 1);
  // Join every pipeline stream back into the caller's stream, after an error too.
  for (int i = 0; i < 4; ++i)
    if (cudaEventRecord(c->pev_join[i], c->pipe[i]) != cudaSuccess ||
        cudaStreamWaitEvent(st, c->pev_join[i], 0) != cudaSuccess)
      ok = false;
  if (s != ATTN_OK) return s;
  return ok ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status attn_rope_table(int rope_dim, int n_pos, const attn_rope_freq* f, float* table) {
  if (!f || !table || rope_dim < 2 || rope_dim % 2 != 0 || n_pos < 1) return ATTN_ERR_INVALID_ARG;
  if (!(f->base > 0.0f) || !(f->factor >= 1.0f)) return ATTN_ERR_INVALID_ARG;
  if (f->scaling != ATTN_ROPE_PLAIN && f->scaling != ATTN_ROPE_NTK && f->scaling != ATTN_ROPE_YARN)
    return ATTN_ERR_INVALID_ARG;
  if (f->scaling == ATTN_ROPE_YARN && (f->original_len < 1 || !(f->beta_fast > f->beta_slow)))
    return ATTN_ERR_INVALID_ARG;
  const int half = rope_dim / 2;
  const double R = rope_dim, s = f->factor;
  double base = f->base;
  if (f->scaling == ATTN_ROPE_NTK) base *= std::pow(s, R / (R - 2.0));
  double m = 1.0;
  if (f->scaling == ATTN_ROPE_YARN && s > 1.0) m = 0.1 * std::log(s) + 1.0;
  const double two_pi = 6.283185307179586476925286766559;
  for (int i = 0; i < half; ++i) {
    double th = std::pow(base, -2.0 * i / R);
    if (f->scaling == ATTN_ROPE_YARN) {
      const double r = f->original_len * th / two_pi;
      double g = (r - f->beta_slow) / (static_cast<double>(f->beta_fast) - f->beta_slow);
      g = g < 0.0 ? 0.0 : (g > 1.0 ? 1.0 : g);
      th = (1.0 - g) * th / s + g * th;
    }
    for (int p = 0; p < n_pos; ++p) {
      const double ang = p * th;
      table[static_cast<size_t>(p) * rope_dim + i] = static_cast<float>(std::cos(ang) * m);
      table[static_cast<size_t>(p) * rope_dim + half + i] = static_cast<float>(std::sin(ang) * m);
    }
  }
  return ATTN_OK;
}

attn_status attn_set_rope_table(attn_ctx* c, const float* table, int n_pos) {
  if (!c || !table || !aligned16(table) || c->p.rope_dim == 0) return ATTN_ERR_INVALID_ARG;
  const long long need = std::max<long long>(static_cast<long long>(c->p.start_pos) + c->p.q_len,
                                             c->p.kv_len);
  if (n_pos < 1 || n_pos < need) return ATTN_ERR_INVALID_ARG;
  c->rope_table = table;
  c->rope_npos = n_pos;
  return ATTN_OK;
}

attn_status attn_rope_apply(attn_ctx* c, const void* x, void* y, int n_heads, int len, int pos0,
                            void* stream) {
  if (!c || c->p.rope_dim == 0 || !c->rope_table || n_heads < 1 || len < 0 || pos0 < 0)
    return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(pos0) + len > c->rope_npos) return ATTN_ERR_INVALID_ARG;
  const bool any = len > 0;
  if (bad_ptr(x, any) || bad_ptr(y, any)) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = static_cast<long long>(c->p.batch) * n_heads * len;
  return mark_done(c, launch_rope_apply(c, x, y, rows, len, pos0, st), st);
}

attn_status attn_forward_host(attn_ctx* c, const void* q_host, const void* k_host,
                              const void* v_host, void* o_host, float* lse_host, void* q_dev,
                              void* k_dev, void* v_dev, void* o_dev, float* lse_dev,
                              const attn_qbufs* qb, int chunks, void* stream) {
  if (!c) return ATTN_ERR_INVALID_ARG;
  return mark_done(c,
                   forward_host_impl(c, q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev,
                                     v_dev, o_dev, lse_dev, qb, chunks, stream),
                   static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation variant of the split-KV forward (see attn_forward_splitkv_noalloc
// in attn.h).  Its split partials live in this file-scope array instead of a
// context workspace: every GPU that loads the library holds these bytes until
// the process exits.  Layout: O partials | per-row statistics | error sink.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocPartFloats = size_t(1) << 20;  // 4 MiB of O partials
constexpr size_t kNoAllocStatFloats = size_t(1) << 15;  // 128 KiB of row statistics
constexpr size_t kNoAllocSinkFloats = 64;               // error word when the caller passes none
constexpr int kNoAllocMaxDevices = 64;
}  // namespace

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocPartFloats +
                                                         kNoAllocStatFloats +
                                                         kNoAllocSinkFloats];

namespace {
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  Host code must not
// use the symbol itself (it is a host-side stand-in, not a device address).
attn_status noalloc_scratch(int dev, float** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_noalloc_ptr[dev];
  return ATTN_OK;
}
}  // namespace

extern "C" attn_status attn_forward_splitkv_noalloc(const attn_params* p, const void* q,
                                                    const void* k, const void* v, void* o,
                                                    float* lse, unsigned* err, void* stream) {
  attn_status st = validate(p);
  if (st != ATTN_OK) return st;
  if (p->num_splits == 1) return ATTN_ERR_INVALID_ARG;  // always split: 0 or > 1
  if (p->precision != ATTN_EXACT || p->rope_dim != 0) return ATTN_ERR_UNSUPPORTED;
  const bool need_q = p->q_len > 0, need_kv = p->kv_len > 0;
  auto bad = [](const void* ptr, bool needed) {
    return needed ? (ptr == nullptr || !aligned16(ptr)) : (ptr != nullptr && !aligned16(ptr));
  };
  if (bad(q, need_q) || bad(o, need_q) || bad(k, need_kv) || bad(v, need_kv) ||
      (lse && !aligned16(lse)) || (err && (reinterpret_cast<uintptr_t>(err) & 3u)))
    return ATTN_ERR_INVALID_ARG;

  int dev = 0, sms = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (major != 10) return ATTN_ERR_UNSUPPORTED;

  // Same split choice as attn_create makes for the split-KV path.
  attn_ctx c{};
  c.p = *p;
  c.device = dev;
  c.num_sms = sms;
  c.G = p->n_q_heads / p->n_kv_heads;
  c.R = c.G * p->q_len;
  c.units = p->batch * p->n_kv_heads;
  c.scale = p->scale > 0.0f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->head_dim));
  const int kv_tiles = ceil_div(p->kv_len, 128);
  int splits = p->num_splits > 1
                   ? p->num_splits
                   : std::max(1, std::min(kv_tiles,
                                          ceil_div(2 * sms, c.units * ceil_div(c.R, 128))));
  splits = std::min(std::max(splits, 1), std::max(kv_tiles, 1));
  splits = std::min(splits, kMergeMaxSplits);
  c.split_path = 1;
  c.tiles_per_split = std::max(1, ceil_div(kv_tiles, splits));
  c.splits = std::max(1, ceil_div(kv_tiles, c.tiles_per_split));
  c.row_tiles = ceil_div(c.R, 128);

  const size_t rows = static_cast<size_t>(c.units) * c.R;
  if (rows == 0) return ATTN_OK;
  const size_t part_floats = static_cast<size_t>(c.splits) * rows * p->head_dim;
  const size_t stat_floats = 2 * static_cast<size_t>(c.splits) * rows;
  if (part_floats > kNoAllocPartFloats || stat_floats > kNoAllocStatFloats)
    return ATTN_ERR_UNSUPPORTED;  // larger than the static scratch: use attn_forward

  float* scratch = nullptr;
  st = noalloc_scratch(dev, &scratch);
  if (st != ATTN_OK) return st;
  c.o_part = scratch;
  c.lse_part = scratch + kNoAllocPartFloats;
  c.err = err ? err : reinterpret_cast<unsigned*>(scratch + kNoAllocPartFloats + kNoAllocStatFloats);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = p->head_dim;
  const bool f16 = p->dtype == ATTN_FP16;
  if (p->kv_len == 0) {  // every row sees no key
    if (cudaMemsetAsync(o, 0, rows * D * 2, s) != cudaSuccess) return ATTN_ERR_CUDA;
    if (lse) fill_lse_kernel<<<ceil_div(rows, 256), 256, 0, s>>>(lse, rows);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }

  const CUtensorMapDataType t16 =
      f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t R = c.R, Sk = p->kv_len, U = c.units;
  FwdMaps m;
  bool ok = true;
  ok &= make_map(&m.q, t16, q, D, R, U, D * 2, R * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&m.k, t16, k, D, Sk, U, D * 2, Sk * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&m.v, t16, v, D, Sk, U, D * 2, Sk * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&m.o, t16, o, D, R, U, D * 2, R * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  m.q16 = m.q;
  m.k16 = m.k;
  if (!ok) return ATTN_ERR_CUDA;

  FwdArgs a{};
  a.R = c.R;
  a.Sq = p->q_len;
  a.Skv = p->kv_len;
  a.G = c.G;
  a.units = c.units;
  a.row_tiles = c.row_tiles;
  a.splits = c.splits;
  a.tiles_per_split = c.tiles_per_split;
  a.start_pos = p->start_pos;
  a.causal = p->causal;
  a.window_lo = p->window_lo;
  a.window_size = p->window_size;
  a.scale_log2 = c.scale * 1.4426950408889634f;
  a.lse = lse;
  a.o_part = c.o_part;
  a.lse_part = c.lse_part;
  a.part_rows = c.units * c.R;  // split path: every row
  a.nblk_q = ceil_div(p->q_len, 128);
  a.nblk_k = kv_tiles;
  a.err = c.err;
  a.debug = 0;
  const int grid = c.units * c.row_tiles * c.splits;
  if (D == 128) {
    st = f16 ? dispatch_fwd<128, false, true>(&c, m, a, grid, s, true)
             : dispatch_fwd<128, false, false>(&c, m, a, grid, s, true);
    if (st == ATTN_OK)
      st = f16 ? launch_merge<128, true>(&c, o, lse, s) : launch_merge<128, false>(&c, o, lse, s);
  } else {
    st = f16 ? dispatch_fwd<64, false, true>(&c, m, a, grid, s, true)
             : dispatch_fwd<64, false, false>(&c, m, a, grid, s, true);
    if (st == ATTN_OK)
      st = f16 ? launch_merge<64, true>(&c, o, lse, s) : launch_merge<64, false>(&c, o, lse, s);
  }
  return st;
}
