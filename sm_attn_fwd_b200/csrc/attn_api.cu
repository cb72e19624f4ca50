// Host side of the C ABI declared in include/attn.h: argument validation,
// split planning, TMA tensor-map encoding and kernel launches.  Nothing here
// allocates device memory or synchronises, except attn_get_device_error.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "attn_bwd_params.h"
#include "attn_params.h"
#include "host_once.h"

namespace attn {
template <int D>
cudaError_t launch_decode(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                          const FwdParams&, dim3, cudaStream_t);
template <int D>
cudaError_t launch_combine(const FwdParams&, cudaStream_t);
template <int D>
cudaError_t launch_prefill(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                           const FwdParams&, int, cudaStream_t);

int* device_error_word();
template <int D>
cudaError_t launch_backward(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                            const CUtensorMap&, const CUtensorMap&, const BwdParams&,
                            cudaStream_t);
cudaError_t launch_selftest_wait(cudaStream_t stream);
template <int D>
cudaError_t launch_short(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                         const FwdParams&, int, cudaStream_t);
}  // namespace attn

namespace {

using attn::FwdParams;
using attn::kBlockM;
using attn::kBlockN;

constexpr long long kMaxGridY = 65535;

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

unsigned long long attn::current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
    ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(ptr);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Encoded tensor maps are a pure function of their arguments; a small
// per-thread cache skips the encode (a driver call) when a caller repeats a
// call on the same buffers and shapes, as decode and training loops do.
struct TmapKey {
  const void* base;
  uint64_t dims[3];
  int rank, box_rows, kind;
  bool operator==(const TmapKey& o) const {
    return base == o.base && rank == o.rank && box_rows == o.box_rows && kind == o.kind &&
           dims[0] == o.dims[0] && dims[1] == o.dims[1] && dims[2] == o.dims[2];
  }
};
constexpr int kTmapCacheSize = 16;
struct TmapCache {
  TmapKey key[kTmapCacheSize];
  CUtensorMap map[kTmapCacheSize];
  bool valid[kTmapCacheSize] = {};
  int next = 0;
};
thread_local TmapCache t_tmaps;

template <class Encode>
bool cached_encode(CUtensorMap* map, const TmapKey& key, Encode&& encode) {
  for (int i = 0; i < kTmapCacheSize; ++i) {
    if (t_tmaps.valid[i] && t_tmaps.key[i] == key) {
      *map = t_tmaps.map[i];
      return true;
    }
  }
  if (!encode(map)) return false;
  const int slot = t_tmaps.next;
  t_tmaps.next = (slot + 1) % kTmapCacheSize;
  t_tmaps.key[slot] = key;
  t_tmaps.map[slot] = *map;
  t_tmaps.valid[slot] = true;
  return true;
}

// bf16 tensor map of rank 2 or 3 (innermost first), boxes of 64 columns by
// box_rows rows, 128-byte swizzle; out-of-range rows read as zero.
bool encode_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 int box_rows = kBlockN) {
  TmapKey key{base, {dims[0], rank > 1 ? dims[1] : 0, rank > 2 ? dims[2] : 0}, rank, box_rows, 0};
  return cached_encode(map, key, [&](CUtensorMap* out) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3];
    cuuint64_t gstride[2];
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estride[3] = {1, 1, 1};
    uint64_t stride = 2;
    for (int i = 0; i < rank; ++i) {
      gdim[i] = dims[i];
      if (i > 0) gstride[i - 1] = stride;
      stride *= dims[i];
    }
    CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                    const_cast<void*>(base), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
  });
}

// fp32 tensor of rank 3 {cols, rows, planes} for bulk reduce-adds from shared
// memory: boxes of 32 columns (128 bytes) by 128 rows, 128-byte swizzle.
bool encode_f32_reduce(CUtensorMap* map, const void* base, const uint64_t* dims) {
  TmapKey key{base, {dims[0], dims[1], dims[2]}, 3, kBlockN, 2};
  return cached_encode(map, key, [&](CUtensorMap* out) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3] = {dims[0], dims[1], dims[2]};
    cuuint64_t gstride[2] = {dims[0] * 4, dims[0] * dims[1] * 4};
    cuuint32_t box[3] = {32, (cuuint32_t)kBlockN, 1};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3u, const_cast<void*>(base), gdim,
                    gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
  });
}

// Token-major packed tensor [total, H, d]: dims {d, H, total}, one head per
// box row group: box {64 columns, 1 head, 128 tokens}, the same shared-memory
// image as a 128-row box of the [B, H, L, d] layout.
bool encode_bf16_packed(CUtensorMap* map, const void* base, int d, int H, int total) {
  TmapKey key{base, {(uint64_t)d, (uint64_t)H, (uint64_t)total}, 3, kBlockN, 1};
  return cached_encode(map, key, [&](CUtensorMap* out) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)total};
    cuuint64_t gstride[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kBlockN};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3u, const_cast<void*>(base), gdim,
                    gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
  });
}

// SM count of the current device (148 when no device answers), queried once
// per device and thread.
int num_sms() {
  thread_local int cached[attn::kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= attn::kMaxDevices) return 148;
  if (cached[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return 148;
    cached[dev] = v;
  }
  return cached[dev];
}

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

// Device address of the kernels' error word, looked up once per device and
// context.
int* error_word_for_current_device() {
  static attn::PerContextOnce once;
  static int* cache[attn::kMaxDevices] = {};
  int* out = nullptr;
  const cudaError_t e = attn::once_per_context(once, [&](int dev) {
    cache[dev] = attn::device_error_word();
    return cache[dev] ? cudaSuccess : cudaErrorInvalidSymbol;
  });
  if (e != cudaSuccess) return nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(once.mu);
  out = cache[dev];
  return out;
}

struct SplitPlan {
  int nsplit;
  int chunk;
  int row_tiles;
};

// Returns false for invalid shape arguments.
bool plan_splits(int B, int Hq, int Hkv, int Lq, int Lk_max, int d, int num_splits,
                 SplitPlan* plan) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk_max < 1 || d < 1 || num_splits < 0) return false;
  if (Hq % Hkv) return false;
  const long long group = Hq / Hkv;
  const long long row_tiles = ceil_div(group * Lq, kBlockM);
  const long long max_splits = ceil_div(Lk_max, kBlockN);
  long long splits;
  if (num_splits > 0) {
    splits = num_splits < max_splits ? num_splits : max_splits;
  } else {
    // At least two waves of CTAs over the SMs, and chunks of at most 12288 keys
    // so that ragged per-sequence lengths balance across the grid.  Shorter
    // chunks cost more than they balance: each split CTA pays a fixed start
    // (Q load, pipeline fill) and end (epilogue, its partial rows written here
    // and read back by the combine, 512 bytes per query row and split).
    const long long units = (long long)B * Hkv * row_tiles;
    long long want = ceil_div(2LL * num_sms(), units);
    const long long by_len = ceil_div(Lk_max, 12288);
    if (by_len > want) want = by_len;
    splits = want < max_splits ? want : max_splits;
  }
  const long long chunk = ceil_div(ceil_div(Lk_max, splits), kBlockN) * kBlockN;
  plan->chunk = (int)chunk;
  plan->nsplit = (int)ceil_div(Lk_max, chunk);
  plan->row_tiles = (int)row_tiles;
  return true;
}

size_t ws_lse_offset(const SplitPlan& pl, long long nrows, int d) {
  const size_t obytes = (size_t)pl.nsplit * (size_t)nrows * (size_t)d * 4;
  return (obytes + 255) / 256 * 256;
}

}  // namespace

namespace {

// Short-query plan: taken when Lq <= 128, the row tiles of all (b, kv head)
// are fewer than twice the SM count, and the key range that any query row can
// see under the mask (before document ids; the lower and upper bounds of a
// row's interval never decrease with its position) spans at least 4 key tiles.
// The cluster of a row tile splits that range into `cluster` chunks of whole
// 128-key tiles, at most 8 CTAs per cluster and at least 8 tiles per CTA.
struct ShortPlan {
  int row_tiles, units, key_lo, chunk, cluster;
};

bool plan_short(int B, int Hq, int Hkv, int Lq, int Lk, int mask_kind, int wl, int wr, int bd,
                ShortPlan* sp) {
  if (Lq > kBlockM) return false;
  const long long group = Hq / Hkv;
  const long long row_tiles = ceil_div(group * Lq, kBlockM);
  const long long units = (long long)B * Hkv * row_tiles;
  const int sms = num_sms();
  if (units >= 2LL * sms || units > kMaxGridY) return false;
  // union of the rows' key intervals: positions Lk - Lq .. Lk - 1
  const long long p_lo = (long long)Lk - Lq, p_hi = (long long)Lk - 1;
  long long lo = 0, hi = (long long)Lk - 1;
  if (mask_kind == ATTN_MASK_CAUSAL) {
    hi = std::min(hi, p_hi);
  } else if (mask_kind == ATTN_MASK_DRAFT_BLOCK) {
    const long long blk = p_hi >= 0 ? p_hi / bd : -((-p_hi + bd - 1) / bd);
    hi = std::min(hi, (blk + 1) * bd - 1);
  }
  if (wl >= 0) lo = std::max(lo, p_lo - wl);
  if (wr >= 0) hi = std::min(hi, p_hi + wr);
  if (hi < lo) return false;  // no row sees a key: the persistent kernel writes the empty rows
  const long long t0 = lo / kBlockN, t1 = hi / kBlockN;
  const long long tiles = t1 - t0 + 1;
  // A few tiles per head are cheaper in the persistent kernel.  A cluster CTA
  // costs several microseconds of start-up and cold loads, so the key range is
  // split only into chunks of at least kMinTilesPerCta tiles.
  constexpr long long kMinTiles = 4, kMinTilesPerCta = 8;
  if (tiles < kMinTiles) return false;
  long long cluster = std::min<long long>(8, ceil_div(2LL * sms, units));
  cluster = std::max<long long>(1, std::min(cluster, tiles / kMinTilesPerCta));
  const long long per = ceil_div(tiles, cluster);
  cluster = ceil_div(tiles, per);
  sp->row_tiles = (int)row_tiles;
  sp->units = (int)units;
  sp->key_lo = (int)(t0 * kBlockN);
  sp->chunk = (int)(per * kBlockN);
  sp->cluster = (int)cluster;
  return true;
}

bool plan_short_possible(int B, int Hq, int Hkv, int Lq, int Lk, int mask_kind, int wl, int wr,
                         int draft_block) {
  ShortPlan sp;
  return plan_short(B, Hq, Hkv, Lq, Lk, mask_kind, wl, wr,
                    mask_kind == ATTN_MASK_DRAFT_BLOCK ? draft_block : 1, &sp);
}

}  // namespace

extern "C" {

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
  }
  return "ATTN_ERR_UNKNOWN";
}

// Score modifier of a call (ALiBi slopes or a relative-position table; at most one).
struct ScoreMod {
  const float* alibi_slopes = nullptr;
  const float* rel_table = nullptr;
  int rel_max = 0;
};

// Checks the score_mod arguments of the *_score_mod entry points.
static attn_status_t parse_score_mod(int kind, const float* params, int arg, ScoreMod* sm) {
  *sm = ScoreMod{};
  if (kind == ATTN_SCORE_MOD_NONE) return ATTN_OK;
  if (!params || !aligned(params, 4)) return ATTN_ERR_INVALID_ARG;
  if (kind == ATTN_SCORE_MOD_ALIBI) {
    sm->alibi_slopes = params;
    return ATTN_OK;
  }
  if (kind == ATTN_SCORE_MOD_REL_BIAS) {
    if (arg < 0 || arg > (1 << 20)) return ATTN_ERR_INVALID_ARG;
    sm->rel_table = params;
    sm->rel_max = arg;
    return ATTN_OK;
  }
  return ATTN_ERR_INVALID_ARG;
}

static attn_status_t validate_dense(const void* q, const void* k, const void* v, const void* o,
                                    const float* lse, int B, int Hq, int Hkv, int Lq, int Lk,
                                    int d, float scale, int mask_kind, int window_l, int window_r,
                                    int draft_block, const int32_t* doc_ids) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_DRAFT_BLOCK) return ATTN_ERR_INVALID_ARG;
  if (window_l < -1 || window_r < -1) return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_DRAFT_BLOCK && draft_block < 1) return ATTN_ERR_INVALID_ARG;
  if (doc_ids && (!aligned(doc_ids, 4) || Lq > Lk)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (ceil_div(Lk, kBlockN) > attn::kMaxKvTiles) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hq > kMaxGridY) return ATTN_ERR_UNSUPPORTED;
  const long long q_tiles = ceil_div(Lq, kBlockM);
  if ((long long)B * Hq * ((q_tiles + 1) / 2) > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

// allow_short = false keeps every shape on the persistent kernel (the chunks
// of attn_fwd_host then compute exactly what one attn_fwd call would).
static attn_status_t fwd_dense(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                               int mask_kind, int window_l, int window_r, int draft_block,
                               const int32_t* doc_ids, const ScoreMod& sm, void* stream,
                               bool allow_short = true) {
  const attn_status_t vs = validate_dense(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale,
                                          mask_kind, window_l, window_r, draft_block, doc_ids);
  if (vs != ATTN_OK) return vs;

  FwdParams p;
  std::memset(&p, 0, sizeof p);
  p.o = o;
  p.lse = lse;
  p.doc_ids = doc_ids;
  p.alibi_slopes = sm.alibi_slopes;
  p.rel_table = sm.rel_table;
  p.rel_max = sm.rel_max;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lk = Lk;
  p.group = Hq / Hkv;
  p.mask_kind = mask_kind;
  p.window_l = window_l;
  p.window_r = window_r;
  p.draft_block = mask_kind == ATTN_MASK_DRAFT_BLOCK ? draft_block : 1;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  p.q_tiles = (int)ceil_div(Lq, kBlockM);
  const long long n_units = (long long)B * Hq * ((p.q_tiles + 1) / 2);
  p.n_units = (int)n_units;
  p.err = error_word_for_current_device();
  if (!p.err) return ATTN_ERR_CUDA;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap tq, tk, tv;
  const uint64_t dk[3] = {(uint64_t)d, (uint64_t)Lk, (uint64_t)B * Hkv};
  if (!encode_bf16(&tk, k, 3, dk) || !encode_bf16(&tv, v, 3, dk)) return ATTN_ERR_CUDA;

  // Short queries: a query tile per (b, kv head) leaves most SMs idle in the
  // persistent kernel, so a cluster per row tile splits the visible keys.
  ShortPlan sp;
  if (allow_short && !sm.alibi_slopes && !sm.rel_table &&
      plan_short(B, Hq, Hkv, Lq, Lk, mask_kind, window_l, window_r, p.draft_block, &sp)) {
    p.row_tiles = sp.row_tiles;
    p.key_lo = sp.key_lo;
    p.chunk = sp.chunk;
    p.nsplit = sp.cluster;
    const uint64_t dq2[2] = {(uint64_t)d, (uint64_t)B * Hq * Lq};
    if (!encode_bf16(&tq, q, 2, dq2)) return ATTN_ERR_CUDA;
    cudaError_t e = d == 64 ? attn::launch_short<64>(tq, tk, tv, p, sp.units, st)
                            : attn::launch_short<128>(tq, tk, tv, p, sp.units, st);
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }

  const uint64_t dq[3] = {(uint64_t)d, (uint64_t)Lq, (uint64_t)B * Hq};
  if (!encode_bf16(&tq, q, 3, dq)) return ATTN_ERR_CUDA;
  const int grid = (int)(n_units < num_sms() ? n_units : num_sms());
  cudaError_t e = d == 64 ? attn::launch_prefill<64>(tq, tk, tv, p, grid, st)
                          : attn::launch_prefill<128>(tq, tk, tv, p, grid, st);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int Lq, int Lk, int d, float scale, int mask_kind,
                       int window_l, int window_r, int draft_block, const int32_t* doc_ids,
                       void* stream) {
  return fwd_dense(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, mask_kind, window_l, window_r,
                   draft_block, doc_ids, ScoreMod{}, stream);
}

attn_status_t attn_fwd_score_mod(const void* q, const void* k, const void* v, void* o,
                                 float* lse, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                                 float scale, int mask_kind, int window_l, int window_r,
                                 int draft_block, const int32_t* doc_ids, int score_mod,
                                 const float* score_mod_params, int score_mod_arg, void* stream) {
  ScoreMod sm;
  const attn_status_t st = parse_score_mod(score_mod, score_mod_params, score_mod_arg, &sm);
  if (st != ATTN_OK) return st;
  return fwd_dense(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, mask_kind, window_l, window_r,
                   draft_block, doc_ids, sm, stream);
}

// ------------------------------------------------- host buffers, pipelined
// attn_fwd_host: the inputs and outputs live in host memory.  The work is cut
// into chunks of whole (b, kv head) pairs (with their query heads); chunk c's
// Q, K and V go up on one copy stream while the kernel of chunk c - 1 runs on
// the caller's stream and the O / LSE of chunk c - 2 come down on another, so
// the PCIe transfers in both directions and the kernels overlap.
namespace {

constexpr int kHostChunks = 8;  // target chunk count (fewer when B * Hkv is smaller)

struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in[kHostChunks] = {}, out[kHostChunks] = {};
};
HostPipe g_pipe[attn::kMaxDevices];
attn::PerContextOnce g_pipe_once;
std::mutex g_pipe_enqueue;  // the events are reused: one enqueue at a time

struct HostLayout {
  size_t q, k, v, o, lse, doc, total;
};

HostLayout host_layout(int B, int Hq, int Hkv, int Lq, int Lk, int d, bool with_doc) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  HostLayout l;
  const size_t qb = (size_t)B * Hq * Lq * d * 2, kb = (size_t)B * Hkv * Lk * d * 2;
  l.q = 0;
  l.k = up(qb);
  l.v = l.k + up(kb);
  l.o = l.v + up(kb);
  l.lse = l.o + up(qb);
  l.doc = l.lse + up((size_t)B * Hq * Lq * 4);
  l.total = l.doc + (with_doc ? up((size_t)B * Lk * 4) : 0);
  return l;
}

// A chunk: batch elements [b0, b0 + nb) times kv heads [h0, h0 + nh).
struct HostChunk {
  int b0, nb, h0, nh;
};

int plan_host_chunks(int B, int Hkv, HostChunk* out) {
  int n = 0;
  if (B >= kHostChunks) {
    const int nb = (B + kHostChunks - 1) / kHostChunks;
    for (int b0 = 0; b0 < B; b0 += nb) out[n++] = {b0, std::min(nb, B - b0), 0, Hkv};
  } else {
    const int parts = std::min(Hkv, kHostChunks / B);
    const int nh = (Hkv + parts - 1) / parts;
    for (int b = 0; b < B; ++b)
      for (int h0 = 0; h0 < Hkv; h0 += nh) out[n++] = {b, 1, h0, std::min(nh, Hkv - h0)};
  }
  return n;
}

}  // namespace

size_t attn_fwd_host_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d,
                                    int with_doc_ids) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || d < 1 || Hq % Hkv != 0) return 0;
  return host_layout(B, Hq, Hkv, Lq, Lk, d, with_doc_ids != 0).total;
}

attn_status_t attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                            int mask_kind, int window_l, int window_r, int draft_block,
                            const int32_t* doc_ids, void* workspace, size_t ws_bytes,
                            void* stream) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || d < 1 || Hq % Hkv != 0)
    return ATTN_ERR_INVALID_ARG;
  const HostLayout lay = host_layout(B, Hq, Hkv, Lq, Lk, d, doc_ids != nullptr);
  if (!workspace || !aligned(workspace, 256) || ws_bytes < lay.total) return ATTN_ERR_WORKSPACE;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  uint8_t *qd = ws + lay.q, *kd = ws + lay.k, *vd = ws + lay.v, *od = ws + lay.o;
  float* ld = reinterpret_cast<float*>(ws + lay.lse);
  int32_t* dd = doc_ids ? reinterpret_cast<int32_t*>(ws + lay.doc) : nullptr;
  // the whole call's arguments, checked on the device-side copies before any work is queued
  const attn_status_t vs = validate_dense(qd, kd, vd, od, ld, B, Hq, Hkv, Lq, Lk, d, scale,
                                          mask_kind, window_l, window_r, draft_block, dd);
  if (vs != ATTN_OK) return vs;
  // chunks stay on the kernel one call over the whole shape would use, so the
  // results match attn_fwd exactly; short-query shapes run as one chunk
  const bool whole_short =
      plan_short_possible(B, Hq, Hkv, Lq, Lk, mask_kind, window_l, window_r, draft_block);
  HostChunk chunks[kHostChunks * 2];
  const int n_chunks = whole_short ? 1 : plan_host_chunks(B, Hkv, chunks);
  if (whole_short) chunks[0] = {0, B, 0, Hkv};

  const cudaError_t se = attn::once_per_context(g_pipe_once, [](int dev) {
    HostPipe& hp = g_pipe[dev];
    cudaError_t e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming);
    for (int i = 0; i < kHostChunks && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&hp.in[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.out[i], cudaEventDisableTiming);
    }
    return e;
  });
  if (se != cudaSuccess) return ATTN_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  HostPipe& hp = g_pipe[dev];
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int group = Hq / Hkv;
  const size_t qrow = (size_t)Lq * d * 2, krow = (size_t)Lk * d * 2;  // bytes per head

  std::lock_guard<std::mutex> lock(g_pipe_enqueue);
  bool ok = cudaEventRecord(hp.start, st) == cudaSuccess &&
            cudaStreamWaitEvent(hp.h2d, hp.start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(hp.d2h, hp.start, 0) == cudaSuccess;
  if (ok && doc_ids)
    ok = cudaMemcpyAsync(dd, doc_ids, (size_t)B * Lk * 4, cudaMemcpyHostToDevice, hp.h2d) ==
         cudaSuccess;
  for (int c = 0; c < n_chunks && ok; ++c) {
    const HostChunk& ch = chunks[c];
    const size_t qh0 = (size_t)ch.b0 * Hq + (size_t)ch.h0 * group;   // first query head
    const size_t kh0 = (size_t)ch.b0 * Hkv + (size_t)ch.h0;          // first kv head
    const size_t nq = (size_t)ch.nb * ch.nh * group, nk = (size_t)ch.nb * ch.nh;
    ok = cudaMemcpyAsync(qd + qh0 * qrow, static_cast<const uint8_t*>(q) + qh0 * qrow, nq * qrow,
                         cudaMemcpyHostToDevice, hp.h2d) == cudaSuccess &&
         cudaMemcpyAsync(kd + kh0 * krow, static_cast<const uint8_t*>(k) + kh0 * krow, nk * krow,
                         cudaMemcpyHostToDevice, hp.h2d) == cudaSuccess &&
         cudaMemcpyAsync(vd + kh0 * krow, static_cast<const uint8_t*>(v) + kh0 * krow, nk * krow,
                         cudaMemcpyHostToDevice, hp.h2d) == cudaSuccess &&
         cudaEventRecord(hp.in[c], hp.h2d) == cudaSuccess;
  }
  attn_status_t status = ok ? ATTN_OK : ATTN_ERR_CUDA;
  for (int c = 0; c < n_chunks && status == ATTN_OK; ++c) {
    const HostChunk& ch = chunks[c];
    const size_t qh0 = (size_t)ch.b0 * Hq + (size_t)ch.h0 * group;
    const size_t kh0 = (size_t)ch.b0 * Hkv + (size_t)ch.h0;
    const size_t nq = (size_t)ch.nb * ch.nh * group;
    if (cudaStreamWaitEvent(st, hp.in[c], 0) != cudaSuccess) {
      status = ATTN_ERR_CUDA;
      break;
    }
    status = fwd_dense(qd + qh0 * qrow, kd + kh0 * krow, vd + kh0 * krow, od + qh0 * qrow,
                       ld + qh0 * Lq, ch.nb, ch.nh * group, ch.nh, Lq, Lk, d, scale, mask_kind,
                       window_l, window_r, draft_block, dd ? dd + (size_t)ch.b0 * Lk : nullptr,
                       ScoreMod{}, stream, whole_short);
    if (status != ATTN_OK) break;
    if (cudaEventRecord(hp.out[c], st) != cudaSuccess ||
        cudaStreamWaitEvent(hp.d2h, hp.out[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(o) + qh0 * qrow, od + qh0 * qrow, nq * qrow,
                        cudaMemcpyDeviceToHost, hp.d2h) != cudaSuccess ||
        cudaMemcpyAsync(lse + qh0 * Lq, ld + qh0 * Lq, nq * Lq * 4, cudaMemcpyDeviceToHost,
                        hp.d2h) != cudaSuccess)
      status = ATTN_ERR_CUDA;
  }
  // the caller's stream resumes after the last download, whatever happened above
  if (cudaEventRecord(hp.done, hp.d2h) != cudaSuccess ||
      cudaStreamWaitEvent(st, hp.done, 0) != cudaSuccess)
    status = ATTN_ERR_CUDA;
  return status;
}

static attn_status_t fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                                int Hq, int Hkv, int total_q, int total_k, int max_seqlen_q, int d,
                                float scale, int mask_kind, int window_l, int window_r,
                                int draft_block, const ScoreMod& sm, void* stream) {
  if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (total_q < 1 || total_k < 1 || max_seqlen_q < 1 || max_seqlen_q > total_q)
    return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_DRAFT_BLOCK) return ATTN_ERR_INVALID_ARG;
  if (window_l < -1 || window_r < -1) return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_DRAFT_BLOCK && draft_block < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;

  FwdParams p;
  std::memset(&p, 0, sizeof p);
  p.o = o;
  p.lse = lse;
  p.cu_seqlens_q = cu_seqlens_q;
  p.cu_seqlens_k = cu_seqlens_k;
  p.alibi_slopes = sm.alibi_slopes;
  p.rel_table = sm.rel_table;
  p.rel_max = sm.rel_max;
  p.total_q = total_q;
  p.total_k = total_k;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = max_seqlen_q;  // sizes the units; each sequence's lengths come from cu_seqlens
  p.Lk = 0;
  p.group = Hq / Hkv;
  p.mask_kind = mask_kind;
  p.window_l = window_l;
  p.window_r = window_r;
  p.draft_block = mask_kind == ATTN_MASK_DRAFT_BLOCK ? draft_block : 1;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  p.q_tiles = (int)ceil_div(max_seqlen_q, kBlockM);
  const long long n_units = (long long)B * Hq * ((p.q_tiles + 1) / 2);
  if (n_units > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  p.n_units = (int)n_units;
  p.err = error_word_for_current_device();
  if (!p.err) return ATTN_ERR_CUDA;

  CUtensorMap tq, tk, tv;
  if (!encode_bf16_packed(&tq, q, d, Hq, total_q) || !encode_bf16_packed(&tk, k, d, Hkv, total_k) ||
      !encode_bf16_packed(&tv, v, d, Hkv, total_k))
    return ATTN_ERR_CUDA;

  const int grid = (int)(n_units < num_sms() ? n_units : num_sms());
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = d == 64 ? attn::launch_prefill<64>(tq, tk, tv, p, grid, st)
                          : attn::launch_prefill<128>(tq, tk, tv, p, grid, st);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                              int Hq, int Hkv, int total_q, int total_k, int max_seqlen_q, int d,
                              float scale, int mask_kind, int window_l, int window_r,
                              int draft_block, void* stream) {
  return fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv, total_q, total_k,
                    max_seqlen_q, d, scale, mask_kind, window_l, window_r, draft_block,
                    ScoreMod{}, stream);
}

attn_status_t attn_fwd_varlen_score_mod(const void* q, const void* k, const void* v, void* o,
                                        float* lse, const int32_t* cu_seqlens_q,
                                        const int32_t* cu_seqlens_k, int B, int Hq, int Hkv,
                                        int total_q, int total_k, int max_seqlen_q, int d,
                                        float scale, int mask_kind, int window_l, int window_r,
                                        int draft_block, int score_mod,
                                        const float* score_mod_params, int score_mod_arg,
                                        void* stream) {
  ScoreMod sm;
  const attn_status_t st = parse_score_mod(score_mod, score_mod_params, score_mod_arg, &sm);
  if (st != ATTN_OK) return st;
  return fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv, total_q, total_k,
                    max_seqlen_q, d, scale, mask_kind, window_l, window_r, draft_block, sm,
                    stream);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Lq, int d) {
  if (B < 1 || Hq < 1 || Lq < 1 || d < 1) return 0;
  const size_t rows = (size_t)B * (size_t)Hq * (size_t)Lq;
  const size_t acc = (rows * (size_t)d * 4 + 255) / 256 * 256;
  return acc + rows * 4;
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                       int Hq, int Hkv, int Lq, int Lk, int d, float scale, int mask_kind,
                       int window_l, int window_r, int draft_block, const int32_t* doc_ids,
                       void* workspace, size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || !aligned(workspace, 256))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_DRAFT_BLOCK) return ATTN_ERR_INVALID_ARG;
  if (window_l < -1 || window_r < -1) return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_DRAFT_BLOCK && draft_block < 1) return ATTN_ERR_INVALID_ARG;
  if (doc_ids && (!aligned(doc_ids, 4) || Lq > Lk)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (ceil_div(Lk, kBlockN) > kMaxGridY || (long long)B * Hkv > 0x7fffffffLL)
    return ATTN_ERR_UNSUPPORTED;
  const size_t need = attn_bwd_workspace_size(B, Hq, Lq, d);
  if (need == 0 || ws_bytes < need) return ATTN_ERR_WORKSPACE;

  attn::BwdParams p;
  std::memset(&p, 0, sizeof p);
  p.o = o;
  p.lse = lse;
  p.dout = dout;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  const size_t rows = (size_t)B * Hq * Lq;
  p.dq_acc = static_cast<float*>(workspace);
  p.dsum = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                    (rows * (size_t)d * 4 + 255) / 256 * 256);
  p.doc_ids = doc_ids;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lk = Lk;
  p.group = Hq / Hkv;
  p.mask_kind = mask_kind;
  p.window_l = window_l;
  p.window_r = window_r;
  p.draft_block = mask_kind == ATTN_MASK_DRAFT_BLOCK ? draft_block : 1;
  p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  p.q_tiles = (int)ceil_div(Lq, kBlockM);
  p.err = error_word_for_current_device();
  if (!p.err) return ATTN_ERR_CUDA;

  CUtensorMap tq, tk, tv, tdo, tdq;
  const uint64_t dq3[3] = {(uint64_t)d, (uint64_t)Lq, (uint64_t)B * Hq};
  const uint64_t dk3[3] = {(uint64_t)d, (uint64_t)Lk, (uint64_t)B * Hkv};
  if (!encode_bf16(&tq, q, 3, dq3) || !encode_bf16(&tk, k, 3, dk3) ||
      !encode_bf16(&tv, v, 3, dk3) || !encode_bf16(&tdo, dout, 3, dq3) ||
      !encode_f32_reduce(&tdq, p.dq_acc, dq3))
    return ATTN_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(p.dq_acc, 0, rows * (size_t)d * 4, st) != cudaSuccess) return ATTN_ERR_CUDA;
  cudaError_t e = d == 64 ? attn::launch_backward<64>(tq, tk, tv, tdo, tdq, p, st)
                          : attn::launch_backward<128>(tq, tk, tv, tdo, tdq, p, st);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_decode_num_splits(int B, int Hq, int Hkv, int Lq, int Lk_max, int d, int num_splits,
                           int* chunk_keys) {
  SplitPlan pl;
  if (!plan_splits(B, Hq, Hkv, Lq, Lk_max, d, num_splits, &pl)) return -1;
  if (chunk_keys) *chunk_keys = pl.chunk;
  return pl.nsplit;
}

size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk_max, int d,
                                  int num_splits) {
  SplitPlan pl;
  if (!plan_splits(B, Hq, Hkv, Lq, Lk_max, d, num_splits, &pl)) return 0;
  const long long nrows = (long long)B * Hq * Lq;
  return ws_lse_offset(pl, nrows, d) + (size_t)pl.nsplit * (size_t)nrows * 4;
}

}  // extern "C"

namespace {

struct PagedKv {
  const int32_t* block_table = nullptr;
  int page_size = 0;
  int pages_per_seq = 0;
  int num_pages = 0;
};

// Shared body of the contiguous and paged split-KV decode.
attn_status_t decode_impl(const void* q, const void* k_cache, const void* v_cache, void* o,
                          float* lse, const int32_t* kv_lens, int B, int Hq, int Hkv, int Lq,
                          int Lk_max, int d, float scale, int num_splits, void* workspace,
                          size_t ws_bytes, void* stream, const PagedKv& pg, const ScoreMod& sm) {
  if (!q || !k_cache || !v_cache || !o || !lse || !kv_lens) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(kv_lens, 4))
    return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  SplitPlan pl;
  if (!plan_splits(B, Hq, Hkv, Lq, Lk_max, d, num_splits, &pl)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (pl.chunk / kBlockN > attn::kMaxKvTiles) return ATTN_ERR_UNSUPPORTED;
  const long long nrows = (long long)B * Hq * Lq;
  if (nrows > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hkv * pl.row_tiles > kMaxGridY) return ATTN_ERR_UNSUPPORTED;
  const size_t need = attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk_max, d, num_splits);
  if (!workspace || !aligned(workspace, 256) || ws_bytes < need) return ATTN_ERR_WORKSPACE;

  FwdParams p;
  std::memset(&p, 0, sizeof p);
  p.o = o;
  p.lse = lse;
  p.ws_o = reinterpret_cast<float*>(workspace);
  p.ws_lse = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) +
                                      ws_lse_offset(pl, nrows, d));
  p.kv_lens = kv_lens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lk = Lk_max;
  p.group = Hq / Hkv;
  p.mask_kind = ATTN_MASK_NONE;
  p.window_l = -1;
  p.window_r = -1;
  p.draft_block = 1;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  p.chunk = pl.chunk;
  p.nsplit = pl.nsplit;
  p.row_tiles = pl.row_tiles;
  p.alibi_slopes = sm.alibi_slopes;
  p.rel_table = sm.rel_table;
  p.rel_max = sm.rel_max;
  p.block_table = pg.block_table;
  p.page_size = pg.page_size;
  p.pages_per_seq = pg.pages_per_seq;
  p.num_pages = pg.num_pages;

  CUtensorMap tq, tk, tv;
  const uint64_t dq[2] = {(uint64_t)d, (uint64_t)nrows};
  if (!encode_bf16(&tq, q, 2, dq)) return ATTN_ERR_CUDA;
  if (pg.block_table) {
    const uint64_t dk[3] = {(uint64_t)d, (uint64_t)pg.page_size,
                            (uint64_t)pg.num_pages * (uint64_t)Hkv};
    const int rows = pg.page_size < kBlockN ? pg.page_size : kBlockN;
    if (!encode_bf16(&tk, k_cache, 3, dk, rows) || !encode_bf16(&tv, v_cache, 3, dk, rows))
      return ATTN_ERR_CUDA;
  } else {
    const uint64_t dk[3] = {(uint64_t)d, (uint64_t)Lk_max, (uint64_t)B * Hkv};
    if (!encode_bf16(&tk, k_cache, 3, dk) || !encode_bf16(&tv, v_cache, 3, dk))
      return ATTN_ERR_CUDA;
  }

  dim3 grid((unsigned)pl.nsplit, (unsigned)(B * Hkv * pl.row_tiles), 1);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = d == 64 ? attn::launch_decode<64>(tq, tk, tv, p, grid, st)
                          : attn::launch_decode<128>(tq, tk, tv, p, grid, st);
  if (e != cudaSuccess) return ATTN_ERR_CUDA;
  e = d == 64 ? attn::launch_combine<64>(p, st) : attn::launch_combine<128>(p, st);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

attn_status_t attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                                  void* o, float* lse, const int32_t* kv_lens, int B, int Hq,
                                  int Hkv, int Lq, int Lk_max, int d, float scale, int num_splits,
                                  void* workspace, size_t ws_bytes, void* stream) {
  return decode_impl(q, k_cache, v_cache, o, lse, kv_lens, B, Hq, Hkv, Lq, Lk_max, d, scale,
                     num_splits, workspace, ws_bytes, stream, PagedKv{}, ScoreMod{});
}

attn_status_t attn_decode_splitkv_score_mod(const void* q, const void* k_cache,
                                            const void* v_cache, void* o, float* lse,
                                            const int32_t* kv_lens, int B, int Hq, int Hkv,
                                            int Lq, int Lk_max, int d, float scale,
                                            int num_splits, int score_mod,
                                            const float* score_mod_params, int score_mod_arg,
                                            void* workspace, size_t ws_bytes, void* stream) {
  ScoreMod sm;
  const attn_status_t st = parse_score_mod(score_mod, score_mod_params, score_mod_arg, &sm);
  if (st != ATTN_OK) return st;
  return decode_impl(q, k_cache, v_cache, o, lse, kv_lens, B, Hq, Hkv, Lq, Lk_max, d, scale,
                     num_splits, workspace, ws_bytes, stream, PagedKv{}, sm);
}

}  // extern "C"

namespace {

attn_status_t paged_impl(const void* q, const void* k_pages, const void* v_pages,
                         const int32_t* block_table, void* o, float* lse, const int32_t* kv_lens,
                         int B, int Hq, int Hkv, int Lq, int page_size, int pages_per_seq,
                         int num_pages, int d, float scale, int num_splits, void* workspace,
                         size_t ws_bytes, void* stream, const ScoreMod& sm) {
  if (!block_table || !aligned(block_table, 4)) return ATTN_ERR_INVALID_ARG;
  if (page_size < 16 || page_size > (1 << 16) || (page_size & (page_size - 1)) != 0)
    return ATTN_ERR_INVALID_ARG;
  if (pages_per_seq < 1 || num_pages < 1 || Hkv < 1) return ATTN_ERR_INVALID_ARG;
  const long long lk = (long long)pages_per_seq * page_size;
  if (lk > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if ((long long)num_pages * Hkv > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  PagedKv pg;
  pg.block_table = block_table;
  pg.page_size = page_size;
  pg.pages_per_seq = pages_per_seq;
  pg.num_pages = num_pages;
  return decode_impl(q, k_pages, v_pages, o, lse, kv_lens, B, Hq, Hkv, Lq, (int)lk, d, scale,
                     num_splits, workspace, ws_bytes, stream, pg, sm);
}

}  // namespace

extern "C" {

attn_status_t attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* block_table, void* o, float* lse,
                                const int32_t* kv_lens, int B, int Hq, int Hkv, int Lq,
                                int page_size, int pages_per_seq, int num_pages, int d,
                                float scale, int num_splits, void* workspace, size_t ws_bytes,
                                void* stream) {
  return paged_impl(q, k_pages, v_pages, block_table, o, lse, kv_lens, B, Hq, Hkv, Lq, page_size,
                    pages_per_seq, num_pages, d, scale, num_splits, workspace, ws_bytes, stream,
                    ScoreMod{});
}

attn_status_t attn_decode_paged_score_mod(const void* q, const void* k_pages, const void* v_pages,
                                          const int32_t* block_table, void* o, float* lse,
                                          const int32_t* kv_lens, int B, int Hq, int Hkv, int Lq,
                                          int page_size, int pages_per_seq, int num_pages, int d,
                                          float scale, int num_splits, int score_mod,
                                          const float* score_mod_params, int score_mod_arg,
                                          void* workspace, size_t ws_bytes, void* stream) {
  ScoreMod sm;
  const attn_status_t st = parse_score_mod(score_mod, score_mod_params, score_mod_arg, &sm);
  if (st != ATTN_OK) return st;
  return paged_impl(q, k_pages, v_pages, block_table, o, lse, kv_lens, B, Hq, Hkv, Lq, page_size,
                    pages_per_seq, num_pages, d, scale, num_splits, workspace, ws_bytes, stream,
                    sm);
}

attn_status_t attn_get_device_error(void* stream, int* raw_bits) {
  if (raw_bits) *raw_bits = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_ERR_CUDA;
  int* word = attn::device_error_word();
  if (!word) return ATTN_ERR_CUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, word, sizeof bits, cudaMemcpyDeviceToHost) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(word, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (raw_bits) *raw_bits = bits;
  if (bits & (attn::kDevErrTimeoutProducer | attn::kDevErrTimeoutMma |
              attn::kDevErrTimeoutSoftmax | attn::kDevErrTimeoutSelftest))
    return ATTN_ERR_TIMEOUT;
  if (bits & (attn::kDevErrBadKvLen | attn::kDevErrBadPage | attn::kDevErrBadSeqlens))
    return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

attn_status_t attn_selftest_wait_timeout(void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return attn::launch_selftest_wait(st) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"
