// Launch parameters shared by the host planner (attn_api.cu) and the kernels
// (attn_kernels.cu).  Plain data only.
#pragma once

#include <cstdint>

namespace attn {

constexpr int kBlockM = 128;     // query rows per tile (tcgen05 M)
constexpr int kBlockN = 128;     // keys per tile (N of S = QK^T, K of O += PV)
constexpr int kMaxKvTiles = 4096;  // key tiles one work unit may span (Lk <= 512K)

enum MaskKind : int { kMaskNone = 0, kMaskCausal = 1, kMaskDraftBlock = 2 };

// Error bits the kernels OR into the device error word.
enum DeviceError : int {
  kDevErrTimeoutProducer = 1 << 0,
  kDevErrTimeoutMma = 1 << 1,
  kDevErrTimeoutSoftmax = 1 << 2,
  kDevErrBadKvLen = 1 << 3,
  kDevErrTimeoutSelftest = 1 << 4,
  kDevErrBadPage = 1 << 5,
  kDevErrBadSeqlens = 1 << 6,
};

struct FwdParams {
  // outputs
  void* o;          // prefill: bf16 [B, Hq, Lq, d]; decode: unused
  float* lse;       // prefill: fp32 [B, Hq, Lq]; decode: unused
  float* ws_o;      // decode: fp32 [nsplit, B*Hq*Lq, d] normalised partial outputs
  float* ws_lse;    // decode: fp32 [nsplit, B*Hq*Lq] partial log-sum-exp
  // optional inputs
  const int32_t* doc_ids;  // [B, Lk] or null
  const int32_t* kv_lens;  // decode: [B]
  // shapes
  int B, Hq, Hkv, Lq, Lk;  // decode: Lk = Lk_max
  int group;               // Hq / Hkv
  // mask (prefill)
  int mask_kind, window_l, window_r, draft_block;
  float scale_log2;  // softmax scale * log2(e)
  // decode split plan
  int chunk;         // keys per split (multiple of kBlockN)
  int nsplit;        // splits covering Lk_max
  int row_tiles;     // 128-row tiles per (b, kv head): ceil(group * Lq / 128)
  int q_tiles;       // prefill: ceil(Lq / 128)
  int n_units;       // prefill: work units (pairs of query tiles x B*Hq)
  int* err;          // device error word
  // score_mod (prefill): ALiBi slopes [Hq] fp32, or null; or a relative-position
  // table [Hq][2 rel_max + 1] fp32, or null
  const float* alibi_slopes;
  const float* rel_table;
  int rel_max;
  // packed sequences (prefill): null for the [B, H, L, d] layout
  const int32_t* cu_seqlens_q;  // [B + 1]
  const int32_t* cu_seqlens_k;  // [B + 1]
  int total_q, total_k;         // tokens in the packed Q and K/V tensors
  // paged KV cache (decode): K/V pages [num_pages, Hkv, page_size, d]
  const int32_t* block_table;  // [B, pages_per_seq] page ids, or null (contiguous cache)
  int page_size;               // keys per page (power of two, >= 16)
  int pages_per_seq;           // row length of block_table; Lk = pages_per_seq * page_size
  int num_pages;               // pages in the pool
  // short-query prefill (one cluster per row tile splits the visible keys)
  int key_lo;                  // first key of the cluster's range (multiple of kBlockN)
};

}  // namespace attn
