/*
 * attn.h — C ABI of the B200 (sm_100a) fused attention forward library.
 *
 * The library computes O = softmax(mask(Q K^T * scale)) V and the per-row
 * log-sum-exp with a fused, tiled kernel: each 128-row query tile streams
 * 128-key K/V tiles through shared memory and keeps a running max and sum
 * (online softmax), so the N x N score matrix never reaches device memory
 * ("FlashAttention 2 原理与 PyTorch 实战", sections 一, 3.1 and 3.2).  A split-KV
 * decode for short queries over a long cache, with GQA, and its LSE-weighted
 * combine follow FlexDecoding / FlashDecoding ("FlexAttention 是什么，以及
 * DFlash2 之谜的完整侦破", section 1).
 *
 * Conventions shared by every entry point
 *   - Element type: bf16 for Q, K, V and O (no dtype argument; the pages'
 *     kernels take bf16/fp16 only, "FlashAttention 2 原理与 PyTorch 实战",
 *     section 七).  LSE is fp32, natural log.
 *   - Layout: contiguous [B, H, L, D] (PyTorch's SDPA layout, same page,
 *     section 二), i.e. element (b, h, l, c) at ((b*H + h)*L + l)*D + c.
 *   - GQA: query head hq reads KV head hq / (Hq / Hkv).
 *   - All pointers are DEVICE pointers owned by the caller; the library keeps
 *     none of them after the call returns.  Q, K, V, O and the workspace must
 *     be 16-byte aligned; LSE, doc_ids and kv_lens 4-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     enqueue work and return; they never synchronise the device and never
 *     allocate device memory.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns a status and enqueues nothing.  A launch failure
 *     returns ATTN_ERR_CUDA.  Kernel-side problems (a bounded wait that ran
 *     out, a kv_lens entry out of range) are recorded in a device error word
 *     read by attn_get_device_error().
 *   - Inputs must be finite, except the decode cache past kv_lens[b], which
 *     may hold anything (it is never used, not even multiplied by zero).
 *   - The device error word is ONE word per device, shared by every stream,
 *     every host thread and every entry point of the library: a bit set by
 *     one caller's kernel is seen (and cleared) by whichever caller next
 *     calls attn_get_device_error on that device.
 *   - Per-device set-up (shared-memory opt-ins, symbol addresses) is done by
 *     a device's first call in each CUDA context, so the library stays usable
 *     after cudaDeviceReset; make that first call outside any stream capture.
 */
#ifndef ATTN_B200_ATTN_H_
#define ATTN_B200_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad shape or mask argument */
  ATTN_ERR_UNSUPPORTED = 2, /* valid request outside what is built (e.g. d not 64/128) */
  ATTN_ERR_WORKSPACE = 3,   /* decode workspace missing or too small */
  ATTN_ERR_CUDA = 4,        /* a CUDA runtime/driver call or launch failed */
  ATTN_ERR_TIMEOUT = 5      /* a kernel gave up on a bounded wait (device error word) */
} attn_status_t;

typedef enum {
  ATTN_MASK_NONE = 0,       /* bidirectional */
  ATTN_MASK_CAUSAL = 1,     /* key j visible iff j <= p */
  ATTN_MASK_DRAFT_BLOCK = 2 /* key j visible iff floor(j/Bd) <= floor(p/Bd) */
} attn_mask_kind_t;

/*
 * attn_fwd — prefill attention forward.
 *
 * Defines ("FlashAttention 2 原理与 PyTorch 实战", section 一; masks from
 * "FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", sections 1 and 3):
 *   for b < B, hq < Hq, query row i < Lq at absolute position p = Lk - Lq + i
 *   (bottom-right alignment), key j < Lk is visible iff
 *     base(p, j)                                     (per mask_kind above)
 *     and (window_l < 0 or j >= p - window_l)        (sliding window, inclusive;
 *     and (window_r < 0 or j <= p + window_r)         -1 = unbounded side)
 *     and (doc_ids == NULL or doc_ids[b][j] == doc_ids[b][p]).
 *   S_ij = scale * <Q[b,hq,i,:], K[b,hkv,j,:]> over visible j;
 *   O[b,hq,i,:] = sum_j softmax_j(S_ij) V[b,hkv,j,:];  LSE[b,hq,i] = log sum_j exp(S_ij).
 *   A row with no visible key gets O = 0 and LSE = -inf.
 *   The block-diffusion draft mask with the symmetric window (w, w) is
 *   mask_kind = ATTN_MASK_DRAFT_BLOCK, draft_block = Bd, window_l = window_r = w.
 *
 * Arguments
 *   q        [B, Hq, Lq, d] bf16, read
 *   k, v     [B, Hkv, Lk, d] bf16, read
 *   o        [B, Hq, Lq, d] bf16, written
 *   lse      [B, Hq, Lq] fp32, written
 *   B, Hq, Hkv, Lq, Lk >= 1, Hq % Hkv == 0; d in {64, 128} (else UNSUPPORTED);
 *   Lk <= 524288 (else UNSUPPORTED)
 *   scale    > 0 and finite (1/sqrt(d) is the usual choice)
 *   mask_kind  one of attn_mask_kind_t; window_l, window_r >= -1;
 *   draft_block >= 1 (read only for ATTN_MASK_DRAFT_BLOCK)
 *   doc_ids  [B, Lk] int32 or NULL; when given, Lq <= Lk is required
 *   stream   cudaStream_t
 * Errors: INVALID_ARG / UNSUPPORTED before any launch; CUDA on launch failure.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int Lq, int Lk, int d, float scale, int mask_kind,
                       int window_l, int window_r, int draft_block, const int32_t* doc_ids,
                       void* stream);

typedef enum {
  ATTN_SCORE_MOD_NONE = 0,    /* S_ij unchanged */
  ATTN_SCORE_MOD_ALIBI = 1,   /* S_ij += slope[hq] * (j - p); params = slope[Hq] */
  ATTN_SCORE_MOD_REL_BIAS = 2 /* S_ij += table[hq][clamp(j - p, -R, R) + R]; params = table,
                                 arg = R */
} attn_score_mod_kind_t;

/*
 * attn_fwd_score_mod — attn_fwd with a score modifier.
 *
 * Defines ("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 1:
 * score_mod(score, b, h, q_idx, kv_idx) -> score, with ALiBi, a position bias
 * and a learnable bias as examples): the scaled score S_ij of attn_fwd is
 * replaced by the modified score before the mask and the softmax; LSE is
 * taken over the modified scores.  p = Lk - Lq + i is the row's absolute
 * position.
 *   ATTN_SCORE_MOD_ALIBI: S_ij = scale * <Q_i, K_j> + slope[hq] * (j - p),
 *   with a caller-given per-query-head slope (for example 2^(-8 (hq+1) / Hq)).
 *   ATTN_SCORE_MOD_REL_BIAS: S_ij = scale * <Q_i, K_j> + table[hq][clamp(j - p,
 *   -R, R) + R]: a relative-position bias, one row of 2R + 1 values per query
 *   head (a learned table, a fixed position bias, or a per-head constant
 *   with R = 0); distances beyond R share the value at the end of the row.
 *
 * Arguments: those of attn_fwd, plus
 *   score_mod         one of attn_score_mod_kind_t
 *   score_mod_params  ALIBI: [Hq] fp32 device array; REL_BIAS: [Hq][2R + 1] fp32
 *                     device array; both 4-byte aligned; NONE: ignored
 *   score_mod_arg     REL_BIAS: R, 0 <= R <= 2^20; otherwise ignored
 * Errors: as attn_fwd; INVALID_ARG for an unknown score_mod, missing params or
 * a bad R.
 */
attn_status_t attn_fwd_score_mod(const void* q, const void* k, const void* v, void* o,
                                 float* lse, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                                 float scale, int mask_kind, int window_l, int window_r,
                                 int draft_block, const int32_t* doc_ids, int score_mod,
                                 const float* score_mod_params, int score_mod_arg, void* stream);

/*
 * attn_fwd_varlen — prefill attention forward over packed sequences.
 *
 * The B sequences are packed one after another along the token axis with no
 * padding ("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 1: a
 * document mask at the packing level; ragged lengths without padding).
 * Sequence b owns query tokens [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key
 * tokens [cu_seqlens_k[b], cu_seqlens_k[b+1]); with Lq_b and Lk_b its lengths,
 * its rows follow attn_fwd above with Lq = Lq_b, Lk = Lk_b (bottom-right
 * alignment, the same mask kinds and window) and no document ids: a token
 * never sees another sequence's keys.
 *
 * Arguments
 *   q        [total_q, Hq, d] bf16, read (token-major, heads interleaved)
 *   k, v     [total_k, Hkv, d] bf16, read
 *   o        [total_q, Hq, d] bf16, written (rows of every sequence)
 *   lse      [Hq, total_q] fp32, written
 *   cu_seqlens_q, cu_seqlens_k  [B + 1] int32 in device memory, non-decreasing,
 *            starting at 0 and ending at total_q / total_k
 *   max_seqlen_q >= every Lq_b (sizes the grid); every Lk_b <= 524288
 *   B, Hq, Hkv, total_q, total_k >= 1; d, scale, mask_kind, window_l,
 *   window_r, draft_block as for attn_fwd
 *   stream   cudaStream_t
 * Errors: INVALID_ARG / UNSUPPORTED before any launch; CUDA on launch failure.
 * cu_seqlens live in device memory, so the kernel checks them: a sequence whose
 * bounds are out of order or out of range, or longer than max_seqlen_q, is
 * skipped and flagged in the device error word (attn_get_device_error then
 * returns ATTN_ERR_INVALID_ARG).
 */
attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                              int Hq, int Hkv, int total_q, int total_k, int max_seqlen_q, int d,
                              float scale, int mask_kind, int window_l, int window_r,
                              int draft_block, void* stream);

/*
 * attn_fwd_varlen_score_mod — attn_fwd_varlen with a score modifier, as in
 * attn_fwd_score_mod: p is the row's absolute position inside its own
 * sequence (Lk_b - Lq_b + i).  Arguments: those of attn_fwd_varlen, plus
 * score_mod, score_mod_params and score_mod_arg as for attn_fwd_score_mod.
 */
attn_status_t attn_fwd_varlen_score_mod(const void* q, const void* k, const void* v, void* o,
                                        float* lse, const int32_t* cu_seqlens_q,
                                        const int32_t* cu_seqlens_k, int B, int Hq, int Hkv,
                                        int total_q, int total_k, int max_seqlen_q, int d,
                                        float scale, int mask_kind, int window_l, int window_r,
                                        int draft_block, int score_mod,
                                        const float* score_mod_params, int score_mod_arg,
                                        void* stream);

/*
 * attn_fwd_host — attn_fwd on tensors that live in host memory: the same
 * operation and layouts, with q, k, v, doc_ids (nullable) read from host
 * buffers and o, lse written to host buffers.
 *
 * The call copies the inputs into `workspace` (device memory, owned by the
 * caller, at least attn_fwd_host_workspace_size bytes, 256-byte aligned), runs
 * the forward and copies O and the LSE back, all queued on `stream`: read the
 * outputs after synchronising it.  The work is cut into chunks of whole
 * (batch, kv head) pairs, and chunk c's uploads, chunk c - 1's kernel and
 * chunk c - 2's downloads run at the same time (two internal copy streams per
 * device and context, joined to `stream` by events).  Page-locked (pinned)
 * host buffers are needed for the copies to overlap; pageable ones work but
 * serialise.  The chunks use the kernel a single attn_fwd call on the whole
 * shape would use, so O and LSE are the same bits as attn_fwd's.
 *
 * Errors: as attn_fwd (checked before anything is queued); WORKSPACE for a
 * missing, misaligned or too small workspace.  Enqueueing is serialised across
 * host threads (the internal events are shared).
 */
size_t attn_fwd_host_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d,
                                    int with_doc_ids);
attn_status_t attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                            int mask_kind, int window_l, int window_r, int draft_block,
                            const int32_t* doc_ids, void* workspace, size_t ws_bytes,
                            void* stream);

/*
 * attn_bwd_workspace_size — bytes of caller workspace attn_bwd needs:
 * an fp32 dQ accumulator [B, Hq, Lq, d] (rounded up to 256 bytes), then fp32
 * D [B, Hq, Lq].  0 for invalid arguments.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int Lq, int d);

/*
 * attn_bwd — gradients of attn_fwd: dQ, dK, dV for a given dO.
 *
 * Defines (the gradient of the definition above; "FlashAttention 2 原理与
 * PyTorch 实战", section 3.2: the scores are recomputed from Q, K and the
 * forward's LSE rather than stored): with P_ij = exp(S_ij - LSE_i) over the
 * visible keys (0 elsewhere and for rows with no visible key),
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P (dP - D),
 *   dQ = scale dS K,  dK = scale dS^T Q,
 * with the dK and dV of a KV head summed over its query heads (GQA).
 *
 * Arguments
 *   q, o, dout  [B, Hq, Lq, d] bf16, read (o and lse from attn_fwd)
 *   lse      [B, Hq, Lq] fp32, read
 *   k, v     [B, Hkv, Lk, d] bf16, read
 *   dq       [B, Hq, Lq, d] bf16, written;  dk, dv  [B, Hkv, Lk, d] bf16, written
 *   B, Hq, Hkv, Lq, Lk, scale, mask_kind, window_l, window_r, draft_block,
 *   doc_ids  as for attn_fwd; d in {64, 128} (else UNSUPPORTED)
 *   workspace  device memory, 256-byte aligned, >= attn_bwd_workspace_size bytes,
 *            owned by the caller, not shared with a concurrent call
 *   stream   cudaStream_t; the call enqueues a memset and three kernels
 * Determinism: dK and dV are bit-identical from run to run; dQ is not, since
 * its fp32 accumulator receives one atomic add per (key tile, query tile)
 * pair in whatever order the CTAs run (differences are rounding-level).
 * Errors: INVALID_ARG / UNSUPPORTED / WORKSPACE before any launch; CUDA on
 * launch failure.
 */
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                       int Hq, int Hkv, int Lq, int Lk, int d, float scale, int mask_kind,
                       int window_l, int window_r, int draft_block, const int32_t* doc_ids,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_decode_num_splits — how many KV splits attn_decode_splitkv uses.
 *
 * The keys [0, Lk_max) are cut into nsplit chunks of `chunk` keys each, a
 * whole number of 128-key tiles; split s covers [s*chunk, (s+1)*chunk) and
 * sequence b uses the first ceil(kv_lens[b] / chunk) splits.  num_splits > 0
 * asks for that many chunks (capped at ceil(Lk_max / 128)); 0 lets the
 * library choose from B * Hkv, Lk_max and the device's SM count.
 * Returns the split count (>= 1) and stores the chunk length in *chunk_keys
 * (nullable); returns -1 for invalid arguments.
 */
int attn_decode_num_splits(int B, int Hq, int Hkv, int Lq, int Lk_max, int d, int num_splits,
                           int* chunk_keys);

/*
 * attn_decode_workspace_size — bytes of caller-owned device workspace that
 * attn_decode_splitkv needs for the same arguments; 0 for invalid arguments.
 *
 * Workspace layout (documented so tests can read the partial results):
 *   offset 0:           fp32 O_s  [nsplit, B*Hq*Lq, d]   (normalised per split)
 *   offset ws_lse_off:  fp32 LSE_s [nsplit, B*Hq*Lq]
 *   where ws_lse_off = round_up(nsplit*B*Hq*Lq*d*4, 256).
 *   Splits that hold no key of their sequence write LSE_s = -inf for their
 *   rows and leave O_s unwritten; the combine gives them weight 0.
 */
size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk_max, int d,
                                  int num_splits);

/*
 * attn_decode_splitkv — split-KV decode attention (non-causal over the cache).
 *
 * Defines: for each b, query head hq and query row i < Lq, the keys visible
 * are exactly [0, kv_lens[b]) of the cache; O and LSE as in attn_fwd with no
 * mask.  Computed in two launches on `stream` ("FlexAttention 是什么，以及
 * DFlash2 之谜的完整侦破", section 1: a short query over a long KV is split
 * across CTAs, then merged): (1) per (b, kv head, split) a partial O_s and
 * LSE_s over that chunk, for all Hq/Hkv query heads of the group at once;
 * (2) the combine LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.
 *
 * Arguments
 *   q        [B, Hq, Lq, d] bf16, read
 *   k_cache, v_cache  [B, Hkv, Lk_max, d] bf16, read only below kv_lens[b]
 *   o        [B, Hq, Lq, d] bf16, written;  lse [B, Hq, Lq] fp32, written
 *   kv_lens  [B] int32 DEVICE array, each in [1, Lk_max]; an entry outside
 *            [0, Lk_max] is clamped and flags the device error word
 *   d in {64, 128}; scale > 0; num_splits as in attn_decode_num_splits
 *   workspace, ws_bytes  caller-owned device buffer of at least
 *            attn_decode_workspace_size(...) bytes (else ATTN_ERR_WORKSPACE)
 * Errors: INVALID_ARG / UNSUPPORTED / WORKSPACE before any launch; CUDA on
 * launch failure.
 */
attn_status_t attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                                  void* o, float* lse, const int32_t* kv_lens, int B, int Hq,
                                  int Hkv, int Lq, int Lk_max, int d, float scale, int num_splits,
                                  void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_decode_splitkv_score_mod — attn_decode_splitkv with a score modifier, as
 * in attn_fwd_score_mod ("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破",
 * section 1: score_mod(score, b, h, q_idx, kv_idx)).  Query row i of sequence b
 * sits at absolute position p = kv_lens[b] - Lq + i (the Lq queries are the
 * last Lq positions of the sequence, the alignment the masks of attn_fwd use):
 *   ATTN_SCORE_MOD_ALIBI:    S_ij = scale * <Q_i, K_j> + slope[hq] * (j - p)
 *   ATTN_SCORE_MOD_REL_BIAS: S_ij = scale * <Q_i, K_j> + table[hq][clamp(j - p,
 *                            -R, R) + R]
 * score_mod, score_mod_params and score_mod_arg as for attn_fwd_score_mod
 * (slopes [Hq] or table [Hq][2R + 1], fp32 device arrays, read only); the
 * other arguments, the workspace and the errors as attn_decode_splitkv, plus
 * INVALID_ARG for an unknown score_mod, missing params or R outside [0, 2^20].
 */
attn_status_t attn_decode_splitkv_score_mod(const void* q, const void* k_cache,
                                            const void* v_cache, void* o, float* lse,
                                            const int32_t* kv_lens, int B, int Hq, int Hkv,
                                            int Lq, int Lk_max, int d, float scale,
                                            int num_splits, int score_mod,
                                            const float* score_mod_params, int score_mod_arg,
                                            void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_decode_paged — the split-KV decode of attn_decode_splitkv over a paged
 * KV cache (the paged block_table call of "FlexAttention 是什么，以及 DFlash2 之谜
 * 的完整侦破", section 4, experiment 1; PagedAttention through a logical-to-
 * physical page table, section 1).
 *
 * Defines: sequence b's logical key j lives in page block_table[b][j / page_size]
 * at row j % page_size; the visible keys are [0, kv_lens[b]); O and LSE as in
 * attn_decode_splitkv.  Equals attn_decode_splitkv on the cache gathered
 * through the block table.
 *
 * Arguments
 *   q                 [B, Hq, Lq, d] bf16
 *   k_pages, v_pages  [num_pages, Hkv, page_size, d] bf16 page pool, read
 *   block_table       [B, pages_per_seq] int32 DEVICE array of page ids in
 *                     [0, num_pages); entries past a sequence's last page are
 *                     never read; an out-of-range id reads as zeros and flags
 *                     the device error word (ATTN_ERR_INVALID_ARG)
 *   o, lse, kv_lens   as attn_decode_splitkv, with Lk_max = pages_per_seq * page_size
 *   page_size         power of two, 16 <= page_size <= 65536
 *   num_splits, workspace, ws_bytes  as attn_decode_splitkv with that Lk_max
 *                     (attn_decode_workspace_size(B, Hq, Hkv, Lq,
 *                      pages_per_seq * page_size, d, num_splits) bytes)
 * Errors: as attn_decode_splitkv; INVALID_ARG also for a null or misaligned
 * block_table or a bad page_size / pages_per_seq / num_pages.
 */
attn_status_t attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* block_table, void* o, float* lse,
                                const int32_t* kv_lens, int B, int Hq, int Hkv, int Lq,
                                int page_size, int pages_per_seq, int num_pages, int d,
                                float scale, int num_splits, void* workspace, size_t ws_bytes,
                                void* stream);

/*
 * attn_decode_paged_score_mod — attn_decode_paged with a score modifier, with
 * the positions and arguments of attn_decode_splitkv_score_mod.
 */
attn_status_t attn_decode_paged_score_mod(const void* q, const void* k_pages, const void* v_pages,
                                          const int32_t* block_table, void* o, float* lse,
                                          const int32_t* kv_lens, int B, int Hq, int Hkv, int Lq,
                                          int page_size, int pages_per_seq, int num_pages, int d,
                                          float scale, int num_splits, int score_mod,
                                          const float* score_mod_params, int score_mod_arg,
                                          void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_decode_splitkv_noalloc — attn_decode_splitkv for callers that cannot
 * allocate device memory.  (No counterpart on the pages: this is a library
 * convenience, not part of the method.)
 *
 * Some callers cannot call cudaMalloc or any other allocator: for example a
 * plugin inside a serving process whose device memory is all handed out by
 * the host application's own pool, or a latency-critical decode loop where an
 * allocation (which may synchronise the device) is not allowed.  They still
 * own and pass q, k_cache, v_cache, o, lse and kv_lens, with the meaning,
 * layout and rules of attn_decode_splitkv; the split workspace comes from a
 * fixed 32 MiB array in device memory that the library declares itself.
 *   - Every GPU that loads the library holds that array until the process
 *     exits.
 *   - The first call on a device looks up the array's device address (with
 *     that device current, and again in a new context after
 *     cudaDeviceReset); make this first call before any stream capture.
 *   - Requests whose attn_decode_workspace_size(...) exceeds 32 MiB return
 *     ATTN_ERR_WORKSPACE and launch nothing (e.g. B=64, Hq=64, Lq=1,
 *     Lk_max=32768, d=128 needs 16.9 MB and fits; the Lq=16 variant does not).
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero (every value the combine reads is
 *     written first by the same call), but two calls that overlap on the GPU
 *     (different streams, or different host threads) race on it: serialise
 *     them.
 * Errors: as attn_decode_splitkv, plus ATTN_ERR_WORKSPACE above.
 */
attn_status_t attn_decode_splitkv_noalloc(const void* q, const void* k_cache,
                                          const void* v_cache, void* o, float* lse,
                                          const int32_t* kv_lens, int B, int Hq, int Hkv, int Lq,
                                          int Lk_max, int d, float scale, int num_splits,
                                          void* stream);

/*
 * attn_get_device_error — synchronise `stream`, then read and clear the
 * device error word of the current device (shared by all callers; see the
 * conventions above).  Returns ATTN_OK, ATTN_ERR_TIMEOUT
 * (a kernel abandoned a bounded wait), ATTN_ERR_INVALID_ARG (a kv_lens entry
 * or a block_table page id was out of range) or ATTN_ERR_CUDA (the
 * synchronisation itself failed).
 * `raw_bits` (nullable) receives the raw error bits.
 */
attn_status_t attn_get_device_error(void* stream, int* raw_bits);

/*
 * attn_selftest_wait_timeout — diagnostic for the failure-detection path (no
 * counterpart on the pages).  Enqueues on `stream` a one-block kernel whose
 * single bounded wait targets an mbarrier that nothing arrives on: the wait
 * gives up after its budget (about one second), records the self-test timeout
 * bit in the device error word and returns.  A following
 * attn_get_device_error() returns ATTN_ERR_TIMEOUT and clears the word; the
 * CUDA context stays usable.  Returns ATTN_ERR_CUDA if the launch fails.
 */
attn_status_t attn_selftest_wait_timeout(void* stream);

/* Static, human-readable name of a status code. */
const char* attn_status_string(attn_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_ATTN_H_ */
