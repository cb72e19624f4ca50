// Split-KV decode for sm_100a (B200): the partial kernel and the combine.
// (The prefill forward is the persistent kernel in attn_prefill.cu.)
//
// Method ("FlashAttention 2 原理与 PyTorch 实战", sections 一, 3.1, 3.2): a CTA owns
// one 128-row query tile, streams 128-key K/V tiles through shared memory,
// computes S = Q K^T, applies the mask, keeps a running row max m and sum l
// (online softmax), rescales the accumulator and adds P V, so the N x N score
// matrix never reaches HBM.  The split-KV decode ("FlexAttention 是什么，以及
// DFlash2 之谜的完整侦破", section 1, FlexDecoding / FlashDecoding) gives each CTA
// one chunk of the KV cache of one sequence (every query row sees the keys
// [0, kv_lens[b]) of its sequence) and leaves a normalised partial output plus
// its log-sum-exp for the combine kernel at the end of this file.
//
// B200 mapping (one CTA per SM, 256 threads):
//   warp 0      TMA producer: Q once, then K and V tiles into a ring of stages
//               (128-byte swizzled boxes, mbarrier transaction counts).
//   warp 1      allocates tensor memory; lane 0 issues tcgen05.mma:
//               S_j = Q K_j^T (both operands in shared memory, fp32 in TMEM),
//               O  += P_j V_j (P from TMEM, V from shared memory, MN-major).
//   warps 2..5  softmax: thread r owns query row r (its TMEM lane), loads S_j,
//               masks partial tiles, adds the score modifier (ALiBi or a
//               relative-position table, compile-time variants), updates m and
//               l in base 2, rescales O only when the running max grew by more
//               than 2^8, writes P_j as bf16 over S_j in TMEM, and finally
//               stores O / l and the LSE.
//   warps 6, 7  extra TMA copy warps for pages shorter than a key tile.
// Tensor memory: S double buffer at columns [0,128) and [128,256), O at
// [256, 256 + d).  Key tiles that the mask empties entirely are never loaded.
// A paged cache whose pages are shorter than a key tile takes one TMA box per
// page and 64-column atom (16 per K tile for 16-key pages at d = 128); the
// boxes of a tile are then issued by three copy warps (warps 0, 6 and 7), as
// one issuing warp bounds the stream.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_params.h"
#include "host_once.h"
#include "ptx.cuh"
#include "softmax_row.cuh"

namespace attn {

__device__ int g_device_error = 0;

namespace {

// warps 0 (producer), 1 (MMA), 2..5 (softmax), 6..7 (extra copy warps for
// pages shorter than a key tile)
constexpr int kThreads = 256;
constexpr int kCopyWarps = 3;
constexpr int kTmemCols = 512;
static_assert(kBlockN == 128, "the softmax handles 128-key tiles");
constexpr uint32_t kTmemO = 256;
// S (and P over it) double buffer: columns [0,128) and [128,256).
__device__ __forceinline__ uint32_t tmem_s(int j) { return (j & 1) ? 128u : 0u; }
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when max grows by > 2^8
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct Cfg {
  static constexpr int kAtoms = D / 64;               // 128-byte swizzle atoms along d
  static constexpr int kAtomBytes = kBlockN * 128;    // one atom column of a 128-row tile
  static constexpr int kTileBytes = kBlockN * D * 2;  // one K or V tile (== Q tile)
  static constexpr int kStages = (D == 64) ? 4 : 3;  // d = 128: 3 x 64 KB of K/V, 226 KB in all
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2],
  // o_done, o_final, mma_drain
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffBits = kOffMisc + 64;
  static constexpr int kBitWords = kMaxKvTiles / 32;
  static constexpr int kSmemBytes = kOffBits + 2 * kBitWords * 4;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment
};

struct Misc {
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int t_lo;
  int t_hi;
};

__device__ __forceinline__ bool bit_get(const uint32_t* bits, int i) {
  return (bits[i >> 5] >> (i & 31)) & 1u;
}

template <int D>
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_saddr, int kk) {
  // K-major operand, 16 elements of d per MMA: atom kk/4, 32 bytes per step inside it.
  uint32_t addr = tile_saddr + (kk >> 2) * Cfg<D>::kAtomBytes + (kk & 3) * 32;
  return ptx::smem_desc_sw128(addr, 16, 1024);
}

template <int D>
__device__ __forceinline__ uint64_t desc_v_mnmajor(uint32_t tile_saddr, int kk) {
  // V as the MN-major B operand of P V: 16 keys (two 8-row groups) per MMA step,
  // 64-element d atoms 16 KB apart (leading offset), 8-key groups 1 KB apart (stride).
  uint32_t addr = tile_saddr + kk * 2048;
  return ptx::smem_desc_sw128(addr, Cfg<D>::kAtomBytes, 1024);
}

}  // namespace

// kMod: the score modifier (row::kModNone, kModAlibi or kModRelBias) with the
// query row's absolute position p = kv_lens[b] - Lq + i.
template <int D, int kMod>
__global__ void __launch_bounds__(kThreads, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::kStages;
  uint64_t* v_full = k_empty + C::kStages;
  uint64_t* v_empty = v_full + C::kStages;
  uint64_t* s_full = v_empty + C::kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* o_final = o_done + 1;
  uint64_t* mma_drain = o_final + 1;
  Misc* misc = reinterpret_cast<Misc*>(smem + C::kOffMisc);
  uint32_t* empty_bits = reinterpret_cast<uint32_t*>(smem + C::kOffBits);
  uint32_t* full_bits = empty_bits + C::kBitWords;
  volatile int* abort_flag = &misc->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ------------------------------------------------------------ work unit
  // (split, b, kv head, 128-row tile of the group's Hq/Hkv x Lq query rows)
  const int split = blockIdx.x;
  const int bh = blockIdx.y / p.row_tiles;
  const int rt = blockIdx.y % p.row_tiles;
  const int b = bh / p.Hkv;
  const int hkv = bh % p.Hkv;
  int kv_len = p.kv_lens[b];
  if (kv_len < 0 || kv_len > p.Lk) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && rt == 0) atomicOr(&g_device_error, kDevErrBadKvLen);
    kv_len = kv_len < 0 ? 0 : p.Lk;
  }
  const int c0 = split * p.chunk;
  const int rows_valid = min(kBlockM, p.group * p.Lq - rt * kBlockM);
  // flat output row of tile row 0
  const long long row_out0 =
      ((long long)b * p.Hq + (long long)hkv * p.group) * p.Lq + (long long)rt * kBlockM;
  if (c0 >= kv_len) {
    // This split holds no keys of sequence b: its rows get LSE = -inf, which
    // the combine reads as weight 0 (their O rows are never written or read).
    if ((int)threadIdx.x < rows_valid)
      p.ws_lse[(long long)split * p.B * p.Hq * p.Lq + row_out0 + threadIdx.x] = -INFINITY;
    return;  // uniform exit
  }
  const int key_end = min(c0 + p.chunk, kv_len);  // keys at or past this are never visible
  const int q_coord_y = (int)row_out0;
  const int kv_z = b * p.Hkv + hkv;
  const int t_lo = c0 / kBlockN;  // candidate key tiles (absolute tile indices)
  const int t_hi = (key_end - 1) / kBlockN;
  // pages shorter than a key tile: three copy warps share the TMA boxes of
  // every K/V tile (one box per page slice and atom; a single issuing warp
  // bounds the stream there)
  const bool small_pages = p.block_table != nullptr && p.page_size < kBlockN;
  const uint32_t kv_arrivals = small_pages ? kCopyWarps : 1u;

  // ------------------------------------------------------------- prologue
  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_q);
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_v);
      ptx::mbar_init(q_full, 1);
      for (int s = 0; s < C::kStages; ++s) {
        ptx::mbar_init(&k_full[s], kv_arrivals);
        ptx::mbar_init(&k_empty[s], 1);
        ptx::mbar_init(&v_full[s], kv_arrivals);
        ptx::mbar_init(&v_empty[s], 1);
      }
      for (int s = 0; s < 2; ++s) {
        ptx::mbar_init(&s_full[s], 1);
        ptx::mbar_init(&p_full[s], 4 * 32);
      }
      ptx::mbar_init(o_done, 1);
      ptx::mbar_init(o_final, 1);
      ptx::mbar_init(mma_drain, 1);
      misc->abort = 0;
      misc->t_lo = t_lo;
      misc->t_hi = t_hi;
      ptx::fence_mbar_init();
    }
    // Tile classification: FULL tiles lie below kv_len and need no mask.
    const int ntc = t_hi - t_lo + 1;
    int n_tiles = 0;
    for (int base = 0; base < ntc; base += 32) {
      const int i = base + lane;
      const long long k0 = (long long)(t_lo + i) * kBlockN;
      const bool empty = i >= ntc;
      const bool full = !empty && (k0 + kBlockN <= key_end);
      const uint32_t eb = __ballot_sync(0xffffffffu, empty);
      const uint32_t fb = __ballot_sync(0xffffffffu, full);
      if (lane == 0) {
        empty_bits[base >> 5] = eb;
        full_bits[base >> 5] = fb;
      }
      n_tiles += __popc(~eb);
    }
    if (lane == 0) misc->n_tiles = n_tiles;
  } else if (warp == 1) {
    ptx::tmem_alloc(&misc->tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  const int n_tiles = misc->n_tiles;

  if (warp == 0 || (warp >= 6 && small_pages)) {
    // ------------------------------------------------------------ producer
    // Copy warp cw (warp 0, and warps 6 and 7 when pages are shorter than a
    // key tile) issues its share of the TMA boxes of every K and V tile and
    // arrives once per tile on k_full / v_full with the bytes of its own
    // boxes; lane 0 of warp 0 also loads Q.
    const int cw = warp == 0 ? 0 : warp - 5;
    if (n_tiles > 0) {
      constexpr uint32_t kTx = C::kTileBytes;
      if (warp == 0 && lane == 0) {
        ptx::mbar_arrive_expect_tx(q_full, kTx);
        for (int a = 0; a < C::kAtoms; ++a)
          ptx::tma_load_2d(sQ + a * C::kAtomBytes, &tm_q, q_full, a * 64, q_coord_y);
      }
      // Contiguous cache: one box per 64-column atom.  Paged cache
      // ([num_pages, Hkv, page_size, d] through the block table): pages of 128
      // keys or more give one box per atom at the key's offset inside its
      // page; smaller pages give one box per page slice, each landing on a
      // whole number of 8-row swizzle atoms, so the assembled tile is laid out
      // exactly like a single box.  Keys past the block table read as zeros
      // (out-of-range coordinate), as do pages whose id is out of range (which
      // also flags the device error word).
      auto page_z = [&](int key) -> int {
        const int idx = key / p.page_size;
        if (idx >= p.pages_per_seq) return -1;
        const int page = __ldg(p.block_table + (long long)b * p.pages_per_seq + idx);
        if (page < 0 || page >= p.num_pages) {
          atomicOr(&g_device_error, kDevErrBadPage);
          return -1;
        }
        return page * p.Hkv + hkv;
      };
      // This warp's boxes of one K or V tile, with its own expect-tx.  Small
      // pages: lane i < `mine` loads item cw + kCopyWarps * i (page slice
      // item / atoms, atom item % atoms) from pool index pz (its page, fetched
      // one tile ahead).
      const int n_items = small_pages ? (kBlockN / p.page_size) * C::kAtoms : 0;
      const int mine = small_pages ? (n_items - cw + kCopyWarps - 1) / kCopyWarps : 0;
      const int item = cw + kCopyWarps * lane;
      auto item_page = [&](int t) -> int {
        if (!small_pages) return lane < C::kAtoms ? page_z(t * kBlockN) : -1;
        return lane < mine ? page_z(t * kBlockN + (item / C::kAtoms) * p.page_size) : -1;
      };
      // K/V tiles are read once: evict them from L2 first, so that the split
      // partials this launch writes stay there for the combine that reads them
      const uint64_t kv_policy = ptx::l2_policy_evict_first();
      auto load_kv = [&](uint8_t* dst, const CUtensorMap* tm, uint64_t* bar, int k0, int pz) {
        if (!small_pages) {
          if (lane == 0) ptx::mbar_arrive_expect_tx(bar, kTx);
          __syncwarp();
          if (lane < C::kAtoms) {
            const int y = p.block_table == nullptr ? k0 : k0 % p.page_size;
            const int z = p.block_table == nullptr ? kv_z : pz;
            ptx::tma_load_3d_hint(dst + lane * C::kAtomBytes, tm, bar, lane * 64, y, z,
                                  kv_policy);
          }
        } else {
          if (lane == 0) ptx::mbar_arrive_expect_tx(bar, (uint32_t)(mine * p.page_size * 128));
          __syncwarp();
          if (lane < mine) {
            const int sub = item / C::kAtoms, a = item % C::kAtoms;
            ptx::tma_load_3d_hint(dst + a * C::kAtomBytes + sub * p.page_size * 128, tm, bar,
                                  a * 64, 0, pz, kv_policy);
          }
        }
      };
      int j = 0;
      bool ok = true;
      const bool paged = p.block_table != nullptr;
      int pz_next = paged ? item_page(t_lo) : 0;
      for (int t = t_lo; t <= t_hi && ok; ++t) {
        if (bit_get(empty_bits, t - t_lo)) continue;
        const int s = j % C::kStages;
        const uint32_t ph = (uint32_t)(j / C::kStages) & 1u;
        const int k0 = t * kBlockN;
        const int pz = pz_next;
        ok = ptx::mbar_wait(&k_empty[s], ph ^ 1u, abort_flag, &g_device_error,
                            kDevErrTimeoutProducer);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        load_kv(sK + s * C::kTileBytes, &tm_k, &k_full[s], k0, pz);
        if (paged && t < t_hi) pz_next = item_page(t + 1);  // in flight during the wait
        ok = ptx::mbar_wait(&v_empty[s], ph ^ 1u, abort_flag, &g_device_error,
                            kDevErrTimeoutProducer);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          ++j;  // the K load of this tile is in flight; drain it below
          break;
        }
        load_kv(sV + s * C::kTileBytes, &tm_v, &v_full[s], k0, pz);
        ++j;
      }
      // Drain: every write into shared memory lands before the CTA exits (in a
      // normal run these phases have completed already).  The phases of
      // k_full / v_full cover every copy warp's loads.
      if (warp == 0 && lane == 0) {
        int dummy_abort = 0;
        ptx::mbar_wait(q_full, 0, &dummy_abort, nullptr, 0);
        for (int jj = max(0, j - C::kStages); jj < j; ++jj) {
          const int s = jj % C::kStages;
          const uint32_t ph = (uint32_t)(jj / C::kStages) & 1u;
          dummy_abort = 0;
          ptx::mbar_wait(&k_full[s], ph, &dummy_abort, nullptr, 0);
          dummy_abort = 0;
          ptx::mbar_wait(&v_full[s], ph, &dummy_abort, nullptr, 0);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
      constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kBlockM, D, 0, 1);
      const uint32_t q_saddr = ptx::smem_u32(sQ);
      const uint32_t k_saddr = ptx::smem_u32(sK);
      const uint32_t v_saddr = ptx::smem_u32(sV);
      bool ok = ptx::mbar_wait(q_full, 0, abort_flag, &g_device_error, kDevErrTimeoutMma);
      auto issue_s = [&](int j) -> bool {
        const int s = j % C::kStages;
        const uint32_t ph = (uint32_t)(j / C::kStages) & 1u;
        if (!ptx::mbar_wait(&k_full[s], ph, abort_flag, &g_device_error, kDevErrTimeoutMma))
          return false;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + tmem_s(j);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          ptx::mma_ss(d_tmem, desc_kmajor<D>(q_saddr, kk),
                      desc_kmajor<D>(k_saddr + s * C::kTileBytes, kk), kIdescS, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(&s_full[j & 1]);
        ptx::mma_commit(&k_empty[s]);
        return true;
      };
      if (ok) ptx::tc_fence_after();
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j + 1 < n_tiles) {
          ok = issue_s(j + 1);
          if (!ok) break;
        }
        const int s = j % C::kStages;
        ok = ptx::mbar_wait(&p_full[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, &g_device_error,
                            kDevErrTimeoutMma);
        if (!ok) break;
        ok = ptx::mbar_wait(&v_full[s], (uint32_t)(j / C::kStages) & 1u, abort_flag,
                            &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t p_tmem = tmem + tmem_s(j);
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          // P occupies 64 columns: two bf16 per 32-bit column, 16 keys per 8 columns.
          ptx::mma_ts(tmem + kTmemO, p_tmem + kk * 8,
                      desc_v_mnmajor<D>(v_saddr + s * C::kTileBytes, kk), kIdescPV,
                      (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(o_done);
        ptx::mma_commit(&v_empty[s]);
      }
      ptx::mma_commit(o_final);
      // Wait for every MMA to finish before tensor memory is released.
      ptx::mma_commit(mma_drain);
      int dummy_abort = 0;
      ptx::mbar_wait(mma_drain, 0, &dummy_abort, nullptr, 0);
    }
  } else if (warp >= 2 && warp < 6) {
    // ----------------------------------------------------------- softmax
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;      // tile row == TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool row_ok = r < rows_valid;
    const float c = p.scale_log2;

    // every query row of the sequence sees the keys [0, kv_len); rows past the
    // tile's valid rows see none
    const long long row_hi = row_ok ? (long long)key_end - 1 : -1;
    // score modifier: the row's query head and absolute position
    const int row_flat = rt * kBlockM + (row_ok ? r : 0);  // (head in group, query) of the tile row
    const int row_g = row_flat / p.Lq;
    const long long row_pos = (long long)kv_len - p.Lq + (row_flat - row_g * p.Lq);
    const int row_hq = hkv * p.group + row_g;
    const float alibi2 =
        kMod == row::kModAlibi ? __ldg(p.alibi_slopes + row_hq) * row::kLog2e : 0.0f;
    const float* rel_row = kMod == row::kModRelBias
                               ? p.rel_table + (long long)row_hq * (2 * p.rel_max + 1) + p.rel_max
                               : nullptr;
    const float c_s = kMod != row::kModNone ? 1.0f : c;  // scale still to apply to the scores

    float m_ref = -INFINITY;  // reference max (base-2 scaled units)
    float l = 0.0f;
    int j = 0;
    bool ok = true;
    for (int t = t_lo; t <= t_hi && ok; ++t) {
      if (bit_get(empty_bits, t - t_lo)) continue;
      const bool full = bit_get(full_bits, t - t_lo);
      const long long k0 = (long long)t * kBlockN;
      ok = ptx::mbar_wait(&s_full[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, &g_device_error,
                          kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);  // warp-collective TMEM access below
      if (!ok) break;
      ptx::tc_fence_after();

      float s[kBlockN];
      row::tmem_ld_row128(t_row + tmem_s(j), s);
      if (!full) {
        // visible keys of this row inside the tile: [0, hi_rel]
        const int hi_rel = (int)max(-1LL, min((long long)kBlockN - 1, row_hi - k0));
#pragma unroll
        for (int i = 0; i < kBlockN; ++i) s[i] = (i <= hi_rel) ? s[i] : -INFINITY;
      }
      if constexpr (kMod != row::kModNone)
        row::score_mod128<kMod>(s, c, (int)(k0 - row_pos), alibi2, rel_row, p.rel_max);
      const float m_tile = ptx::row_max128(s) * c_s;
      const float m_new = fmaxf(m_ref, m_tile);
      const bool need = m_new > m_ref + kRescaleThreshold;
      const float alpha = need ? ptx::ex2(m_ref - m_new) : 1.0f;  // 0 when m_ref = -inf
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds P_{<j} V; it must be final before it is rescaled.
        ok = ptx::mbar_wait(o_done, (uint32_t)(j - 1) & 1u, abort_flag, &g_device_error,
                            kDevErrTimeoutSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t raw[32];
          ptx::tmem_ld32(t_row + kTmemO + cc * 32, raw);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
          ptx::tmem_st32(t_row + kTmemO + cc * 32, raw);
        }
      }
      if (need) {
        l *= alpha;
        m_ref = m_new;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
      {
        // P over S: 64 columns of bf16 pairs
        uint32_t pk_lo[32], pk_hi[32];
        l += row::exp2_pack128(s, c_s, m_use, pk_lo, pk_hi);
        ptx::tmem_st32(t_row + tmem_s(j), pk_lo);
        ptx::tmem_st32(t_row + tmem_s(j) + 32, pk_hi);
      }
      {
        // Keys past the end of this sequence: their V rows may hold anything
        // (even NaN), and 0 * NaN would poison O.  Zero them in shared memory.
        if (!full) {
          const int s_stage = j % C::kStages;
          const bool zero_row = (k0 + r >= key_end);
          if (__any_sync(0xffffffffu, zero_row)) {
            ok = ptx::mbar_wait(&v_full[s_stage], (uint32_t)(j / C::kStages) & 1u, abort_flag,
                                &g_device_error, kDevErrTimeoutSoftmax);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (zero_row) {
#pragma unroll
              for (int a = 0; a < C::kAtoms; ++a) {
                uint4* row_ptr = reinterpret_cast<uint4*>(sV + s_stage * C::kTileBytes +
                                                          a * C::kAtomBytes + r * 128);
#pragma unroll
                for (int q = 0; q < 8; ++q) row_ptr[q] = make_uint4(0, 0, 0, 0);
              }
              ptx::fence_proxy_async_smem();
            }
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&p_full[j & 1]);
      ++j;
    }

    // ---------------------------------------------------------- epilogue
    ok = __all_sync(0xffffffffu, ok);
    if (ok && n_tiles > 0) {
      ok = ptx::mbar_wait(o_final, 0, abort_flag, &g_device_error, kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      ptx::tc_fence_after();
    }
    const bool have = ok && n_tiles > 0 && l > 0.0f;
    const float inv_l = have ? 1.0f / l : 0.0f;
    const float lse_row = have ? (m_ref + ptx::lg2(l)) * kLn2 : -INFINITY;
    const long long out_row = row_out0 + r;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t raw[32];
      if (ok && n_tiles > 0) {
        ptx::tmem_ld32(t_row + kTmemO + cc * 32, raw);
        ptx::tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) raw[i] = 0u;
      }
      if (row_ok) {
        float* dst = p.ws_o + ((long long)split * p.B * p.Hq * p.Lq + out_row) * D + cc * 32;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          float4 v4 = make_float4(__uint_as_float(raw[i]) * inv_l,
                                  __uint_as_float(raw[i + 1]) * inv_l,
                                  __uint_as_float(raw[i + 2]) * inv_l,
                                  __uint_as_float(raw[i + 3]) * inv_l);
          *reinterpret_cast<float4*>(dst + i) = v4;
        }
      }
    }
    if (row_ok) p.ws_lse[(long long)split * p.B * p.Hq * p.Lq + out_row] = lse_row;
  }

  // ------------------------------------------------------------- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Split-KV combine (the LSE-weighted merge of FlashDecoding-style partials):
//   LSE = log sum_s exp(LSE_s),  O = sum_s exp(LSE_s - LSE) O_s.
// One warp per output row; lane i owns d/32 consecutive elements.  The split
// LSEs are read one per lane (32 splits per load), and the partial rows of
// kUnroll splits are loaded together: a row costs two memory round trips (the
// LSEs, then the partial rows), not two per split.
template <int D>
__global__ void __launch_bounds__(256) attn_decode_combine_kernel(const FwdParams p) {
  constexpr int kPer = D / 32;
  constexpr int kUnroll = 8;
  constexpr float kLog2e = 1.44269504088896340736f;
  const long long nrows = (long long)p.B * p.Hq * p.Lq;
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= nrows) return;  // warp-uniform
  // every split wrote this row's LSE (-inf where it held no key of the sequence)
  const int ns = p.nsplit;
  float mx = -INFINITY;
  for (int s0 = 0; s0 < ns; s0 += 32) {
    if (s0 + lane < ns) mx = fmaxf(mx, p.ws_lse[(long long)(s0 + lane) * nrows + row]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.0f;
  float sum = 0.0f;
  if (mx != -INFINITY) {
    for (int s0 = 0; s0 < ns; s0 += 32) {
      // lane i: weight of split s0 + i (0 for a split with no visible key)
      const float ls = s0 + lane < ns ? p.ws_lse[(long long)(s0 + lane) * nrows + row] : -INFINITY;
      const float w_lane = ls == -INFINITY ? 0.0f : ptx::ex2((ls - mx) * kLog2e);
      sum += w_lane;
      const int n = min(32, ns - s0);
      for (int i0 = 0; i0 < n; i0 += kUnroll) {
        float wv[kUnroll];
        float v[kUnroll][kPer];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          wv[u] = __shfl_sync(0xffffffffu, w_lane, (i0 + u) & 31);
          const bool use = i0 + u < n && wv[u] != 0.0f;
          const float* src =
              p.ws_o + ((long long)(s0 + i0 + u) * nrows + row) * D + lane * kPer;
          if constexpr (kPer == 4) {
            const float4 t = use ? *reinterpret_cast<const float4*>(src)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            v[u][0] = t.x;
            v[u][1] = t.y;
            v[u][2] = t.z;
            v[u][3] = t.w;
          } else {
            const float2 t = use ? *reinterpret_cast<const float2*>(src) : make_float2(0.f, 0.f);
            v[u][0] = t.x;
            v[u][1] = t.y;
          }
          if (!use) wv[u] = 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
#pragma unroll
          for (int i = 0; i < kPer; ++i) acc[i] += wv[u] * v[u][i];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.o) + row * D + lane * kPer;
  if constexpr (kPer == 4) {
    uint2 o2;
    o2.x = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
    o2.y = ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = o2;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0) p.lse[row] = sum > 0.0f ? mx + ptx::lg2(sum) * kLn2 : -INFINITY;
}

// Failure-detection self-test: one thread waits, with the same bounded wait the
// attention kernels use, on an mbarrier that nothing ever arrives on.  The wait
// must give up after its budget, record kDevErrTimeoutSelftest and return, so
// the host sees ATTN_ERR_TIMEOUT and the context stays usable.
__global__ void attn_selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = ptx::mbar_wait_a(ptx::smem_u32(&bar), 0, &abort_flag, &g_device_error,
                                     kDevErrTimeoutSelftest);
    if (ok) atomicOr(&g_device_error, kDevErrBadKvLen);  // cannot happen: nobody arrives
  }
}

cudaError_t launch_selftest_wait(cudaStream_t stream) {
  attn_selftest_wait_kernel<<<1, 32, 0, stream>>>();
  return cudaGetLastError();
}

// ------------------------------------------------------------- launchers
template <int D, int kMod>
cudaError_t launch_decode_kernel(const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const FwdParams& p, dim3 grid,
                                 cudaStream_t stream) {
  auto kern = attn_decode_kernel<D, kMod>;
  constexpr int smem = Cfg<D>::kSmemAlloc;
  // The shared-memory opt-in is set once per device and context, normally by
  // a first call outside any stream capture that a later call may be part of.
  static PerContextOnce once;
  const cudaError_t e = once_per_context(once, [&](int) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const FwdParams& p, dim3 grid, cudaStream_t stream) {
  if (p.alibi_slopes)
    return launch_decode_kernel<D, row::kModAlibi>(tq, tk, tv, p, grid, stream);
  if (p.rel_table)
    return launch_decode_kernel<D, row::kModRelBias>(tq, tk, tv, p, grid, stream);
  return launch_decode_kernel<D, row::kModNone>(tq, tk, tv, p, grid, stream);
}

template <int D>
cudaError_t launch_combine(const FwdParams& p, cudaStream_t stream) {
  const long long nrows = (long long)p.B * p.Hq * p.Lq;
  const int warps = 8;
  const long long blocks = (nrows + warps - 1) / warps;
  attn_decode_combine_kernel<D><<<(unsigned)blocks, warps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

template cudaError_t launch_decode<64>(const CUtensorMap&, const CUtensorMap&,
                                        const CUtensorMap&, const FwdParams&, dim3, cudaStream_t);
template cudaError_t launch_decode<128>(const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const FwdParams&, dim3, cudaStream_t);
template cudaError_t launch_combine<64>(const FwdParams&, cudaStream_t);
template cudaError_t launch_combine<128>(const FwdParams&, cudaStream_t);

int* device_error_word() {
  int* ptr = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_device_error) != cudaSuccess)
    return nullptr;
  return ptr;
}

}  // namespace attn
