// Device helpers shared by the prefill kernels (the persistent kernel in
// attn_prefill.cu and the short-query kernel in attn_short.cu): the work-unit
// numbering, the per-row visible key interval of the mask predicate, the
// document ranges of rows and key tiles, and the per-unit tile schedule
// (EMPTY / PARTIAL / FULL per key tile and query tile).
//
// Masks: the mask_mod predicate of "FlexAttention 是什么，以及 DFlash2 之谜的完整
// 侦破" (section 1: causal, sliding window, non-causal, document ids; section 3:
// symmetric window, block-diffusion draft mask).  Every mask kind gives each
// query row one contiguous key interval [lo, hi]; document ids then keep the
// keys of the row's own document.
#pragma once

#include <cstdint>

#include "attn_params.h"

namespace attn {
namespace prefill {

// A work unit: two adjacent 128-row query tiles (A and B) of one (batch, head).
struct Unit {
  int b, hq, hkv, bh;
  int q0[2];          // first query row of tile A / B (within its sequence)
  int rows[2];        // valid rows of tile A / B (0 if the tile is past Lq)
  long long pos0[2];  // absolute position of row 0 of tile A / B
  int Lk;             // keys of the sequence
  int q_base, k_base; // packed sequences: first token of the sequence in Q and in K/V
  bool bad;           // packed sequences: out-of-range cu_seqlens (the unit is skipped)
};

__device__ __forceinline__ long long floor_div_ll(long long a, long long b) {
  return a >= 0 ? a / b : -((-a + b - 1) / b);
}

// Visible key interval [lo, hi] of the row at absolute position pos (before
// document ids), clamped above to Lk - 1.
__device__ __forceinline__ void key_bounds(const FwdParams& p, int Lk, long long pos,
                                           long long& lo, long long& hi) {
  lo = 0;
  hi = (long long)Lk - 1;
  if (p.mask_kind == kMaskCausal) {
    hi = min(hi, pos);
  } else if (p.mask_kind == kMaskDraftBlock) {
    const long long bd = p.draft_block;
    hi = min(hi, (floor_div_ll(pos, bd) + 1) * bd - 1);
  }
  if (p.window_l >= 0) lo = max(lo, pos - (long long)p.window_l);
  if (p.window_r >= 0) hi = min(hi, pos + (long long)p.window_r);
}

__device__ __forceinline__ bool bit_get(const uint32_t* bits, int i) {
  return (bits[i >> 5] >> (i & 31)) & 1u;
}

// The u-th unit (0 = heaviest): pairs of query tiles, last pair first.  With
// packed sequences, unit u is the pair `u / (B*Hq)` places before the last
// pair of its sequence (units past a short sequence's first pair are empty).
__device__ __forceinline__ void decode_unit(const FwdParams& p, int u, Unit& w) {
  const int BH = p.B * p.Hq;
  const int n_pairs = (p.q_tiles + 1) / 2;
  w.bh = u % BH;
  w.b = w.bh / p.Hq;
  w.hq = w.bh % p.Hq;
  w.hkv = w.hq / p.group;
  int Lq = p.Lq, pair = n_pairs - 1 - u / BH;
  w.Lk = p.Lk;
  w.q_base = w.k_base = 0;
  w.bad = false;
  if (p.cu_seqlens_q != nullptr) {
    const int cq0 = __ldg(p.cu_seqlens_q + w.b), cq1 = __ldg(p.cu_seqlens_q + w.b + 1);
    const int ck0 = __ldg(p.cu_seqlens_k + w.b), ck1 = __ldg(p.cu_seqlens_k + w.b + 1);
    Lq = cq1 - cq0;
    const int pairs_b = ((Lq + 127) / 128 + 1) / 2;  // <= n_pairs when Lq <= p.Lq
    w.bad = cq0 < 0 || cq1 < cq0 || cq1 > p.total_q || ck0 < 0 || ck1 < ck0 ||
            ck1 > p.total_k || ck1 - ck0 > kMaxKvTiles * kBlockN || Lq > p.Lq;
    pair = pairs_b - 1 - u / BH;
    if (w.bad || pair < 0) {  // nothing to do: no rows in either tile
      Lq = 0;
      pair = 0;
    }
    w.Lk = w.bad ? 0 : ck1 - ck0;
    w.q_base = w.bad ? 0 : cq0;
    w.k_base = w.bad ? 0 : ck0;
  }
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int q0 = (2 * pair + x) * 128;
    w.q0[x] = q0;
    w.rows[x] = max(0, min(128, Lq - q0));
    w.pos0[x] = (long long)w.Lk - Lq + q0;
  }
}

// Unit handled by CTA `cta` in round `r` (snake order), or -1.
__device__ __forceinline__ int unit_of(const FwdParams& p, int cta, int r) {
  const int G = gridDim.x;
  const int idx = r * G + ((r & 1) ? (G - 1 - cta) : cta);
  return idx < p.n_units ? idx : -1;
}

__device__ __forceinline__ void warp_min_max(int& mn, int& mx) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
}

// Whole warp: [mn, mx] of the document ids doc_b[pos(r)] of rows r < rows
// (rows <= 128).  All four loads of a lane are issued before any is used, so
// the warp pays one memory round trip, not one per 32 rows.  An empty range
// gives mn = INT_MAX, mx = INT_MIN.
template <typename PosFn>
__device__ __forceinline__ void doc_range_rows(const int32_t* doc_b, int rows, int lane, PosFn pos,
                                               int& mn, int& mx) {
  int d[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int r = lane + 32 * m;
    d[m] = r < rows ? __ldg(doc_b + pos(r)) : 0;
  }
  mn = 0x7fffffff;
  mx = (int)0x80000000;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    if (lane + 32 * m < rows) {
      mn = min(mn, d[m]);
      mx = max(mx, d[m]);
    }
  }
  warp_min_max(mn, mx);
}

// Whole warp: document range [mn[u], mx[u]] of key tiles t0 + u, u < kBatch,
// of kBN keys each (keys at or past Lk and tiles at or past t_end ignored).
// The kBatch * kBN / 32 loads of a lane are all in flight together; when the
// whole batch lies inside [0, Lk) and before t_end they come from one base
// address with constant offsets and need no predicates.
template <int kBN, int kBatch>
__device__ __forceinline__ void doc_range_tiles(const int32_t* doc_b, int Lk, int t0, int t_end,
                                                int lane, int (&mn)[kBatch], int (&mx)[kBatch]) {
  constexpr int kPer = kBN / 32;
  const long long k_first = (long long)t0 * kBN;
  const int32_t* base = doc_b + k_first + lane;
  if (t0 + kBatch <= t_end && k_first + kBatch * kBN <= Lk) {
    int d[kBatch][kPer];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
#pragma unroll
      for (int m = 0; m < kPer; ++m) d[u][m] = __ldg(base + u * kBN + 32 * m);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      mn[u] = mx[u] = d[u][0];
#pragma unroll
      for (int m = 1; m < kPer; ++m) {
        mn[u] = min(mn[u], d[u][m]);
        mx[u] = max(mx[u], d[u][m]);
      }
    }
  } else {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      mn[u] = 0x7fffffff;
      mx[u] = (int)0x80000000;
      if (t0 + u < t_end) {
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
          if (k_first + u * kBN + lane + 32 * m < Lk) {
            const int d = __ldg(base + u * kBN + 32 * m);
            mn[u] = min(mn[u], d);
            mx[u] = max(mx[u], d);
          }
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kBatch; ++u) warp_min_max(mn[u], mx[u]);
}

// Tile schedule of one unit for key tiles of kBN keys: bit i of empty[x] /
// full[x] describes key tile t_lo + i for query tile x.
template <int kBN>
struct Sched {
  static constexpr int kTiles = kMaxKvTiles * kBlockN / kBN;
  static constexpr int kWords = kTiles / 32;
  int t_lo, t_hi;   // union of the two query tiles' candidate key tiles
  int n[2];         // non-empty key tiles per query tile
  int last[2];      // last non-empty key tile per query tile (-1: none)
  int pad[2];
  uint32_t empty[2][kWords];
  uint32_t full[2][kWords];
};

// Whole warp: classify the key tiles (kBN keys each) of unit w into s.  A tile
// is EMPTY for a query tile when no row of it sees any key of the tile, FULL
// when every row sees every key (then no mask code runs), else PARTIAL.
template <int kBN>
__device__ void build_sched(const FwdParams& p, const Unit& w, Sched<kBN>* s, int lane) {
  long long lo_first[2], hi_first[2], lo_last[2], hi_last[2];
  int t_lo = 0x7fffffff, t_hi = -1;
  bool any[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    any[x] = false;
    lo_first[x] = hi_last[x] = 0;
    hi_first[x] = lo_last[x] = -1;
    if (w.rows[x] > 0) {
      key_bounds(p, w.Lk, w.pos0[x], lo_first[x], hi_first[x]);
      key_bounds(p, w.Lk, w.pos0[x] + w.rows[x] - 1, lo_last[x], hi_last[x]);
      if (hi_last[x] >= lo_first[x] && hi_last[x] >= 0) {
        any[x] = true;
        t_lo = min(t_lo, (int)(lo_first[x] / kBN));
        t_hi = max(t_hi, (int)(hi_last[x] / kBN));
      }
    }
  }
  if (t_hi < 0) {
    t_lo = 0;
    t_hi = -1;
  }
  const int ntc = t_hi - t_lo + 1;
  const int32_t* doc_b = p.doc_ids ? p.doc_ids + (long long)w.b * p.Lk : nullptr;
  int qdmin[2] = {0, 0}, qdmax[2] = {0, 0};
  if (doc_b) {
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const long long p0 = w.pos0[x];
      doc_range_rows(doc_b, w.rows[x], lane, [&](int r) { return p0 + r; }, qdmin[x], qdmax[x]);
    }
  }
  int cnt[2] = {0, 0}, last[2] = {-1, -1};
  for (int base = 0; base < ntc; base += 32) {
    const int i = base + lane;
    const long long k0 = (long long)(t_lo + i) * kBN;
    bool empty[2], full[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      empty[x] = (i >= ntc) || !any[x] || k0 > hi_last[x] || k0 + kBN - 1 < lo_first[x];
      full[x] = !empty[x] && (k0 + kBN <= w.Lk) && (lo_last[x] <= k0) &&
                (hi_first[x] >= k0 + kBN - 1);
    }
    if (doc_b) {
      constexpr int kBatch = 4;
      for (int ww0 = 0; ww0 < 32 && base + ww0 < ntc; ww0 += kBatch) {
        int mn[kBatch], mx[kBatch];
        doc_range_tiles<kBN, kBatch>(doc_b, p.Lk, t_lo + base + ww0, t_lo + ntc, lane, mn, mx);
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          if (lane == ww0 + u) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (mx[u] < qdmin[x] || mn[u] > qdmax[x]) empty[x] = true;
              if (!(mn[u] == mx[u] && qdmin[x] == qdmax[x] && mn[u] == qdmin[x])) full[x] = false;
            }
          }
        }
      }
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const uint32_t eb = __ballot_sync(0xffffffffu, empty[x]);
      const uint32_t fb = __ballot_sync(0xffffffffu, full[x] && !empty[x]);
      if (lane == 0) {
        s->empty[x][base >> 5] = eb;
        s->full[x][base >> 5] = fb;
      }
      cnt[x] += __popc(~eb);
      if (~eb) last[x] = t_lo + base + 31 - __clz(~eb);
    }
  }
  if (lane == 0) {
    s->t_lo = t_lo;
    s->t_hi = t_hi;
    s->n[0] = cnt[0];
    s->n[1] = cnt[1];
    s->last[0] = last[0];
    s->last[1] = last[1];
  }
}

template <int kBN>
__device__ __forceinline__ bool tile_used(const Sched<kBN>* s, int t) {
  const int i = t - s->t_lo;
  return !(bit_get(s->empty[0], i) && bit_get(s->empty[1], i));
}

// Shared-memory descriptors (128-byte swizzle, 1024-byte stride between 8-row
// groups): the high word is the same for every operand here, the low word
// holds the start address and the leading offset (16-byte units).
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);

__device__ __forceinline__ uint64_t make_desc(uint32_t addr, uint32_t lbo_bytes) {
  const uint32_t lo = ((addr >> 4) & 0x3FFFu) | ((lbo_bytes >> 4) << 16);
  return ((uint64_t)kDescHi << 32) | lo;
}

}  // namespace prefill
}  // namespace attn
