// Short-query prefill forward for sm_100a: a handful of query rows (at most
// 128 per KV head and row tile) over a long, masked key range, in one launch
// and without workspace.
//
// Method: the fused forward of "FlashAttention 2 原理与 PyTorch 实战" (sections
// 一, 3.1, 3.2) with the mask_mod predicates of "FlexAttention 是什么，以及 DFlash2
// 之谜的完整侦破" (section 1; the symmetric window and block-diffusion draft
// mask of sections 3 and 4), split over the keys like FlexDecoding /
// FlashDecoding (same page, section 1) and merged by log-sum-exp.  The
// DFlash draft call this serves ("a handful of draft queries" under a
// symmetric window, section 4, experiment 1) leaves the persistent prefill
// kernel with one mostly empty query tile per head, so it is latency-bound
// there.
//
// B200 mapping.  One thread-block cluster per (b, kv head, 128-row tile of the
// group's Hq/Hkv x Lq query rows); the cluster's CTAs split the key range that
// any of those rows can see (known on the host from the mask, before document
// ids) into chunks of whole 128-key tiles.  Inside a CTA (192 threads):
//   warp 0      classifies the chunk's key tiles (EMPTY / PARTIAL / FULL from
//               the rows' key intervals and document ids), then TMA-loads Q
//               and the non-empty K/V tiles into a ring of stages.
//   warp 1      allocates tensor memory; lane 0 issues tcgen05.mma:
//               S_j = Q K_j^T and O += P_j V_j (as in the split-KV decode).
//   warps 2..5  softmax: thread r owns tile row r (its TMEM lane); a warp with
//               no valid row skips the arithmetic.  Partial O / l and the
//               base-2 log-sum-exp of each row go to this CTA's shared memory.
// The partials never leave the cluster: after a cluster barrier, CTA 0 reads
// every CTA's partial rows over distributed shared memory, merges them,
// writes O (bf16) and the LSE, and a second cluster barrier keeps the others
// resident until it is done.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_params.h"
#include "host_once.h"
#include "prefill_common.cuh"
#include "ptx.cuh"
#include "softmax_row.cuh"

namespace attn {

namespace {

constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr uint32_t kTmemO = 256;
__device__ __forceinline__ uint32_t tmem_s(int j) { return (j & 1) ? 128u : 0u; }
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kMaxCluster = 8;

template <int D>
struct Cfg {
  static constexpr int kAtoms = D / 64;
  static constexpr int kAtomBytes = kBlockN * 128;
  static constexpr int kTileBytes = kBlockN * D * 2;
  static constexpr int kStages = (D == 64) ? 4 : 3;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffBits = kOffMisc + 64;
  static constexpr int kBitWords = kMaxKvTiles / 32;
  static constexpr int kSmemBytes = kOffBits + 2 * kBitWords * 4;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  // the partial results reuse the K/V ring once every load and MMA is done:
  // O_part [128 rows][D + 4] fp32 (padded rows), then LSE_part [128] fp32
  static constexpr int kPartStride = D + 4;
  static constexpr int kOffPartO = kOffK;
  static constexpr int kOffPartL = kOffPartO + 128 * kPartStride * 4;
  static_assert(kOffPartL + 128 * 4 <= kOffBar, "partials fit in the K/V ring");
};

struct Misc {
  uint32_t tmem_base;
  int abort;
  int n_tiles;
};

template <int D>
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_saddr, int kk) {
  uint32_t addr = tile_saddr + (kk >> 2) * Cfg<D>::kAtomBytes + (kk & 3) * 32;
  return ptx::smem_desc_sw128(addr, 16, 1024);
}

template <int D>
__device__ __forceinline__ uint64_t desc_v_mnmajor(uint32_t tile_saddr, int kk) {
  uint32_t addr = tile_saddr + kk * 2048;
  return ptx::smem_desc_sw128(addr, Cfg<D>::kAtomBytes, 1024);
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_short_kernel(const __grid_constant__ CUtensorMap tm_q,
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
  float* part_o = reinterpret_cast<float*>(smem + C::kOffPartO);
  float* part_l = reinterpret_cast<float*>(smem + C::kOffPartL);
  volatile int* abort_flag = &misc->abort;  // errors go to the device error word p.err

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ------------------------------------------------------------ work unit
  const uint32_t rank = ptx::cluster_ctarank();  // chunk of the key range
  const int bh = blockIdx.y / p.row_tiles;
  const int rt = blockIdx.y % p.row_tiles;
  const int b = bh / p.Hkv;
  const int hkv = bh % p.Hkv;
  const int c0 = p.key_lo + (int)rank * p.chunk;
  const int c1 = min(c0 + p.chunk, p.Lk);  // keys [c0, c1) (may be empty)
  const int rows_valid = min(kBlockM, p.group * p.Lq - rt * kBlockM);
  const long long row_out0 =
      ((long long)b * p.Hq + (long long)hkv * p.group) * p.Lq + (long long)rt * kBlockM;
  const int kv_z = b * p.Hkv + hkv;
  const int t_lo = c0 / kBlockN;
  const int t_hi = c1 > c0 ? (c1 - 1) / kBlockN : t_lo - 1;
  const int32_t* doc_b = p.doc_ids ? p.doc_ids + (long long)b * p.Lk : nullptr;
  // tile row r is query row i = (rt * 128 + r) % Lq of head hkv * group + ..., at
  // absolute position Lk - Lq + i (bottom-right alignment)
  auto row_pos = [&](int r) -> long long {
    return (long long)p.Lk - p.Lq + (long long)((rt * kBlockM + r) % p.Lq);
  };

  // ------------------------------------------------------------- prologue
  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_q);
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_v);
      ptx::mbar_init(q_full, 1);
      for (int s = 0; s < C::kStages; ++s) {
        ptx::mbar_init(&k_full[s], 1);
        ptx::mbar_init(&k_empty[s], 1);
        ptx::mbar_init(&v_full[s], 1);
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
      ptx::fence_mbar_init();
      // Q does not depend on the classification below: its load starts now
      ptx::mbar_arrive_expect_tx(q_full, C::kTileBytes);
      for (int a = 0; a < C::kAtoms; ++a)
        ptx::tma_load_2d(sQ + a * C::kAtomBytes, &tm_q, q_full, a * 64, (int)row_out0);
    }
    // Tile classification over the valid rows: the union [u_lo, u_hi] of their
    // key intervals decides EMPTY, the intersection [i_lo, i_hi] FULL; with
    // document ids a tile whose documents miss every row's document is EMPTY,
    // and FULL needs one document shared by the whole tile and every row.
    long long u_lo = 0x7fffffffffffLL, u_hi = -1, i_lo = 0, i_hi = 0x7fffffffffffLL;
    for (int r = lane; r < rows_valid; r += 32) {
      long long lo, hi;
      prefill::key_bounds(p, p.Lk, row_pos(r), lo, hi);
      lo = max(lo, 0LL);
      if (hi >= lo) {
        u_lo = min(u_lo, lo);
        u_hi = max(u_hi, hi);
      }
      i_lo = max(i_lo, lo);
      i_hi = min(i_hi, hi);
    }
    for (int o = 16; o > 0; o >>= 1) {
      u_lo = min(u_lo, __shfl_xor_sync(0xffffffffu, u_lo, o));
      u_hi = max(u_hi, __shfl_xor_sync(0xffffffffu, u_hi, o));
      i_lo = max(i_lo, __shfl_xor_sync(0xffffffffu, i_lo, o));
      i_hi = min(i_hi, __shfl_xor_sync(0xffffffffu, i_hi, o));
    }
    // document ids: Lq <= Lk, so every row position is a key index
    int qdmin = 0x7fffffff, qdmax = (int)0x80000000;
    if (doc_b != nullptr) prefill::doc_range_rows(doc_b, rows_valid, lane, row_pos, qdmin, qdmax);
    const int ntc = t_hi - t_lo + 1;
    int n_tiles = 0;
    for (int base = 0; base < ntc; base += 32) {
      const int i = base + lane;
      const long long k0 = (long long)(t_lo + i) * kBlockN;
      bool empty = i >= ntc || u_hi < 0 || k0 > u_hi || k0 + kBlockN - 1 < u_lo;
      bool full = !empty && (k0 + kBlockN <= p.Lk) && i_lo <= k0 && i_hi >= k0 + kBlockN - 1;
      if (doc_b != nullptr) {
        constexpr int kBatch = 4;
        for (int ww0 = 0; ww0 < 32 && base + ww0 < ntc; ww0 += kBatch) {
          int mn[kBatch], mx[kBatch];
          prefill::doc_range_tiles<kBlockN, kBatch>(doc_b, p.Lk, t_lo + base + ww0, t_lo + ntc,
                                                    lane, mn, mx);
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            if (lane == ww0 + u) {
              if (mx[u] < qdmin || mn[u] > qdmax) empty = true;
              if (!(mn[u] == mx[u] && qdmin == qdmax && mn[u] == qdmin)) full = false;
            }
          }
        }
      }
      const uint32_t eb = __ballot_sync(0xffffffffu, empty);
      const uint32_t fb = __ballot_sync(0xffffffffu, full && !empty);
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

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (n_tiles > 0 && lane == 0) {
      constexpr uint32_t kTx = C::kTileBytes;
      int j = 0;
      bool ok = true;
      for (int t = t_lo; t <= t_hi && ok; ++t) {
        if (prefill::bit_get(empty_bits, t - t_lo)) continue;
        const int s = j % C::kStages;
        const uint32_t ph = (uint32_t)(j / C::kStages) & 1u;
        const int k0 = t * kBlockN;
        ok = ptx::mbar_wait(&k_empty[s], ph ^ 1u, abort_flag, p.err,
                            kDevErrTimeoutProducer);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(&k_full[s], kTx);
        for (int a = 0; a < C::kAtoms; ++a)
          ptx::tma_load_3d(sK + s * C::kTileBytes + a * C::kAtomBytes, &tm_k, &k_full[s], a * 64,
                           k0, kv_z);
        ok = ptx::mbar_wait(&v_empty[s], ph ^ 1u, abort_flag, p.err,
                            kDevErrTimeoutProducer);
        if (!ok) {
          ++j;  // the K load of this tile is in flight; drain it below
          break;
        }
        ptx::mbar_arrive_expect_tx(&v_full[s], kTx);
        for (int a = 0; a < C::kAtoms; ++a)
          ptx::tma_load_3d(sV + s * C::kTileBytes + a * C::kAtomBytes, &tm_v, &v_full[s], a * 64,
                           k0, kv_z);
        ++j;
      }
      // Drain: every TMA write into shared memory lands before the partials
      // reuse the ring (in a normal run these phases completed long ago).
      int dummy_abort = 0;
      for (int jj = max(0, j - C::kStages); jj < j; ++jj) {
        const int s = jj % C::kStages;
        const uint32_t ph = (uint32_t)(jj / C::kStages) & 1u;
        dummy_abort = 0;
        ptx::mbar_wait(&k_full[s], ph, &dummy_abort, nullptr, 0);
        dummy_abort = 0;
        ptx::mbar_wait(&v_full[s], ph, &dummy_abort, nullptr, 0);
      }
    }
    if (lane == 0) {  // the Q load was issued in the prologue, whatever n_tiles is
      int dummy_abort = 0;
      ptx::mbar_wait(q_full, 0, &dummy_abort, nullptr, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
      constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kBlockM, D, 0, 1);
      const uint32_t q_saddr = ptx::smem_u32(sQ);
      const uint32_t k_saddr = ptx::smem_u32(sK);
      const uint32_t v_saddr = ptx::smem_u32(sV);
      bool ok = ptx::mbar_wait(q_full, 0, abort_flag, p.err, kDevErrTimeoutMma);
      auto issue_s = [&](int j) -> bool {
        const int s = j % C::kStages;
        const uint32_t ph = (uint32_t)(j / C::kStages) & 1u;
        if (!ptx::mbar_wait(&k_full[s], ph, abort_flag, p.err, kDevErrTimeoutMma))
          return false;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + tmem_s(j);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          ptx::mma_ss(d_tmem, desc_kmajor<D>(q_saddr, kk),
                      desc_kmajor<D>(k_saddr + s * C::kTileBytes, kk), kIdescS, kk > 0 ? 1u : 0u);
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
        ok = ptx::mbar_wait(&p_full[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, p.err,
                            kDevErrTimeoutMma);
        if (!ok) break;
        ok = ptx::mbar_wait(&v_full[s], (uint32_t)(j / C::kStages) & 1u, abort_flag,
                            p.err, kDevErrTimeoutMma);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t p_tmem = tmem + tmem_s(j);
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          ptx::mma_ts(tmem + kTmemO, p_tmem + kk * 8,
                      desc_v_mnmajor<D>(v_saddr + s * C::kTileBytes, kk), kIdescPV,
                      (j > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_commit(o_done);
        ptx::mma_commit(&v_empty[s]);
      }
      ptx::mma_commit(o_final);
      ptx::mma_commit(mma_drain);
      int dummy_abort = 0;
      ptx::mbar_wait(mma_drain, 0, &dummy_abort, nullptr, 0);
    }
  } else {
    // ----------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // tile row == TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool row_ok = r < rows_valid;
    const bool warp_active = quarter * 32 < rows_valid;  // warp-uniform
    const float c = p.scale_log2;
    int row_lo = 0, row_hi = -1, row_doc = 0;
    if (row_ok) {
      long long lo, hi;
      const long long pos = row_pos(r);
      prefill::key_bounds(p, p.Lk, pos, lo, hi);
      row_lo = (int)max(0LL, min(lo, (long long)p.Lk));
      row_hi = (int)max(-1LL, min(hi, (long long)p.Lk - 1));
      if (doc_b != nullptr) row_doc = __ldg(doc_b + pos);
    }
    float m_ref = -INFINITY;  // reference max (base-2 scaled units)
    float l = 0.0f;
    int j = 0;
    bool ok = true;
    for (int t = t_lo; t <= t_hi && ok; ++t) {
      if (prefill::bit_get(empty_bits, t - t_lo)) continue;
      const bool full = prefill::bit_get(full_bits, t - t_lo);
      const int k0 = t * kBlockN;
      ok = ptx::mbar_wait(&s_full[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag, p.err,
                          kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (warp_active) {
        ptx::tc_fence_after();
        uint32_t dm[4] = {~0u, ~0u, ~0u, ~0u};
        if (!full) {
          const int lo_rel = max(0, min(kBlockN, row_lo - k0));
          const int hi_rel = max(-1, min(kBlockN - 1, row_hi - k0));
          if (doc_b != nullptr) {
            const int kmax = min(kBlockN, p.Lk - k0);
            int kd[4];
#pragma unroll
            for (int g = 0; g < 4; ++g)
              kd[g] = (32 * g + lane < kmax) ? __ldg(doc_b + k0 + 32 * g + lane) : 0;
            uint32_t todo = 0xffffffffu;
            while (todo != 0u) {  // at most 32 rounds: each clears its leader's bit
              const int dv = __shfl_sync(0xffffffffu, row_doc, __ffs(todo) - 1);
              const uint32_t same = __ballot_sync(0xffffffffu, row_doc == dv);
              uint32_t bw[4];
#pragma unroll
              for (int g = 0; g < 4; ++g) bw[g] = __ballot_sync(0xffffffffu, kd[g] == dv);
              if ((same >> lane) & 1u) {
#pragma unroll
                for (int g = 0; g < 4; ++g) dm[g] = bw[g];
              }
              todo &= ~same;
            }
          }
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int a = lo_rel - 32 * g, bb = hi_rel - 32 * g;
            dm[g] &= (bb < 0 || a > 31 || a > bb) ? 0u
                                                   : (~0u << max(a, 0)) & (~0u >> (31 - min(bb, 31)));
          }
        }
        float s[kBlockN];
        row::tmem_ld_row128(t_row + tmem_s(j), s);
        if (!full) {
#pragma unroll
          for (int i = 0; i < kBlockN; ++i)
            s[i] = ((dm[i >> 5] >> (i & 31)) & 1u) ? s[i] : -INFINITY;
        }
        const float m_new = fmaxf(m_ref, ptx::row_max128(s) * c);
        const bool need = m_new > m_ref + kRescaleThreshold;
        const float alpha = need ? ptx::ex2(m_ref - m_new) : 1.0f;  // 0 when m_ref = -inf
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O holds P_{<j} V; it must be final before it is rescaled
          ok = ptx::mbar_wait(o_done, (uint32_t)(j - 1) & 1u, abort_flag, p.err,
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
            for (int i = 0; i < 32; ++i)
              raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
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
          l += row::exp2_pack128(s, c, m_use, pk_lo, pk_hi);
          ptx::tmem_st32(t_row + tmem_s(j), pk_lo);
          ptx::tmem_st32(t_row + tmem_s(j) + 32, pk_hi);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
      }
      ptx::mbar_arrive(&p_full[j & 1]);
      ++j;
    }

    // ------------------------------------------- this CTA's partial rows
    ok = __all_sync(0xffffffffu, ok);
    if (ok && n_tiles > 0) {
      ok = ptx::mbar_wait(o_final, 0, abort_flag, p.err, kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      ptx::tc_fence_after();
    }
    // every load of this CTA landed and every MMA is done before the ring is
    // reused for the partials (the producer drained its loads; o_final covers
    // the MMAs, and without tiles nothing was issued)
    const bool have = ok && n_tiles > 0 && l > 0.0f;
    const float inv_l = have ? 1.0f / l : 0.0f;
    if (warp_active) {
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
          float* dst = part_o + r * C::kPartStride + cc * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) =
                make_float4(have ? __uint_as_float(raw[i]) * inv_l : 0.0f,
                            have ? __uint_as_float(raw[i + 1]) * inv_l : 0.0f,
                            have ? __uint_as_float(raw[i + 2]) * inv_l : 0.0f,
                            have ? __uint_as_float(raw[i + 3]) * inv_l : 0.0f);
        }
      }
    }
    if (row_ok) part_l[r] = have ? m_ref + ptx::lg2(l) : -INFINITY;  // base 2
  }

  // ------------------------------------------------ merge over the cluster
  ptx::tc_fence_before();
  __syncwarp();
  ptx::cluster_sync();  // every CTA's partial rows are in its shared memory
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  if (rank == 0 && warp >= 2) {
    const int r = (warp - 2) * 32 + lane;
    if (r < rows_valid) {
      const uint32_t nparts = (uint32_t)p.nsplit;
      const uint32_t l_addr = ptx::smem_u32(part_l + r);
      const uint32_t o_addr = ptx::smem_u32(part_o + r * C::kPartStride);
      float lse2[kMaxCluster];
      float mx = -INFINITY;
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        lse2[q] = (uint32_t)q < nparts ? ptx::ld_cluster_f32(ptx::mapa(l_addr, (uint32_t)q))
                                       : -INFINITY;
        mx = fmaxf(mx, lse2[q]);
      }
      float w[kMaxCluster];
      float sum = 0.0f;
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        w[q] = (mx == -INFINITY || lse2[q] == -INFINITY) ? 0.0f : ptx::ex2(lse2[q] - mx);
        sum += w[q];
      }
      const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.o) + (row_out0 + r) * D;
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 8) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) {
          if (w[q] == 0.0f) continue;
          const uint32_t a = ptx::mapa(o_addr, (uint32_t)q) + (uint32_t)cc * 4u;
          const float4 v0 = ptx::ld_cluster_v4(a);
          const float4 v1 = ptx::ld_cluster_v4(a + 16u);
          acc[0] = fmaf(w[q], v0.x, acc[0]);
          acc[1] = fmaf(w[q], v0.y, acc[1]);
          acc[2] = fmaf(w[q], v0.z, acc[2]);
          acc[3] = fmaf(w[q], v0.w, acc[3]);
          acc[4] = fmaf(w[q], v1.x, acc[4]);
          acc[5] = fmaf(w[q], v1.y, acc[5]);
          acc[6] = fmaf(w[q], v1.z, acc[6]);
          acc[7] = fmaf(w[q], v1.w, acc[7]);
        }
        uint4 out;
        out.x = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
        out.y = ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv);
        out.z = ptx::pack_bf16x2(acc[4] * inv, acc[5] * inv);
        out.w = ptx::pack_bf16x2(acc[6] * inv, acc[7] * inv);
        *reinterpret_cast<uint4*>(dst + cc) = out;
      }
      p.lse[row_out0 + r] = sum > 0.0f ? (mx + ptx::lg2(sum)) * kLn2 : -INFINITY;
    }
  }
  __syncwarp();
  ptx::cluster_sync();  // the other CTAs stay resident until CTA 0 has read them
}

template <int D>
cudaError_t launch_short(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const FwdParams& p, int units, cudaStream_t stream) {
  auto kern = attn_short_kernel<D>;
  constexpr int smem = Cfg<D>::kSmemAlloc;
  static PerContextOnce once;
  cudaError_t e = once_per_context(once, [&](int) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.nsplit, (unsigned)units, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.nsplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template cudaError_t launch_short<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                      const FwdParams&, int, cudaStream_t);
template cudaError_t launch_short<128>(const CUtensorMap&, const CUtensorMap&,
                                       const CUtensorMap&, const FwdParams&, int, cudaStream_t);

}  // namespace attn
