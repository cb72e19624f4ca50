// Prefill attention forward for sm_100a: persistent CTAs, two query tiles per
// work unit.
//
// Method ("FlashAttention 2 原理与 PyTorch 实战", sections 一, 3.1, 3.2): query
// tiles stream K/V tiles through shared memory; S = Q K^T, mask, online softmax
// with a running max and sum, rescale of the accumulator, O += P V; O and the
// log-sum-exp are written at the end and the N x N scores never reach HBM.
// Masks: the mask_mod predicate of "FlexAttention 是什么，以及 DFlash2 之谜的完整
// 侦破" (section 1: causal, sliding window, non-causal, document ids; section 3:
// symmetric window, block-diffusion draft mask).
//
// B200 mapping.  A work unit is two adjacent 128-row query tiles (A and B) of
// one (batch, head); both consume the same K/V tiles, so one TMA stream feeds
// four tcgen05 MMAs per key tile (S_A, S_B, P_A V, P_B V).  384 threads:
//   warpgroup 0   warp 3: builds each unit's tile schedule (EMPTY / PARTIAL /
//                 FULL per key tile and query tile, in shared memory, double
//                 buffered), one unit ahead of the others, so the document-id
//                 loads of the classification never hold up the loads;
//                 warp 0: issues the TMA loads (Q_A, Q_B, K/V ring);
//                 warp 1 (and warp 2 for d = 64, one per query tile):
//                 allocate tensor memory and issue every MMA (elect.sync picks
//                 the issuing lane); registers lowered to 80 per thread.
//   warpgroup 1   softmax of tile A (one query row per thread = TMEM lane);
//   warpgroup 2   softmax of tile B; registers raised to 208 per thread.
// While warpgroup 1 turns S_A into P_A, the tensor core computes S_B and P_B V,
// and the other way round.  Tensor memory: S_A [0,128), S_B [128,256), O_A at
// 256, O_B at 256 + d.  P (bf16, 64 columns) is written over S when d = 128;
// when d = 64 it has columns of its own ([384,448), [448,512)), so the next
// key tile's S_x is computed while the softmax still works on this one.
// A CTA walks its units in a snake order over units sorted heaviest first.
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

using prefill::bit_get;
using prefill::build_sched;
using prefill::decode_unit;
using prefill::key_bounds;
using prefill::make_desc;
using prefill::Unit;
using prefill::unit_of;

constexpr int kThreads = 384;
constexpr int kRegsLow = 80;    // warpgroup 0 (producer, MMA)
constexpr int kRegsHigh = 208;  // softmax warpgroups: 80*128 + 2*208*128 <= 168*384
constexpr int kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
using row::kModAlibi;
using row::kModNone;
using row::kModRelBias;

using Sched = prefill::Sched<128>;

__device__ __forceinline__ bool tile_used(const Sched* s, int t) {
  return prefill::tile_used<128>(s, t);
}

template <int D>
struct Cfg {
  static constexpr int kAtoms = D / 64;
  static constexpr int kAtomBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kStages = (D == 64) ? 4 : 2;
  static constexpr int kOffQ = 0;  // Q_A, Q_B
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kNumBars = 21 + 4 * kStages;  // see the barrier slots below
  // d = 64 leaves tensor-memory columns for P of its own ([384,448) and
  // [448,512)), so S_x of the next key tile can be computed while the softmax
  // still works on this one; d = 128 writes P over S.
  static constexpr bool kSepP = (D == 64);
  static constexpr int kOffMisc = kOffBar + ((kNumBars * 8 + 15) / 16) * 16;
  static constexpr int kOffSched = kOffMisc + 64;
  static constexpr int kSmemBytes = kOffSched + 2 * (int)sizeof(Sched);
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
};

struct Misc {
  uint32_t tmem_base;
  int abort;
};

// Barrier slots (8 bytes each).  [2] = one per query tile (or per schedule buffer).
enum : int {
  kQFull = 0,        // [2] TMA -> MMA: Q_x landed
  kQEmpty = 2,       // [2] MMA -> TMA: last S_x of the unit issued and done
  kSFull = 4,        // [2] MMA -> softmax x: S_x ready
  kPFull = 6,        // [2] softmax x (128 arrivals) -> MMA: P_x written, O_x rescaled
  kODone = 8,        // [2] MMA -> softmax x: P_x V done
  kOFree = 10,       // [2] softmax x (128) -> MMA: O_x read out, may be overwritten
  kSchedFull = 12,   // [2] schedule builder -> TMA, MMA, softmax
  kSchedEmpty = 14,  // [2] TMA + MMA + 8 softmax warps -> schedule builder
  kDrain = 16,       // MMA: all MMAs done
  kSFree = 17,       // [2] softmax x (128) -> MMA: S_x loaded into registers (separate-P mode)
  kTurn = 19,        // [2] softmax 1-x (128) -> softmax x: x may run its exponentials
  kKvBase = 21,      // k_full[S], k_empty[S], v_full[S], v_empty[S]
};

template <int D>
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_saddr, int kk) {
  return make_desc(tile_saddr + (kk >> 2) * Cfg<D>::kAtomBytes + (kk & 3) * 32, 16);
}

template <int D>
__device__ __forceinline__ uint64_t desc_v(uint32_t tile_saddr, int kk) {
  return make_desc(tile_saddr + kk * 2048, Cfg<D>::kAtomBytes);
}

}  // namespace

// kMod: the score modifier (p the row's absolute position):
//   kModNone;  kModAlibi: S_ij += slope_h * (j - p), p.alibi_slopes[hq];
//   kModRelBias: S_ij += table[hq][clamp(j - p, -R, R) + R], p.rel_table, R = p.rel_max.
template <int D, int kMod>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Cfg<D>;
  constexpr int S = C::kStages;
  constexpr int kMmaWarps = C::kSepP ? 2 : 1;  // warps issuing MMAs
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // 32-bit shared-memory addresses of the tiles and barriers
  const uint32_t sq = ptx::smem_u32(smem + C::kOffQ);
  const uint32_t sk = ptx::smem_u32(smem + C::kOffK);
  const uint32_t sv_ = ptx::smem_u32(smem + C::kOffV);
  const uint32_t bar0 = ptx::smem_u32(smem + C::kOffBar);
  auto BAR = [bar0](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  Misc* misc = reinterpret_cast<Misc*>(smem + C::kOffMisc);
  Sched* scheds = reinterpret_cast<Sched*>(smem + C::kOffSched);
  volatile int* abort_flag = &misc->abort;
  int* err = p.err;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const bool packed = p.cu_seqlens_q != nullptr;  // token-major packed sequences

  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    for (int x = 0; x < 2; ++x) {
      ptx::mbar_init(&bars[kQFull + x], 1);
      ptx::mbar_init(&bars[kQEmpty + x], 1);
      ptx::mbar_init(&bars[kSFull + x], 1);
      ptx::mbar_init(&bars[kPFull + x], 128);
      ptx::mbar_init(&bars[kODone + x], 1);
      ptx::mbar_init(&bars[kOFree + x], 128);
      ptx::mbar_init(&bars[kSchedFull + x], 1);
      ptx::mbar_init(&bars[kSchedEmpty + x], 1 + kMmaWarps + 8);
      ptx::mbar_init(&bars[kSFree + x], 128);
      ptx::mbar_init(&bars[kTurn + x], 128);
    }
    for (int st = 0; st < S; ++st) {
      ptx::mbar_init(&bars[kKvBase + st], 1);          // k_full
      ptx::mbar_init(&bars[kKvBase + S + st], kMmaWarps);      // k_empty
      ptx::mbar_init(&bars[kKvBase + 2 * S + st], 1);  // v_full
      ptx::mbar_init(&bars[kKvBase + 3 * S + st], kMmaWarps);  // v_empty
    }
    ptx::mbar_init(&bars[kDrain], kMmaWarps);
    misc->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&misc->tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  auto K_FULL = [&](int st) { return BAR(kKvBase + st); };
  auto K_EMPTY = [&](int st) { return BAR(kKvBase + S + st); };
  auto V_FULL = [&](int st) { return BAR(kKvBase + 2 * S + st); };
  auto V_EMPTY = [&](int st) { return BAR(kKvBase + 3 * S + st); };

  if (warp < 4) {
    ptx::regs_dec<kRegsLow>();
    if (warp == 3) {
      // -------------------------------------------------- schedule builder
      for (int r = 0;; ++r) {
        const int u = unit_of(p, cta, r);
        if (u < 0) break;
        Unit w;
        decode_unit(p, u, w);
        if (w.bad && lane == 0) atomicOr(err, kDevErrBadSeqlens);
        bool ok = ptx::mbar_wait_a(BAR(kSchedEmpty + (r & 1)), (((uint32_t)r >> 1) & 1u) ^ 1u,
                                   abort_flag, err, kDevErrTimeoutProducer);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        build_sched(p, w, &scheds[r & 1], lane);
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_a(BAR(kSchedFull + (r & 1)));
      }
    } else if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      int jkv = 0;
      int rounds = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_of(p, cta, r);
        if (u < 0) break;
        rounds = r + 1;
        Unit w;
        decode_unit(p, u, w);
        const Sched* s = &scheds[r & 1];
        if (lane == 0) {
          ok = ptx::mbar_wait_a(BAR(kSchedFull + (r & 1)), ((uint32_t)r >> 1) & 1u, abort_flag,
                                err, kDevErrTimeoutProducer);
          constexpr uint32_t kTx = C::kTileBytes;
          for (int x = 0; x < 2 && ok; ++x) {
            ok = ptx::mbar_wait_a(BAR(kQEmpty + x), ((uint32_t)r & 1u) ^ 1u, abort_flag, err,
                                  kDevErrTimeoutProducer);
            if (!ok) break;
            if (w.rows[x] == 0) {  // tile past the sequence: nothing reads Q_x
              ptx::mbar_arrive_a(BAR(kQFull + x));
              continue;
            }
            ptx::mbar_arrive_expect_tx_a(BAR(kQFull + x), kTx);
            // [B, Hq, Lq, d]: (column, row, b*Hq + hq); packed: (column, hq, token)
            const int qy = packed ? w.hq : w.q0[x];
            const int qz = packed ? w.q_base + w.q0[x] : w.bh;
            for (int a = 0; a < C::kAtoms; ++a)
              ptx::tma_load_3d_a(sq + x * C::kTileBytes + a * C::kAtomBytes, &tm_q,
                                 BAR(kQFull + x), a * 64, qy, qz);
          }
          // [B, Hkv, Lk, d]: (column, key, b*Hkv + hkv); packed: (column, hkv, token)
          const int kv_z = packed ? 0 : w.b * p.Hkv + w.hkv;
          const int t_hi = s->t_hi;
          for (int t = s->t_lo; t <= t_hi && ok; ++t) {
            if (!tile_used(s, t)) continue;
            const int st = jkv % S;
            const uint32_t ph = (uint32_t)(jkv / S) & 1u;
            ok = ptx::mbar_wait_a(K_EMPTY(st), ph ^ 1u, abort_flag, err, kDevErrTimeoutProducer);
            if (!ok) break;
            ptx::mbar_arrive_expect_tx_a(K_FULL(st), kTx);
            for (int a = 0; a < C::kAtoms; ++a)
              ptx::tma_load_3d_a(sk + st * C::kTileBytes + a * C::kAtomBytes, &tm_k, K_FULL(st),
                                 a * 64, packed ? w.hkv : t * 128,
                                 packed ? w.k_base + t * 128 : kv_z);
            ok = ptx::mbar_wait_a(V_EMPTY(st), ph ^ 1u, abort_flag, err, kDevErrTimeoutProducer);
            if (!ok) {
              ++jkv;  // its K load is in flight: drain it below
              break;
            }
            ptx::mbar_arrive_expect_tx_a(V_FULL(st), kTx);
            for (int a = 0; a < C::kAtoms; ++a)
              ptx::tma_load_3d_a(sv_ + st * C::kTileBytes + a * C::kAtomBytes, &tm_v, V_FULL(st),
                                 a * 64, packed ? w.hkv : t * 128,
                                 packed ? w.k_base + t * 128 : kv_z);
            ++jkv;
          }
          ptx::mbar_arrive_a(BAR(kSchedEmpty + (r & 1)));  // done reading the schedule
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        jkv = __shfl_sync(0xffffffffu, jkv, 0);
      }
      // Drain: every TMA write into shared memory lands before the CTA exits
      // (in a normal run these phases completed long ago).
      if (lane == 0) {
        int dummy = 0;
        for (int jj = max(0, jkv - S); jj < jkv; ++jj) {
          const uint32_t ph = (uint32_t)(jj / S) & 1u;
          dummy = 0;
          ptx::mbar_wait_a(K_FULL(jj % S), ph, &dummy, nullptr, 0);
          dummy = 0;
          ptx::mbar_wait_a(V_FULL(jj % S), ph, &dummy, nullptr, 0);
        }
        if (rounds > 0) {
          for (int x = 0; x < 2; ++x) {
            dummy = 0;
            ptx::mbar_wait_a(BAR(kQFull + x), (uint32_t)(rounds - 1) & 1u, &dummy, nullptr, 0);
          }
        }
      }
    } else if (C::kSepP && (warp == 1 || warp == 2)) {
      // ------------------------------------ MMA issuers, d = 64: one per query tile
      // Warp 1 issues every MMA of query tile A and warp 2 those of tile B, so
      // neither waits on the other tile's softmax.  With separate P columns,
      // S_x of key tile t only needs the softmax to have loaded the previous
      // S_x, and P_x V of the previous tile follows when P_x is written.  Both
      // warps release every K/V stage (two arrivals), each after that stage's
      // load has landed, so the ring's phases stay in order.
      const int x = warp - 1;
      constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, 0, 1);
      const uint32_t d_tmem = tmem + (x ? 128u : 0u);
      const uint32_t p_tmem = tmem + 384u + (uint32_t)(x * 64);
      const uint32_t o_tmem = tmem + 256u + (uint32_t)(x * D);
      const uint64_t q_desc = desc_kmajor<D>(sq + x * C::kTileBytes, 0);
      int jkv = 0, ns = 0, np = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_of(p, cta, r);
        if (u < 0) break;
        const Sched* s = &scheds[r & 1];
        ok = ptx::mbar_wait_a(BAR(kSchedFull + (r & 1)), ((uint32_t)r >> 1) & 1u, abort_flag, err,
                              kDevErrTimeoutMma);
        if (ok)
          ok = ptx::mbar_wait_a(BAR(kQFull + x), (uint32_t)r & 1u, abort_flag, err,
                                kDevErrTimeoutMma);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
        const int t_lo = s->t_lo, t_hi = s->t_hi;
        const int last = s->last[x];
        bool first = true;
        // P_x V of key tile tp (union index jp), then release its V stage
        auto issue_pv = [&](int jp, bool mine) -> bool {
          const int stp = jp % S;
          bool w_ok = ptx::mbar_wait_a(V_FULL(stp), (uint32_t)(jp / S) & 1u, abort_flag, err,
                                       kDevErrTimeoutMma);
          if (w_ok && mine && first && r > 0)
            w_ok = ptx::mbar_wait_a(BAR(kOFree + x), (uint32_t)(r - 1) & 1u, abort_flag, err,
                                    kDevErrTimeoutMma);
          if (w_ok && mine)
            w_ok = ptx::mbar_wait_a(BAR(kPFull + x), (uint32_t)np & 1u, abort_flag, err,
                                    kDevErrTimeoutMma);
          if (!__all_sync(0xffffffffu, w_ok)) return false;
          ptx::tc_fence_after();
          if (mine) {
            ptx::mma_pv_chain8(o_tmem, p_tmem, desc_v<D>(sv_ + stp * C::kTileBytes, 0), kIdescPV,
                               first ? 0u : 1u);
            ptx::mma_commit_warp(BAR(kODone + x));
            ++np;
            first = false;
          }
          ptx::mma_commit_warp(V_EMPTY(stp));
          return true;
        };
        int t_prev = -1, j_prev = 0;
        bool mine_prev = false;
        // the schedule's bits for 32 key tiles at a time, in registers
        int w_idx = -1;
        uint32_t w_e0 = 0u, w_e1 = 0u;
        for (int t = t_lo; t <= t_hi && ok; ++t) {
          const int ti = t - t_lo;
          if ((ti >> 5) != w_idx) {
            w_idx = ti >> 5;
            w_e0 = s->empty[0][w_idx];
            w_e1 = s->empty[1][w_idx];
          }
          const uint32_t tbit = 1u << (ti & 31);
          if (w_e0 & w_e1 & tbit) continue;  // no query tile of the unit uses key tile t
          const int st = jkv % S;
          const bool mine = ((x ? w_e1 : w_e0) & tbit) == 0u;
          // the softmax has loaded the previous S_x; K(t) has landed
          if (mine && ns > 0)
            ok = ptx::mbar_wait_a(BAR(kSFree + x), (uint32_t)(ns - 1) & 1u, abort_flag, err,
                                  kDevErrTimeoutMma);
          if (ok)
            ok = ptx::mbar_wait_a(K_FULL(st), (uint32_t)(jkv / S) & 1u, abort_flag, err,
                                  kDevErrTimeoutMma);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ptx::tc_fence_after();
          if (mine) {
            const uint64_t k_desc = desc_kmajor<D>(sk + st * C::kTileBytes, 0);
            if constexpr (D == 64)
              ptx::mma_qk_chain_d64(d_tmem, q_desc, k_desc, kIdescS);
            else
              ptx::mma_qk_chain_d128(d_tmem, q_desc, k_desc, kIdescS);
            ptx::mma_commit_warp(BAR(kSFull + x));
            ++ns;
            if (t == last) ptx::mma_commit_warp(BAR(kQEmpty + x));  // Q_x no longer read
          }
          ptx::mma_commit_warp(K_EMPTY(st));
          if (t_prev >= 0) ok = issue_pv(j_prev, mine_prev);
          t_prev = t;
          j_prev = jkv;
          mine_prev = mine;
          ++jkv;
        }
        if (ok && t_prev >= 0) ok = issue_pv(j_prev, mine_prev);
        if (last < 0) ptx::mma_commit_warp(BAR(kQEmpty + x));  // no key tile: Q_x unused
        if (lane == 0) ptx::mbar_arrive_a(BAR(kSchedEmpty + (r & 1)));
      }
      ptx::mma_commit_warp(BAR(kDrain));
      int dummy = 0;
      ptx::mbar_wait_a(BAR(kDrain), 0, &dummy, nullptr, 0);
    } else if (!C::kSepP && warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      // The whole warp runs this loop with warp-uniform values; elect.sync
      // picks the lane that issues each tcgen05.mma / commit.
      {
        constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, 0, 1);
        int jkv = 0;
        int ns0 = 0, ns1 = 0;  // S MMAs issued per query tile (global count)
        bool ok = true;
        for (int r = 0; ok; ++r) {
          const int u = unit_of(p, cta, r);
          if (u < 0) break;
          const Sched* s = &scheds[r & 1];
          ok = ptx::mbar_wait_a(BAR(kSchedFull + (r & 1)), ((uint32_t)r >> 1) & 1u, abort_flag,
                                err, kDevErrTimeoutMma);
          for (int x = 0; x < 2 && ok; ++x)
            ok = ptx::mbar_wait_a(BAR(kQFull + x), (uint32_t)r & 1u, abort_flag, err,
                                  kDevErrTimeoutMma);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ptx::tc_fence_after();
          const int t_lo = s->t_lo, t_hi = s->t_hi;
          const int last0 = s->last[0], last1 = s->last[1];
          bool first0 = true, first1 = true;
          // S_x(t) = Q_x K(t)^T into S_x; K(t) sits in stage st
          auto issue_s = [&](int t, int st, int x) {
            const uint32_t d_tmem = tmem + (x ? 128u : 0u);
            const uint64_t qd = desc_kmajor<D>(sq + x * C::kTileBytes, 0);
            const uint64_t kd = desc_kmajor<D>(sk + st * C::kTileBytes, 0);
            if constexpr (D == 64)
              ptx::mma_qk_chain_d64(d_tmem, qd, kd, kIdescS);
            else
              ptx::mma_qk_chain_d128(d_tmem, qd, kd, kIdescS);
            ptx::mma_commit_warp(BAR(kSFull + x));
            if (x) ++ns1; else ++ns0;
            if (t == (x ? last1 : last0)) ptx::mma_commit_warp(BAR(kQEmpty + x));
          };
          int t = t_lo;
          while (t <= t_hi && !tile_used(s, t)) ++t;
          if (t <= t_hi) {
            const int st = jkv % S;
            ok = ptx::mbar_wait_a(K_FULL(st), (uint32_t)(jkv / S) & 1u, abort_flag, err,
                                  kDevErrTimeoutMma);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
              ptx::tc_fence_after();
              for (int x = 0; x < 2; ++x)
                if (!bit_get(s->empty[x], t - t_lo)) issue_s(t, st, x);
              ptx::mma_commit_warp(K_EMPTY(st));
            }
          }
          while (ok && t <= t_hi) {
            int tn = t + 1;
            while (tn <= t_hi && !tile_used(s, tn)) ++tn;
            const bool has_next = tn <= t_hi;
            const int st = jkv % S;
            const int stn = (jkv + 1) % S;
            bool k_ready = false;
            for (int x = 0; x < 2 && ok; ++x) {
              if (!bit_get(s->empty[x], t - t_lo)) {
                // O_x free (first P V of the unit), P_x(t) written, V(t) landed
                if ((x ? first1 : first0) && r > 0) {
                  ok = ptx::mbar_wait_a(BAR(kOFree + x), (uint32_t)(r - 1) & 1u, abort_flag, err,
                                        kDevErrTimeoutMma);
                  ok = __all_sync(0xffffffffu, ok);
                  if (!ok) break;
                }
                ok = ptx::mbar_wait_a(BAR(kPFull + x), (uint32_t)((x ? ns1 : ns0) - 1) & 1u,
                                      abort_flag, err, kDevErrTimeoutMma);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ok = ptx::mbar_wait_a(V_FULL(st), (uint32_t)(jkv / S) & 1u, abort_flag, err,
                                      kDevErrTimeoutMma);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t p_tmem = tmem + (x ? 128u : 0u);
                const uint32_t o_tmem = tmem + 256u + (uint32_t)(x * D);
                const uint32_t va = sv_ + st * C::kTileBytes;
                const uint32_t acc0 = (x ? first1 : first0) ? 0u : 1u;
                ptx::mma_pv_chain8(o_tmem, p_tmem, desc_v<D>(va, 0), kIdescPV, acc0);
                ptx::mma_commit_warp(BAR(kODone + x));
                if (x) first1 = false; else first0 = false;
              }
              // S_x of the next key tile right behind this tile's P_x V
              if (has_next && !bit_get(s->empty[x], tn - t_lo)) {
                if (!k_ready) {
                  ok = ptx::mbar_wait_a(K_FULL(stn), (uint32_t)((jkv + 1) / S) & 1u, abort_flag,
                                        err, kDevErrTimeoutMma);
                  ok = __all_sync(0xffffffffu, ok);
                  if (!ok) break;
                  ptx::tc_fence_after();
                  k_ready = true;
                }
                issue_s(tn, stn, x);
              }
            }
            if (!ok) break;
            ptx::mma_commit_warp(V_EMPTY(st));
            if (has_next) ptx::mma_commit_warp(K_EMPTY(stn));  // both S of the next tile issued
            ++jkv;
            t = tn;
          }
          // a query tile with no key tile at all still releases its Q buffer
          if (last0 < 0) ptx::mma_commit_warp(BAR(kQEmpty + 0));
          if (last1 < 0) ptx::mma_commit_warp(BAR(kQEmpty + 1));
          if (lane == 0) ptx::mbar_arrive_a(BAR(kSchedEmpty + (r & 1)));
        }
        ptx::mma_commit_warp(BAR(kDrain));
        int dummy = 0;
        ptx::mbar_wait_a(BAR(kDrain), 0, &dummy, nullptr, 0);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax
    ptx::regs_inc<kRegsHigh>();
    const int x = (warp - 4) >> 2;  // query tile A (0) or B (1)
    const int quarter = warp & 3;
    const int r_row = quarter * 32 + lane;
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_col = x ? 128u : 0u;
    const uint32_t o_col = 256u + (uint32_t)(x * D);
    const uint32_t p_col = C::kSepP ? 384u + (uint32_t)(x * 64) : s_col;
    const uint32_t bar_s_full = BAR(kSFull + x);
    const uint32_t bar_p_full = BAR(kPFull + x);
    const uint32_t bar_o_done = BAR(kODone + x);
    const uint32_t bar_o_free = BAR(kOFree + x);
    const float c = p.scale_log2;
    const float c_s = kMod != kModNone ? 1.0f : c;  // scale still to apply to the loaded scores
    int ns = 0;  // S tiles consumed (global count)
    // The two softmax warpgroups take turns on the exponentials of each key
    // tile (A, B, A, B, ...), so that one loads S, finds the row max and stores
    // P while the other keeps the MUFU unit busy.  kTurn[x] completes once per
    // turn handed to x; B hands A the first turn.
    const uint32_t bar_my_turn = BAR(kTurn + x);
    const uint32_t bar_other_turn = BAR(kTurn + (x ^ 1));
    int turns = 0;
    if (x == 1) ptx::mbar_arrive_a(bar_other_turn);
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int u = unit_of(p, cta, r);
      if (u < 0) break;
      Unit w;
      decode_unit(p, u, w);
      const Sched* s = &scheds[r & 1];
      ok = ptx::mbar_wait_a(BAR(kSchedFull + (r & 1)), ((uint32_t)r >> 1) & 1u, abort_flag, err,
                            kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const bool row_ok = r_row < w.rows[x];
      // ALiBi: the row's absolute position and the head's slope times log2(e)
      const long long row_pos = w.pos0[x] + r_row;
      const float alibi2 = kMod == kModAlibi ? __ldg(p.alibi_slopes + w.hq) * kLog2e : 0.0f;
      // relative-position table of the head, centred on j - p = 0
      const float* rel_row =
          kMod == kModRelBias ? p.rel_table + (long long)w.hq * (2 * p.rel_max + 1) + p.rel_max
                              : nullptr;
      int row_lo = 0, row_hi = -1;  // visible key range, clamped to [0, Lk-1]
      int row_doc = 0;
      // document ids of this batch row (warp-uniform: every lane takes part in
      // the ballots below, rows past Lq included)
      const int32_t* doc_b = p.doc_ids ? p.doc_ids + (long long)w.b * p.Lk : nullptr;
      if (row_ok) {
        const long long pos = w.pos0[x] + r_row;
        long long lo, hi;
        key_bounds(p, w.Lk, pos, lo, hi);
        row_lo = (int)max(0LL, min(lo, (long long)w.Lk));
        row_hi = (int)max(-1LL, min(hi, (long long)w.Lk - 1));
        if (doc_b != nullptr) row_doc = __ldg(doc_b + pos);
      }
      const int t_lo = s->t_lo, t_hi = s->t_hi;
      const int n_mine = s->n[x];
      float m_ref = -INFINITY;
      float l = 0.0f;
      int jl = 0;
      // the schedule's bits for 32 key tiles at a time, in registers
      int w_idx = -1;
      uint32_t w_e0 = 0u, w_e1 = 0u, w_full = 0u;
      for (int t = t_lo; t <= t_hi && ok; ++t) {
        const int ti = t - t_lo;
        if ((ti >> 5) != w_idx) {
          w_idx = ti >> 5;
          w_e0 = s->empty[0][w_idx];
          w_e1 = s->empty[1][w_idx];
          w_full = s->full[x][w_idx];
        }
        const uint32_t tbit = 1u << (ti & 31);
        if (w_e0 & w_e1 & tbit) continue;  // no query tile of the unit uses key tile t
        if ((x ? w_e1 : w_e0) & tbit) {
          // no key tile of ours here: pass the turn on
          ok = ptx::mbar_wait_a(bar_my_turn, (uint32_t)turns & 1u, abort_flag, err,
                                kDevErrTimeoutSoftmax);
          ok = __all_sync(0xffffffffu, ok);
          ++turns;
          ptx::mbar_arrive_a(bar_other_turn);
          continue;
        }
        const bool full = (w_full & tbit) != 0u;
        const int k0 = t * 128;
        ok = ptx::mbar_wait_a(bar_s_full, (uint32_t)ns & 1u, abort_flag, err,
                              kDevErrTimeoutSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
        float sv[128];
        {
          // all four 32-column loads in flight, one wait
          uint32_t r0[32], r1[32], r2[32], r3[32];
          ptx::tmem_ld32(t_row + s_col + 0, r0);
          ptx::tmem_ld32(t_row + s_col + 32, r1);
          ptx::tmem_ld32(t_row + s_col + 64, r2);
          ptx::tmem_ld32(t_row + s_col + 96, r3);
          ptx::tmem_wait_ld();
          if constexpr (C::kSepP) {
            // S_x is in registers: its columns may take the next tile's S_x
            ptx::tc_fence_before();
            ptx::mbar_arrive_a(BAR(kSFree + x));
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            sv[i] = __uint_as_float(r0[i]);
            sv[32 + i] = __uint_as_float(r1[i]);
            sv[64 + i] = __uint_as_float(r2[i]);
            sv[96 + i] = __uint_as_float(r3[i]);
          }
        }
        if (!full) {
          // visible keys of this row inside the tile: [lo_rel, hi_rel], and with
          // document ids one visibility bit per key (dm0..dm3 = keys 0..127)
          const int lo_rel = max(0, min(128, row_lo - k0));
          const int hi_rel = max(-1, min(127, row_hi - k0));
          uint32_t dm0 = ~0u, dm1 = ~0u, dm2 = ~0u, dm3 = ~0u;
          if (doc_b != nullptr) {
            // lane i holds the document of keys k0 + 32g + i (g = 0..3); for each
            // distinct row document in the warp one ballot per word gives every
            // row with that document its visibility bits.  Keys past Lk are
            // outside [lo_rel, hi_rel] whatever their bit says.
            const int kmax = min(128, p.Lk - k0);
            int kd[4];
#pragma unroll
            for (int g = 0; g < 4; ++g)
              kd[g] = (32 * g + lane < kmax) ? __ldg(doc_b + k0 + 32 * g + lane) : 0;
            uint32_t todo = 0xffffffffu;
            while (todo != 0u) {  // at most 32 rounds: each clears its leader's bit
              const int dv = __shfl_sync(0xffffffffu, row_doc, __ffs(todo) - 1);
              const uint32_t same = __ballot_sync(0xffffffffu, row_doc == dv);
              const uint32_t w0 = __ballot_sync(0xffffffffu, kd[0] == dv);
              const uint32_t w1 = __ballot_sync(0xffffffffu, kd[1] == dv);
              const uint32_t w2 = __ballot_sync(0xffffffffu, kd[2] == dv);
              const uint32_t w3 = __ballot_sync(0xffffffffu, kd[3] == dv);
              if ((same >> lane) & 1u) {
                dm0 = w0;
                dm1 = w1;
                dm2 = w2;
                dm3 = w3;
              }
              todo &= ~same;
            }
          }
          // fold the key range into the four words: word g holds keys 32g..32g+31
          {
            auto range_bits = [&](int g) -> uint32_t {
              const int a = lo_rel - 32 * g, b = hi_rel - 32 * g;
              if (b < 0 || a > 31 || a > b) return 0u;
              return (~0u << max(a, 0)) & (~0u >> (31 - min(b, 31)));
            };
            dm0 &= range_bits(0);
            dm1 &= range_bits(1);
            dm2 &= range_bits(2);
            dm3 &= range_bits(3);
          }
#pragma unroll
          for (int i = 0; i < 128; ++i) {
            const uint32_t word = i < 32 ? dm0 : (i < 64 ? dm1 : (i < 96 ? dm2 : dm3));
            sv[i] = ((word >> (i & 31)) & 1u) ? sv[i] : -INFINITY;
          }
        }
        // scores to the base-2 domain with the score modifier (masked scores stay
        // -inf); the max and the exponentials below then use a scale of 1
        if constexpr (kMod != kModNone)
          row::score_mod128<kMod>(sv, c, (int)(k0 - row_pos), alibi2, rel_row, p.rel_max);
        // row max: sixteen independent chains of two-input max, then a tree
        float mx16[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) mx16[j] = fmaxf(sv[j], sv[16 + j]);
#pragma unroll
        for (int i = 32; i < 128; i += 16) {
#pragma unroll
          for (int j = 0; j < 16; ++j) mx16[j] = fmaxf(mx16[j], sv[i + j]);
        }
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
          for (int j = 0; j < w; ++j) mx16[j] = fmaxf(mx16[j], mx16[j + w]);
        }
        const float mx = mx16[0];
        const float m_new = fmaxf(m_ref, mx * c_s);
        const bool need = m_new > m_ref + kRescaleThreshold;
        const float alpha = need ? ptx::ex2(m_ref - m_new) : 1.0f;
        if (need) {
          l *= alpha;
          m_ref = m_new;
        }
        const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
        // P = 2^(s*c - m) as packed bf16 pairs, all in registers first, so the
        // wait for the previous P V (below) overlaps the exponentials.
        // four 16-column pieces, each the register range of one tcgen05.st
        uint32_t pk0[16], pk1[16], pk2[16], pk3[16];
        float sum8[8];  // four packed (even, odd) partial sums
#pragma unroll
        for (int j = 0; j < 8; ++j) sum8[j] = 0.0f;
        // The exponentials of pair i are issued kAhead pairs before their sum
        // and bf16 packing, so the MUFU results are ready when those read them
        // and one warp keeps the unit fed (measured: 4 pairs ahead is best).
        ok = ptx::mbar_wait_a(bar_my_turn, (uint32_t)turns & 1u, abort_flag, err,
                              kDevErrTimeoutSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++turns;
        {
          constexpr int kAhead = 4;
          float e0[kAhead], e1[kAhead];
#pragma unroll
          for (int i = 0; i < 64 + kAhead; ++i) {
            // slot i % kAhead: first consume pair i - kAhead, then refill it with pair i
            if (i >= kAhead) {
              const int j = i - kAhead;
              const float p0 = e0[j % kAhead], p1 = e1[j % kAhead];
              ptx::add2_acc(sum8[(j & 3) * 2], sum8[(j & 3) * 2 + 1], p0, p1);
              const uint32_t packed = ptx::pack_bf16x2(p0, p1);
              if (j < 16) pk0[j] = packed;
              else if (j < 32) pk1[j - 16] = packed;
              else if (j < 48) pk2[j - 32] = packed;
              else pk3[j - 48] = packed;
            }
            if (i < 64) {
              const int i0 = 2 * i, i1 = i0 + 1;
              float a0, a1;
              ptx::fma2_bc(a0, a1, sv[i0], sv[i1], c_s, -m_use);  // s * c - m, two at once
              e0[i % kAhead] = ptx::ex2(a0);
              e1[i % kAhead] = ptx::ex2(a1);
            }
          }
        }
        ptx::mbar_arrive_a(bar_other_turn);
#pragma unroll
        for (int j = 0; j < 4; ++j) sum8[j] += sum8[j + 4];
        l += (sum8[0] + sum8[1]) + (sum8[2] + sum8[3]);
        // P_x V of the previous tile must be done before O_x is rescaled and,
        // with separate P columns, before P_x is overwritten.  With P over S it
        // is already done (it was issued before the S just read).
        const bool any_need = __any_sync(0xffffffffu, need);
        if (jl > 0 && (C::kSepP || any_need)) {
          ok = ptx::mbar_wait_a(bar_o_done, (uint32_t)(ns - 1) & 1u, abort_flag, err,
                                kDevErrTimeoutSoftmax);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ptx::tc_fence_after();
        }
        if (jl > 0 && any_need) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t raw[32];
            ptx::tmem_ld32(t_row + o_col + cc * 32, raw);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
            ptx::tmem_st32(t_row + o_col + cc * 32, raw);
          }
        }
        ptx::tmem_st16(t_row + p_col + 0, pk0);
        ptx::tmem_st16(t_row + p_col + 16, pk1);
        ptx::tmem_st16(t_row + p_col + 32, pk2);
        ptx::tmem_st16(t_row + p_col + 48, pk3);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive_a(bar_p_full);
        ++ns;
        ++jl;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_a(BAR(kSchedEmpty + (r & 1)));
      ok = __all_sync(0xffffffffu, ok);
      // ------------------------------------------------------------- epilogue
      const bool have_o = ok && n_mine > 0 && jl == n_mine;
      if (have_o) {
        ok = ptx::mbar_wait_a(bar_o_done, (uint32_t)(ns - 1) & 1u, abort_flag, err,
                              kDevErrTimeoutSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        ptx::tc_fence_after();
      }
      const bool have = have_o && ok && l > 0.0f;
      const float inv_l = have ? 1.0f / l : 0.0f;
      const float lse_row = have ? (m_ref + ptx::lg2(l)) * kLn2 : -INFINITY;
      // [B, Hq, Lq, d] / [B, Hq, Lq]; packed: [total_q, Hq, d] / [Hq, total_q]
      const long long tok = (long long)w.q_base + w.q0[x] + r_row;
      const long long out_row = packed ? tok * p.Hq + w.hq : (long long)w.bh * p.Lq + w.q0[x] + r_row;
      const long long lse_idx = packed ? (long long)w.hq * p.total_q + tok : out_row;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t raw[32];
        if (have_o && ok) {
          ptx::tmem_ld32(t_row + o_col + cc * 32, raw);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) raw[i] = 0u;
        }
        if (row_ok) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.o) + out_row * D + cc * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v4;
            v4.x = ptx::pack_bf16x2(__uint_as_float(raw[i]) * inv_l,
                                    __uint_as_float(raw[i + 1]) * inv_l);
            v4.y = ptx::pack_bf16x2(__uint_as_float(raw[i + 2]) * inv_l,
                                    __uint_as_float(raw[i + 3]) * inv_l);
            v4.z = ptx::pack_bf16x2(__uint_as_float(raw[i + 4]) * inv_l,
                                    __uint_as_float(raw[i + 5]) * inv_l);
            v4.w = ptx::pack_bf16x2(__uint_as_float(raw[i + 6]) * inv_l,
                                    __uint_as_float(raw[i + 7]) * inv_l);
            *reinterpret_cast<uint4*>(dst + i) = v4;
          }
        }
      }
      if (row_ok) p.lse[lse_idx] = lse_row;
      ptx::tc_fence_before();
      ptx::mbar_arrive_a(bar_o_free);
    }
  }

  // ------------------------------------------------------------------ teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int kMod>
cudaError_t launch_prefill_kernel(const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const FwdParams& p, int grid,
                                  cudaStream_t stream) {
  auto kern = attn_prefill_kernel<D, kMod>;
  constexpr int smem = Cfg<D>::kSmemAlloc;
  static PerContextOnce once;
  const cudaError_t e = once_per_context(once, [&](int) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const FwdParams& p, int grid, cudaStream_t stream) {
  if (p.alibi_slopes) return launch_prefill_kernel<D, kModAlibi>(tq, tk, tv, p, grid, stream);
  if (p.rel_table) return launch_prefill_kernel<D, kModRelBias>(tq, tk, tv, p, grid, stream);
  return launch_prefill_kernel<D, kModNone>(tq, tk, tv, p, grid, stream);
}

template cudaError_t launch_prefill<64>(const CUtensorMap&, const CUtensorMap&,
                                        const CUtensorMap&, const FwdParams&, int, cudaStream_t);
template cudaError_t launch_prefill<128>(const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const FwdParams&, int, cudaStream_t);

}  // namespace attn
