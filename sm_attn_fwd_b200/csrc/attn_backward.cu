// Backward pass of the attention forward for sm_100a (B200): dQ, dK, dV.
//
// Method ("FlashAttention 2 原理与 PyTorch 实战", section 3.2: the forward keeps
// only O and the row statistics; the backward recomputes the scores tile by
// tile instead of storing the N x N matrix).  With P the masked softmax of
// S = scale * Q K^T:
//   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q,
// and P_ij = exp(S_ij - LSE_i) from the forward's log-sum-exp.
//
// B200 mapping.  Two gradient kernels: attn_bwd64_pipe_kernel (d = 64, below,
// with its own description) and attn_bwd_kernel<D>, which the library runs for
// d = 128.  attn_bwd_kernel: one CTA per (b, kv head, 128-key tile), 192
// threads, the heaviest key tiles dispatched first; it keeps its K and V tiles
// in shared memory and walks every query tile of every query head of its
// group:
//   warp 0     TMA producer: K and V once; per query tile Q, dO and, by all
//              lanes, the tile's row statistics (-LSE in base 2, -D, document
//              ids), loaded one tile ahead.
//   warp 1     tcgen05.mma issue (elect.sync): S^T = K Q^T and dP^T = V dO^T
//              (both operands K-major in shared memory), then dV += P^T dO and
//              dK += dS^T Q (P^T, dS^T from tensor memory, dO, Q MN-major), and
//              dQ_tile = dS K (dS from shared memory, MN-major, K MN-major).
//   warps 2-5  one key per thread (its TMEM lane): P^T and dS^T for 128 query
//              columns, written to tensor memory (bf16, over S^T and dP^T) and
//              dS^T to shared memory; then, one query per thread, the dQ tile
//              is staged in shared memory and added into an fp32 accumulator in
//              global memory by TMA reduce-adds; at the end dK (times scale)
//              and dV are stored as bf16.
// Tensor memory (512 columns) at d = 128: dV [256,384), dK [384,512); P^T and
// dS^T (bf16) take the lower 64 columns of S^T [0,128) and dP^T [128,256), and
// the dQ tile (fp32, 128 columns) is computed as two 64-column halves into the
// freed upper halves, [64,128) and [192,256), so S^T of the next query tile
// waits for the dQ read-out; Q, dO and the row statistics have one buffer (a
// second does not fit in shared memory).
// Small kernels before and after: D_i, and dQ from its fp32 accumulator.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_bwd_params.h"
#include "attn_params.h"
#include "host_once.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kBwdThreads = 192;
constexpr int kBwdTmemCols = 512;
constexpr float kLog2eB = 1.44269504088896340736f;

template <int D>
struct BwdCfg {
  static constexpr int kQBufs = (D == 64) ? 2 : 1;   // buffers of Q, dO and row statistics
  static constexpr int kAtomBytes = 128 * 128;       // one 64-column atom of a 128-row tile
  static constexpr int kTileBytes = 128 * D * 2;     // one Q, K, V or dO tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;          // [kQBufs]
  static constexpr int kOffDO = kOffQ + kQBufs * kTileBytes;  // [kQBufs]
  static constexpr int kOffDS = kOffDO + kQBufs * kTileBytes;  // dS^T: [128 keys][128 queries] bf16
  // per buffer: -LSE2 [128], -D [128], qdoc [128], the tile's qdoc min and max, padding
  static constexpr int kStatWords = 400;
  static constexpr int kOffStat = kOffDS + 2 * kAtomBytes;     // [kQBufs] x kStatWords
  // dQ staging: 64 columns of fp32 as two 128-byte-swizzled boxes of 32 columns
  // by 128 rows, reduced into the accumulator by TMA (d = 128: two rounds)
  static constexpr int kOffStage = (kOffStat + kQBufs * kStatWords * 4 + 1023) / 1024 * 1024;
  static constexpr int kStageBoxBytes = 128 * 128;
  static constexpr int kOffBar = kOffStage + 2 * kStageBoxBytes;
  static constexpr int kNumBars = 12;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  // at least 120 KB, so one CTA per SM holds the whole tensor memory
  static constexpr int kSmemAlloc = (kSmemBytes + 1024 > 120 * 1024) ? kSmemBytes + 1024 : 120 * 1024;
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
  // tensor-memory columns (dQ: two 64-column halves for d = 128)
  static constexpr uint32_t kST = 0, kDPT = 128, kDV = 256, kDK = 256 + D;
  static constexpr uint32_t kDQ0 = (D == 64) ? 384u : 64u;
  static constexpr uint32_t kDQ1 = (D == 64) ? 416u : 192u;  // columns of d = 32.. or 64..
};

enum : int { kBarKv = 0, kBarQFull, kBarQFull1, kBarQEmpty, kBarQEmpty1, kBarSFull, kBarPFull,
             kBarDqFull, kBarDqFree, kBarAcc, kBarStageFull, kBarStageFree };
constexpr int kStageIssuer = 64;  // thread that issues the dQ reduce-adds (warp 2, lane 0)

__device__ __forceinline__ uint64_t bdesc(uint32_t addr, uint32_t lbo_bytes) {
  return ptx::smem_desc_sw128(addr, lbo_bytes, 1024);
}

// Query positions [qlo, qhi] that key j may be seen from, before the document
// test (every mask kind here gives an interval); hi < lo means none.
__device__ __forceinline__ void query_bounds(const BwdParams& p, int j, int& qlo, int& qhi) {
  const int off = p.Lk - p.Lq;  // query row i sits at position off + i
  long long lo = 0, hi = (long long)p.Lq - 1;
  if (p.mask_kind == kMaskCausal) {
    lo = max(lo, (long long)j - off);
  } else if (p.mask_kind == kMaskDraftBlock) {
    const long long bd = p.draft_block;
    lo = max(lo, (long long)(j / bd) * bd - off);
  }
  if (p.window_r >= 0) lo = max(lo, (long long)j - p.window_r - off);
  if (p.window_l >= 0) hi = min(hi, (long long)j + p.window_l - off);
  qlo = (int)max(-1LL, min(lo, (long long)p.Lq));
  qhi = (int)max(-2LL, min(hi, (long long)p.Lq - 1));
}

// Does the key tile [k0, k0+127] meet the query tile [q0, q0+127]?  (Before the
// document test, so a true answer may still have no visible pair.)
__device__ __forceinline__ bool pair_live(const BwdParams& p, int k0, int q0) {
  const int k_last = min(k0 + 127, p.Lk - 1);
  int lo_a, hi_a, lo_b, hi_b;
  query_bounds(p, k0, lo_a, hi_a);
  query_bounds(p, k_last, lo_b, hi_b);
  // the lower and upper bounds grow with the key index
  return !(lo_a > q0 + 127 || hi_b < q0 || lo_a > hi_b);
}

// dQ_tile = dS K over 128 keys: 8 MMAs, A = dS in shared memory (MN-major,
// 2048 bytes per 16 keys), B = K in shared memory (MN-major, same step).
__device__ __forceinline__ void mma_ss_chain8_mn(uint32_t d_tmem, uint64_t a_desc,
                                                 uint64_t b_desc, uint32_t idesc) {
  for (int kk = 0; kk < 8; ++kk)
    ptx::mma_ss_warp(d_tmem, a_desc + (uint64_t)(kk * 128), b_desc + (uint64_t)(kk * 128), idesc,
                     kk > 0 ? 1u : 0u);
}

}  // namespace

// D_i = sum_c dO_ic O_ic, one warp per query row.
template <int D>
__global__ void attn_bwd_dsum_kernel(const BwdParams p) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)p.B * p.Hq * p.Lq;
  if (row >= nrows) return;
  const __nv_bfloat16* o = reinterpret_cast<const __nv_bfloat16*>(p.o) + row * D;
  const __nv_bfloat16* g = reinterpret_cast<const __nv_bfloat16*>(p.dout) + row * D;
  float acc = 0.0f;
#pragma unroll
  for (int c = lane; c < D; c += 32) acc += __bfloat162float(o[c]) * __bfloat162float(g[c]);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) p.dsum[row] = acc;
}

// dQ (bf16) from its fp32 accumulator, four elements per thread (n4 = n / 4;
// n is a multiple of 64).
__global__ void attn_bwd_dq_kernel(const BwdParams p, long long n4) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(p.dq_acc)[i];
  uint2 out;
  out.x = ptx::pack_bf16x2(v.x, v.y);
  out.y = ptx::pack_bf16x2(v.z, v.w);
  reinterpret_cast<uint2*>(p.dq)[i] = out;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int QB = C::kQBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sk = ptx::smem_u32(smem + C::kOffK);
  const uint32_t sv = ptx::smem_u32(smem + C::kOffV);
  const uint32_t sq = ptx::smem_u32(smem + C::kOffQ);
  const uint32_t sdo = ptx::smem_u32(smem + C::kOffDO);
  const uint32_t sds = ptx::smem_u32(smem + C::kOffDS);
  const uint32_t sstage = ptx::smem_u32(smem + C::kOffStage);
  // row statistics of buffer slot: lse2 [128], dsum [128], qdoc [128]
  float* stat_s = reinterpret_cast<float*>(smem + C::kOffStat);
  const uint32_t bar0 = ptx::smem_u32(smem + C::kOffBar);
  auto BAR = [bar0](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* err = p.err;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // blockIdx.x: (b, kv head), fastest; blockIdx.y: key tile.  Blocks are
  // dispatched x-fastest, so every head's key tile 0 (the most query tiles
  // under a causal or draft mask) goes out first and the light last tiles
  // fill the tail.
  const int k0 = blockIdx.y * 128;
  const int b = blockIdx.x / p.Hkv;
  const int hkv = blockIdx.x % p.Hkv;
  const int n_iter = p.group * p.q_tiles;  // (query head of the group, query tile)

  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::prefetch_tmap(&tm_do);
    ptx::prefetch_tmap(&tm_dq);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    ptx::mbar_init(&bars[kBarKv], 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars[kBarQFull + i], 1);
      ptx::mbar_init(&bars[kBarQEmpty + i], 1);
    }
    ptx::mbar_init(&bars[kBarSFull], 1);
    ptx::mbar_init(&bars[kBarPFull], 128);
    ptx::mbar_init(&bars[kBarDqFull], 1);
    ptx::mbar_init(&bars[kBarDqFree], 128);
    ptx::mbar_init(&bars[kBarAcc], 1);
    ptx::mbar_init(&bars[kBarStageFull], 128);
    ptx::mbar_init(&bars[kBarStageFree], 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kBwdTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the live (query head, query tile) pairs of this key tile, in order
  auto iter_q0 = [&](int it) { return (it % p.q_tiles) * 128; };
  auto iter_hq = [&](int it) { return hkv * p.group + it / p.q_tiles; };

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    bool ok = true;
    constexpr uint32_t kTx = C::kTileBytes;
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx_a(BAR(kBarKv), 2 * kTx);
      for (int a = 0; a < D / 64; ++a) {
        ptx::tma_load_3d_a(sk + a * C::kAtomBytes, &tm_k, BAR(kBarKv), a * 64, k0, b * p.Hkv + hkv);
        ptx::tma_load_3d_a(sv + a * C::kAtomBytes, &tm_v, BAR(kBarKv), a * 64, k0, b * p.Hkv + hkv);
      }
    }
    // The row statistics of the next live query tile (this lane's rows r =
    // lane + 32 m) are loaded into registers while the producer waits for its
    // buffer, so the Q / dO loads go out as soon as the buffer is free.
    auto next_live = [&](int it) {
      while (it < n_iter && !pair_live(p, k0, iter_q0(it))) ++it;
      return it;
    };
    float f_nl2[4], f_nds[4];
    int f_doc[4];
    auto fetch = [&](int it) {
      const int q0 = iter_q0(it);
      const long long bh = (long long)b * p.Hq + iter_hq(it);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int qi = q0 + lane + 32 * m;
        f_nl2[m] = -INFINITY;
        f_nds[m] = 0.0f;
        f_doc[m] = 0;
        if (it < n_iter && qi < p.Lq) {
          const float lse = __ldg(p.lse + bh * p.Lq + qi);
          f_nl2[m] = (lse == -INFINITY) ? -INFINITY : -(lse * kLog2eB);
          f_nds[m] = -__ldg(p.dsum + bh * p.Lq + qi);
          if (p.doc_ids != nullptr)
            f_doc[m] = __ldg(p.doc_ids + (long long)b * p.Lk + (p.Lk - p.Lq + qi));
        }
      }
    };
    int n = 0;  // live pairs so far
    int it = next_live(0);
    fetch(it);
    while (it < n_iter && ok) {
      const int q0 = iter_q0(it);
      const int hq = iter_hq(it);
      const long long bh = (long long)b * p.Hq + hq;
      const int slot = n % QB;
      if (n >= QB) {  // the slot's previous tile has been used up
        ok = ptx::mbar_wait_a(BAR(kBarQEmpty + slot), (uint32_t)(n / QB - 1) & 1u, abort_flag, err,
                              kDevErrTimeoutProducer);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      if (lane == 0) {
        ptx::mbar_expect_tx_a(BAR(kBarQFull + slot), 2 * kTx);
        for (int a = 0; a < D / 64; ++a) {
          ptx::tma_load_3d_a(sq + slot * C::kTileBytes + a * C::kAtomBytes, &tm_q,
                             BAR(kBarQFull + slot), a * 64, q0, (int)bh);
          ptx::tma_load_3d_a(sdo + slot * C::kTileBytes + a * C::kAtomBytes, &tm_do,
                             BAR(kBarQFull + slot), a * 64, q0, (int)bh);
        }
      }
      // row statistics of the query tile, negated for the packed FMA and add of
      // the softmax warps: -LSE in base 2 (-inf for rows past Lq or with no
      // visible key, so their P is exactly 0), -D; the rows' documents and
      // their min / max over the tile
      float* nl2_s = stat_s + slot * C::kStatWords;
      float* nds_s = nl2_s + 128;
      int* qdoc_s = reinterpret_cast<int*>(nds_s + 128);
      int dmin = 0x7fffffff, dmax = (int)0x80000000;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int r = lane + 32 * m;
        nl2_s[r] = f_nl2[m];
        nds_s[r] = f_nds[m];
        qdoc_s[r] = f_doc[m];
        if (q0 + r < p.Lq) {
          dmin = min(dmin, f_doc[m]);
          dmax = max(dmax, f_doc[m]);
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        dmin = min(dmin, __shfl_xor_sync(0xffffffffu, dmin, o));
        dmax = max(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
      }
      if (lane == 0) {
        qdoc_s[128] = p.doc_ids != nullptr ? dmin : 0;
        qdoc_s[129] = p.doc_ids != nullptr ? dmax : 0;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_a(BAR(kBarQFull + slot));
      ++n;
      it = next_live(it + 1);
      fetch(it);  // in flight while the next buffer frees up
    }
    // drain: the last loads land before the CTA exits
    if (lane == 0) {
      int dummy = 0;
      ptx::mbar_wait_a(BAR(kBarKv), 0, &dummy, nullptr, 0);
      for (int jj = max(0, n - QB); jj < n; ++jj) {
        dummy = 0;
        ptx::mbar_wait_a(BAR(kBarQFull + jj % QB), (uint32_t)(jj / QB) & 1u, &dummy, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issue
    constexpr uint32_t kIdS = ptx::idesc_bf16_f32(128, 128, 0, 0);   // K-major A and B
    constexpr uint32_t kIdAcc = ptx::idesc_bf16_f32(128, D, 0, 1);   // A from TMEM, B MN-major
    constexpr uint32_t kIdDq = ptx::idesc_bf16_f32(128, 64, 1, 1);   // A and B MN-major, 64 of d
    bool ok = ptx::mbar_wait_a(BAR(kBarKv), 0, abort_flag, err, kDevErrTimeoutMma);
    ok = __all_sync(0xffffffffu, ok);
    int n = 0;
    for (int it = 0; it < n_iter && ok; ++it) {
      if (!pair_live(p, k0, iter_q0(it))) continue;
      const int slot = n % QB;
      const uint32_t sq_n = sq + slot * C::kTileBytes, sdo_n = sdo + slot * C::kTileBytes;
      ok = ptx::mbar_wait_a(BAR(kBarQFull + slot), (uint32_t)(n / QB) & 1u, abort_flag, err,
                            kDevErrTimeoutMma);
      // d = 128: the previous dQ tile lives in the upper halves of S^T and dP^T
      if (ok && D == 128 && n > 0)
        ok = ptx::mbar_wait_a(BAR(kBarDqFree), (uint32_t)(n - 1) & 1u, abort_flag, err,
                              kDevErrTimeoutMma);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      // S^T = K Q^T and dP^T = V dO^T (over P^T and dS^T of the previous tile,
      // which the previous dV and dK MMAs, issued before, have read)
      if constexpr (D == 64) {
        ptx::mma_qk_chain_d64(tmem + C::kST, bdesc(sk, 16), bdesc(sq_n, 16), kIdS);
        ptx::mma_qk_chain_d64(tmem + C::kDPT, bdesc(sv, 16), bdesc(sdo_n, 16), kIdS);
      } else {
        ptx::mma_qk_chain_d128(tmem + C::kST, bdesc(sk, 16), bdesc(sq_n, 16), kIdS);
        ptx::mma_qk_chain_d128(tmem + C::kDPT, bdesc(sv, 16), bdesc(sdo_n, 16), kIdS);
      }
      ptx::mma_commit_warp(BAR(kBarSFull));
      // P^T, dS^T written (tensor memory and shared memory)
      ok = ptx::mbar_wait_a(BAR(kBarPFull), (uint32_t)n & 1u, abort_flag, err, kDevErrTimeoutMma);
      if (ok && D == 64 && n > 0)  // the previous dQ tile has been read out
        ok = ptx::mbar_wait_a(BAR(kBarDqFree), (uint32_t)(n - 1) & 1u, abort_flag, err,
                              kDevErrTimeoutMma);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t acc = n > 0 ? 1u : 0u;
      ptx::mma_pv_chain8(tmem + C::kDV, tmem + C::kST, bdesc(sdo_n, C::kAtomBytes), kIdAcc, acc);
      ptx::mma_pv_chain8(tmem + C::kDK, tmem + C::kDPT, bdesc(sq_n, C::kAtomBytes), kIdAcc, acc);
      // dQ_tile = dS K, 64 columns of d per chain
      mma_ss_chain8_mn(tmem + C::kDQ0, bdesc(sds, C::kAtomBytes), bdesc(sk, C::kAtomBytes), kIdDq);
      if constexpr (D == 128)
        mma_ss_chain8_mn(tmem + C::kDQ1, bdesc(sds, C::kAtomBytes),
                         bdesc(sk + C::kAtomBytes, C::kAtomBytes), kIdDq);
      ptx::mma_commit_warp(BAR(kBarQEmpty + slot));
      ptx::mma_commit_warp(BAR(kBarDqFull));
      ++n;
    }
    ptx::mma_commit_warp(BAR(kBarAcc));
  } else {
    // ------------------------------------------------ P^T, dS^T and outputs
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;      // key of the tile (S^T lanes); query for dQ
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
    const int key = k0 + row;
    int qlo = 0, qhi = -1;
    if (key < p.Lk) query_bounds(p, key, qlo, qhi);
    const int kdoc = (p.doc_ids != nullptr && key < p.Lk)
                         ? __ldg(p.doc_ids + (long long)b * p.Lk + key) : 0;
    const float c = p.scale_log2;
    bool ok = true;
    int n = 0;
    for (int it = 0; it < n_iter && ok; ++it) {
      const int q0 = iter_q0(it);
      if (!pair_live(p, k0, q0)) continue;
      const int hq = iter_hq(it);
      const uint32_t stats = ptx::smem_u32(stat_s + (n % QB) * C::kStatWords);
      const int* qdoc_s = reinterpret_cast<const int*>(stat_s + (n % QB) * C::kStatWords + 256);
      ok = ptx::mbar_wait_a(BAR(kBarSFull), (uint32_t)n & 1u, abort_flag, err,
                            kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      // every key of the warp sees every query row of the tile: no mask code
      // (rows past Lq carry -LSE2 = -inf, so their P is 0 either way)
      bool sees_all = key < p.Lk && qlo <= q0 && qhi >= q0 + 127;
      if (p.doc_ids != nullptr) sees_all = sees_all && qdoc_s[128] == kdoc && qdoc_s[129] == kdoc;
      const bool full = __all_sync(0xffffffffu, sees_all);
      // 32 query columns at a time.  d = 128 loads the next chunk's scores from
      // tensor memory while this one is computed (the packed P^T / dS^T of
      // chunk cc land in columns [16 cc, 16 cc + 16), which no later chunk
      // still has to read); at d = 64 that measured 5 % slower, so each chunk
      // is loaded when its turn comes.
      constexpr bool kAhead = (D == 128);
      uint32_t sa[32], da[32], sb[32], db[32];  // sb, db only with kAhead
      ptx::tmem_ld32(t_row + C::kST, sa);
      ptx::tmem_ld32(t_row + C::kDPT, da);
#pragma unroll(kAhead ? 4 : 1)
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t(&rs)[32] = (kAhead && (cc & 1)) ? sb : sa;
        uint32_t(&rd)[32] = (kAhead && (cc & 1)) ? db : da;
        if (!kAhead && cc > 0) {
          ptx::tmem_ld32(t_row + C::kST + cc * 32, rs);
          ptx::tmem_ld32(t_row + C::kDPT + cc * 32, rd);
        }
        ptx::tmem_wait_ld();
        if (kAhead && cc + 1 < 4) {
          ptx::tmem_ld32(t_row + C::kST + (cc + 1) * 32, (kAhead && (cc & 1)) ? sa : sb);
          ptx::tmem_ld32(t_row + C::kDPT + (cc + 1) * 32, (kAhead && (cc & 1)) ? da : db);
        }
        float nl[32], nd[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t w0, w1, w2, w3;
          ptx::ld_shared_v4(stats + (uint32_t)(cc * 128 + j * 16), w0, w1, w2, w3);
          nl[4 * j] = __uint_as_float(w0);
          nl[4 * j + 1] = __uint_as_float(w1);
          nl[4 * j + 2] = __uint_as_float(w2);
          nl[4 * j + 3] = __uint_as_float(w3);
          ptx::ld_shared_v4(stats + (uint32_t)(512 + cc * 128 + j * 16), w0, w1, w2, w3);
          nd[4 * j] = __uint_as_float(w0);
          nd[4 * j + 1] = __uint_as_float(w1);
          nd[4 * j + 2] = __uint_as_float(w2);
          nd[4 * j + 3] = __uint_as_float(w3);
        }
        if (!full) {
          // masked: an invisible pair gets -LSE2 = -inf, so its P (and dS) is 0
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int qi = q0 + cc * 32 + i;
            bool vis = qi >= qlo && qi <= qhi;
            if (p.doc_ids != nullptr) vis = vis && (qdoc_s[cc * 32 + i] == kdoc);
            nl[i] = vis ? nl[i] : -INFINITY;
          }
        }
        uint32_t pp[16], dp[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          // P = 2^(S c - LSE2), dS = P (dP - D), two query columns per packed op
          float x0, x1, d0, d1;
          ptx::fma2_bv(x0, x1, __uint_as_float(rs[i]), __uint_as_float(rs[i + 1]), c, nl[i],
                       nl[i + 1]);
          const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
          ptx::addmul2(d0, d1, __uint_as_float(rd[i]), __uint_as_float(rd[i + 1]), nd[i],
                       nd[i + 1], p0, p1);
          pp[i / 2] = ptx::pack_bf16x2(p0, p1);
          dp[i / 2] = ptx::pack_bf16x2(d0, d1);
        }
        // P^T and dS^T over the columns already read (16 columns per 32 queries)
        ptx::tmem_st16(t_row + C::kST + cc * 16, pp);
        ptx::tmem_st16(t_row + C::kDPT + cc * 16, dp);
        // dS^T into shared memory as the MN-major A operand of dQ = dS K:
        // row = key, 64 queries per 128-byte row of a swizzle atom
        const uint32_t atom = sds + (uint32_t)((cc >> 1) * C::kAtomBytes) + (uint32_t)row * 128u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t chunk = (uint32_t)((cc & 1) * 4 + j);
          const uint32_t addr = atom + ((chunk ^ (uint32_t)(row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dp[4 * j]),
                       "r"(dp[4 * j + 1]), "r"(dp[4 * j + 2]), "r"(dp[4 * j + 3])
                       : "memory");
        }
      }
      ptx::tmem_wait_st();
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive_a(BAR(kBarPFull));
      // dQ tile: TMEM lane = query of the tile.  scale * dQ goes through a
      // 32 KB staging tile in shared memory (64 columns per round: one round
      // for d = 64, two for d = 128) and is added into the fp32 accumulator by
      // two TMA bulk reduce-adds per round, issued by one thread; the staging
      // tile is rewritten only after the previous round's reduce has read it.
      ok = ptx::mbar_wait_a(BAR(kBarDqFull), (uint32_t)n & 1u, abort_flag, err,
                            kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const long long bh = (long long)b * p.Hq + hq;
#pragma unroll 1
      for (int h = 0; h < D / 64 && ok; ++h) {
        const int g = n * (D / 64) + h;  // staging round
        if (g > 0) {
          if (threadIdx.x == kStageIssuer) {
            ptx::bulk_wait_group_read0();
            ptx::mbar_arrive_a(BAR(kBarStageFree));
          }
          ok = ptx::mbar_wait_a(BAR(kBarStageFree), (uint32_t)(g - 1) & 1u, abort_flag, err,
                                kDevErrTimeoutSoftmax);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        // the round's two 32-column blocks of d, both loads in flight at once
        uint32_t r[2][32];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const int cb = h * 2 + c2;  // 32-column block of d
          // columns of d [32 cb, 32 cb + 32): first and second 64-column half
          const uint32_t col = D == 64 ? C::kDQ0 + (uint32_t)(cb * 32)
                                       : (cb < 2 ? C::kDQ0 : C::kDQ1) + (uint32_t)((cb & 1) * 32);
          ptx::tmem_ld32(t_row + col, r[c2]);
        }
        ptx::tmem_wait_ld();
        if (h == D / 64 - 1) {  // the dQ columns are read out
          ptx::tc_fence_before();
          ptx::mbar_arrive_a(BAR(kBarDqFree));
        }
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const uint32_t rowp = sstage + (uint32_t)(c2 * C::kStageBoxBytes) + (uint32_t)row * 128u;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint32_t addr = rowp + (((uint32_t)ch ^ (uint32_t)(row & 7)) << 4);
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "f"(__uint_as_float(r[c2][4 * ch]) * p.scale),
                         "f"(__uint_as_float(r[c2][4 * ch + 1]) * p.scale),
                         "f"(__uint_as_float(r[c2][4 * ch + 2]) * p.scale),
                         "f"(__uint_as_float(r[c2][4 * ch + 3]) * p.scale)
                         : "memory");
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive_a(BAR(kBarStageFull));
        if (threadIdx.x == kStageIssuer) {
          ok = ptx::mbar_wait_a(BAR(kBarStageFull), (uint32_t)g & 1u, abort_flag, err,
                                kDevErrTimeoutSoftmax);
          if (ok) {
            // rows past Lq fall outside the map and are not written
            ptx::tma_reduce_add_3d(&tm_dq, sstage, h * 64, q0, (int)bh);
            ptx::tma_reduce_add_3d(&tm_dq, sstage + C::kStageBoxBytes, h * 64 + 32, q0, (int)bh);
            ptx::bulk_commit_group();
          }
        }
        ok = __all_sync(0xffffffffu, ok);
      }
      ++n;
    }
    // the last reduce-adds are complete before the CTA exits
    if (threadIdx.x == kStageIssuer) ptx::bulk_wait_group0();
    // dK (times scale) and dV of this key tile
    if (ok) {
      ok = ptx::mbar_wait_a(BAR(kBarAcc), 0, abort_flag, err, kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
    }
    ptx::tc_fence_after();
    // tcgen05.ld is warp-collective: every lane loads, only keys below Lk store
    const long long base = (((long long)b * p.Hkv + hkv) * p.Lk + key) * D;
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(which ? p.dv : p.dk) + base;
      const float f = which ? 1.0f : p.scale;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        if (ok && n > 0) {  // warp-uniform
          ptx::tmem_ld32(t_row + (which ? C::kDV : C::kDK) + cc * 32, r);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0u;
        }
        if (key < p.Lk) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v4;
            v4.x = ptx::pack_bf16x2(__uint_as_float(r[i]) * f, __uint_as_float(r[i + 1]) * f);
            v4.y = ptx::pack_bf16x2(__uint_as_float(r[i + 2]) * f, __uint_as_float(r[i + 3]) * f);
            v4.z = ptx::pack_bf16x2(__uint_as_float(r[i + 4]) * f, __uint_as_float(r[i + 5]) * f);
            v4.w = ptx::pack_bf16x2(__uint_as_float(r[i + 6]) * f, __uint_as_float(r[i + 7]) * f);
            *reinterpret_cast<uint4*>(out + cc * 32 + i) = v4;
          }
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kBwdTmemCols);
  }
}

// ---------------------------------------------------------------------------
// d = 64: the pipelined backward.  Tensor memory has room for P^T of its own
// ([448, 512)), and dK = dS^T Q reads dS^T from shared memory (the K-major
// reading of the tile the dQ MMA reads as MN-major), so the score columns are
// free as soon as the softmax warps have loaded them: S^T and dP^T of the next
// query tile are computed while the softmax warps still work on this one, and
// the gradient MMAs of this tile run while they start on the next.  448
// threads:
//   warp 0       TMA producer (Q, dO and row statistics in three buffers)
//   warp 1       MMA issue
//   warps 2-9    softmax, two warps per TMEM lane quarter, each taking 64 of
//                the 128 query columns of its keys: P^T to tensor memory,
//                dS^T to shared memory; at the end dK and dV (32 columns of d
//                each)
//   warps 10-13  dQ: read the dQ tile out of tensor memory into the staging
//                tile, which TMA bulk reduce-adds into the fp32 accumulator
namespace {

constexpr int kPipeThreads = 448;
constexpr int kPipeSmThreads = 256;  // softmax threads
constexpr int kPipeDqIssuer = 320;   // warp 10, lane 0

struct PipeCfg {
  static constexpr int kQBufs = 3;
  static constexpr int kAtomBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * 64 * 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;                  // [kQBufs]
  static constexpr int kOffDO = kOffQ + kQBufs * kTileBytes;        // [kQBufs]
  static constexpr int kOffDS = kOffDO + kQBufs * kTileBytes;       // dS^T [128 keys][128 queries]
  static constexpr int kOffStage = kOffDS + 2 * kAtomBytes;         // dQ staging, two boxes
  static constexpr int kStageBoxBytes = 128 * 128;
  static constexpr int kStatWords = 400;
  static constexpr int kOffStat = kOffStage + 2 * kStageBoxBytes;   // [kQBufs] x kStatWords
  static constexpr int kOffBar = kOffStat + kQBufs * kStatWords * 4;
  static constexpr int kNumBars = 16;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
  // tensor-memory columns
  static constexpr uint32_t kST = 0, kDPT = 128, kDV = 256, kDK = 320, kDQ = 384, kPT = 448;
};

enum : int { kPKv = 0, kPQFull = 1, kPQEmpty = 4, kPSFull = 7, kPSFree, kPPFull, kPGradDone,
             kPDqFree, kPAcc, kPStageFull, kPStageFree };

}  // namespace

__global__ void __launch_bounds__(kPipeThreads, 1)
    attn_bwd64_pipe_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using C = PipeCfg;
  constexpr int QB = C::kQBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sk = ptx::smem_u32(smem + C::kOffK);
  const uint32_t sv = ptx::smem_u32(smem + C::kOffV);
  const uint32_t sq = ptx::smem_u32(smem + C::kOffQ);
  const uint32_t sdo = ptx::smem_u32(smem + C::kOffDO);
  const uint32_t sds = ptx::smem_u32(smem + C::kOffDS);
  const uint32_t sstage = ptx::smem_u32(smem + C::kOffStage);
  float* stat_s = reinterpret_cast<float*>(smem + C::kOffStat);
  const uint32_t bar0 = ptx::smem_u32(smem + C::kOffBar);
  auto BAR = [bar0](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* err = p.err;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // blockIdx.x: (b, kv head), fastest; blockIdx.y: key tile (heaviest first)
  const int k0 = blockIdx.y * 128;
  const int b = blockIdx.x / p.Hkv;
  const int hkv = blockIdx.x % p.Hkv;
  const int n_iter = p.group * p.q_tiles;  // (query head of the group, query tile)

  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::prefetch_tmap(&tm_do);
    ptx::prefetch_tmap(&tm_dq);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    ptx::mbar_init(&bars[kPKv], 1);
    for (int i = 0; i < QB; ++i) {
      ptx::mbar_init(&bars[kPQFull + i], 1);
      ptx::mbar_init(&bars[kPQEmpty + i], 1);
    }
    ptx::mbar_init(&bars[kPSFull], 1);
    ptx::mbar_init(&bars[kPSFree], kPipeSmThreads);
    ptx::mbar_init(&bars[kPPFull], kPipeSmThreads);
    ptx::mbar_init(&bars[kPGradDone], 1);
    ptx::mbar_init(&bars[kPDqFree], 128);
    ptx::mbar_init(&bars[kPAcc], 1);
    ptx::mbar_init(&bars[kPStageFull], 128);
    ptx::mbar_init(&bars[kPStageFree], 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kBwdTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto iter_q0 = [&](int it) { return (it % p.q_tiles) * 128; };
  auto iter_hq = [&](int it) { return hkv * p.group + it / p.q_tiles; };
  auto next_live = [&](int it) {
    while (it < n_iter && !pair_live(p, k0, iter_q0(it))) ++it;
    return it;
  };

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    bool ok = true;
    constexpr uint32_t kTx = C::kTileBytes;
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx_a(BAR(kPKv), 2 * kTx);
      ptx::tma_load_3d_a(sk, &tm_k, BAR(kPKv), 0, k0, b * p.Hkv + hkv);
      ptx::tma_load_3d_a(sv, &tm_v, BAR(kPKv), 0, k0, b * p.Hkv + hkv);
    }
    float f_nl2[4], f_nds[4];
    int f_doc[4];
    auto fetch = [&](int it) {
      const int q0 = iter_q0(it);
      const long long bh = (long long)b * p.Hq + iter_hq(it);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int qi = q0 + lane + 32 * m;
        f_nl2[m] = -INFINITY;
        f_nds[m] = 0.0f;
        f_doc[m] = 0;
        if (it < n_iter && qi < p.Lq) {
          const float lse = __ldg(p.lse + bh * p.Lq + qi);
          f_nl2[m] = (lse == -INFINITY) ? -INFINITY : -(lse * kLog2eB);
          f_nds[m] = -__ldg(p.dsum + bh * p.Lq + qi);
          if (p.doc_ids != nullptr)
            f_doc[m] = __ldg(p.doc_ids + (long long)b * p.Lk + (p.Lk - p.Lq + qi));
        }
      }
    };
    int n = 0;
    int it = next_live(0);
    fetch(it);
    while (it < n_iter && ok) {
      const int q0 = iter_q0(it);
      const long long bh = (long long)b * p.Hq + iter_hq(it);
      const int slot = n % QB;
      if (n >= QB) {
        ok = ptx::mbar_wait_a(BAR(kPQEmpty + slot), (uint32_t)(n / QB - 1) & 1u, abort_flag, err,
                              kDevErrTimeoutProducer);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      if (lane == 0) {
        ptx::mbar_expect_tx_a(BAR(kPQFull + slot), 2 * kTx);
        ptx::tma_load_3d_a(sq + slot * C::kTileBytes, &tm_q, BAR(kPQFull + slot), 0, q0, (int)bh);
        ptx::tma_load_3d_a(sdo + slot * C::kTileBytes, &tm_do, BAR(kPQFull + slot), 0, q0,
                           (int)bh);
      }
      float* nl2_s = stat_s + slot * C::kStatWords;
      float* nds_s = nl2_s + 128;
      int* qdoc_s = reinterpret_cast<int*>(nds_s + 128);
      int dmin = 0x7fffffff, dmax = (int)0x80000000;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int r = lane + 32 * m;
        nl2_s[r] = f_nl2[m];
        nds_s[r] = f_nds[m];
        qdoc_s[r] = f_doc[m];
        if (q0 + r < p.Lq) {
          dmin = min(dmin, f_doc[m]);
          dmax = max(dmax, f_doc[m]);
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        dmin = min(dmin, __shfl_xor_sync(0xffffffffu, dmin, o));
        dmax = max(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
      }
      if (lane == 0) {
        qdoc_s[128] = p.doc_ids != nullptr ? dmin : 0;
        qdoc_s[129] = p.doc_ids != nullptr ? dmax : 0;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_a(BAR(kPQFull + slot));
      ++n;
      it = next_live(it + 1);
      fetch(it);
    }
    if (lane == 0) {
      int dummy = 0;
      ptx::mbar_wait_a(BAR(kPKv), 0, &dummy, nullptr, 0);
      for (int jj = max(0, n - QB); jj < n; ++jj) {
        dummy = 0;
        ptx::mbar_wait_a(BAR(kPQFull + jj % QB), (uint32_t)(jj / QB) & 1u, &dummy, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issue
    constexpr uint32_t kIdS = ptx::idesc_bf16_f32(128, 128, 0, 0);   // K-major A and B
    constexpr uint32_t kIdAcc = ptx::idesc_bf16_f32(128, 64, 0, 1);  // A K-major / TMEM, B MN
    constexpr uint32_t kIdDq = ptx::idesc_bf16_f32(128, 64, 1, 1);   // A and B MN-major
    bool ok = ptx::mbar_wait_a(BAR(kPKv), 0, abort_flag, err, kDevErrTimeoutMma);
    ok = __all_sync(0xffffffffu, ok);
    int it = next_live(0);
    auto issue_scores = [&](int n) -> bool {
      const int slot = n % QB;
      bool good = ptx::mbar_wait_a(BAR(kPQFull + slot), (uint32_t)(n / QB) & 1u, abort_flag, err,
                                   kDevErrTimeoutMma);
      good = __all_sync(0xffffffffu, good);
      if (!good) return false;
      ptx::tc_fence_after();
      ptx::mma_qk_chain_d64(tmem + C::kST, bdesc(sk, 16), bdesc(sq + slot * C::kTileBytes, 16),
                            kIdS);
      ptx::mma_qk_chain_d64(tmem + C::kDPT, bdesc(sv, 16), bdesc(sdo + slot * C::kTileBytes, 16),
                            kIdS);
      ptx::mma_commit_warp(BAR(kPSFull));
      return true;
    };
    if (ok && it < n_iter) ok = issue_scores(0);
    int n = 0;
    while (ok && it < n_iter) {
      const int it_next = next_live(it + 1);
      const int slot = n % QB;
      const uint32_t sq_n = sq + slot * C::kTileBytes, sdo_n = sdo + slot * C::kTileBytes;
      if (it_next < n_iter) {
        // the next tile's scores, once the softmax warps hold this tile's in registers
        ok = ptx::mbar_wait_a(BAR(kPSFree), (uint32_t)n & 1u, abort_flag, err, kDevErrTimeoutMma);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
        ok = issue_scores(n + 1);
        if (!ok) break;
      }
      ok = ptx::mbar_wait_a(BAR(kPPFull), (uint32_t)n & 1u, abort_flag, err, kDevErrTimeoutMma);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t acc = n > 0 ? 1u : 0u;
      // dV += P^T dO (P^T from tensor memory)
      ptx::mma_pv_chain8(tmem + C::kDV, tmem + C::kPT, bdesc(sdo_n, C::kAtomBytes), kIdAcc, acc);
      // dK += dS^T Q (dS^T K-major from shared memory: 64 queries per atom)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        ptx::mma_ss_warp(tmem + C::kDK,
                         bdesc(sds + (uint32_t)((kk >> 2) * C::kAtomBytes + (kk & 3) * 32), 16),
                         bdesc(sq_n + (uint32_t)(kk * 2048), C::kAtomBytes), kIdAcc,
                         (n > 0 || kk > 0) ? 1u : 0u);
      if (n > 0) {  // the previous dQ tile has been read out
        ok = ptx::mbar_wait_a(BAR(kPDqFree), (uint32_t)(n - 1) & 1u, abort_flag, err,
                              kDevErrTimeoutMma);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
      }
      // dQ_tile = dS K
      mma_ss_chain8_mn(tmem + C::kDQ, bdesc(sds, C::kAtomBytes), bdesc(sk, C::kAtomBytes), kIdDq);
      ptx::mma_commit_warp(BAR(kPQEmpty + slot));
      ptx::mma_commit_warp(BAR(kPGradDone));
      ++n;
      it = it_next;
    }
    ptx::mma_commit_warp(BAR(kPAcc));
  } else if (warp < 10) {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;        // query columns [64 half, 64 half + 64)
    const int row = quarter * 32 + lane;     // key of the tile (TMEM lane)
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
    const int key = k0 + row;
    int qlo = 0, qhi = -1;
    if (key < p.Lk) query_bounds(p, key, qlo, qhi);
    const int kdoc = (p.doc_ids != nullptr && key < p.Lk)
                         ? __ldg(p.doc_ids + (long long)b * p.Lk + key) : 0;
    const float c = p.scale_log2;
    bool ok = true;
    int n = 0;
    for (int it = next_live(0); it < n_iter && ok; it = next_live(it + 1)) {
      const int q0 = iter_q0(it);
      const uint32_t stats = ptx::smem_u32(stat_s + (n % QB) * C::kStatWords);
      const int* qdoc_s = reinterpret_cast<const int*>(stat_s + (n % QB) * C::kStatWords + 256);
      ok = ptx::mbar_wait_a(BAR(kPSFull), (uint32_t)n & 1u, abort_flag, err,
                            kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      bool sees_all = key < p.Lk && qlo <= q0 && qhi >= q0 + 127;
      if (p.doc_ids != nullptr) sees_all = sees_all && qdoc_s[128] == kdoc && qdoc_s[129] == kdoc;
      const bool full = __all_sync(0xffffffffu, sees_all);
#pragma unroll 1
      for (int j = 0; j < 2 && ok; ++j) {
        const int cc = 2 * half + j;  // 32 query columns
        uint32_t rs[32], rd[32];
        ptx::tmem_ld32(t_row + C::kST + cc * 32, rs);
        ptx::tmem_ld32(t_row + C::kDPT + cc * 32, rd);
        ptx::tmem_wait_ld();
        if (j == 1) {  // every score column of this tile is in registers
          ptx::tc_fence_before();
          ptx::mbar_arrive_a(BAR(kPSFree));
        }
        uint32_t pp[16], dp[16];
#pragma unroll
        for (int g4 = 0; g4 < 8; ++g4) {  // four query columns per step
          uint32_t w0, w1, w2, w3;
          float nl[4], nd[4];
          ptx::ld_shared_v4(stats + (uint32_t)(cc * 128 + g4 * 16), w0, w1, w2, w3);
          nl[0] = __uint_as_float(w0);
          nl[1] = __uint_as_float(w1);
          nl[2] = __uint_as_float(w2);
          nl[3] = __uint_as_float(w3);
          ptx::ld_shared_v4(stats + (uint32_t)(512 + cc * 128 + g4 * 16), w0, w1, w2, w3);
          nd[0] = __uint_as_float(w0);
          nd[1] = __uint_as_float(w1);
          nd[2] = __uint_as_float(w2);
          nd[3] = __uint_as_float(w3);
          if (!full) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int col = cc * 32 + 4 * g4 + i;
              bool vis = q0 + col >= qlo && q0 + col <= qhi;
              if (p.doc_ids != nullptr) vis = vis && (qdoc_s[col] == kdoc);
              nl[i] = vis ? nl[i] : -INFINITY;
            }
          }
#pragma unroll
          for (int i = 0; i < 4; i += 2) {
            const int e = 4 * g4 + i;
            float x0, x1, d0, d1;
            ptx::fma2_bv(x0, x1, __uint_as_float(rs[e]), __uint_as_float(rs[e + 1]), c, nl[i],
                         nl[i + 1]);
            const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
            ptx::addmul2(d0, d1, __uint_as_float(rd[e]), __uint_as_float(rd[e + 1]), nd[i],
                         nd[i + 1], p0, p1);
            pp[e / 2] = ptx::pack_bf16x2(p0, p1);
            dp[e / 2] = ptx::pack_bf16x2(d0, d1);
          }
        }
        if (j == 0 && n > 0) {  // P^T and dS^T of the previous tile have been used
          ok = ptx::mbar_wait_a(BAR(kPGradDone), (uint32_t)(n - 1) & 1u, abort_flag, err,
                                kDevErrTimeoutSoftmax);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ptx::tc_fence_after();
        }
        ptx::tmem_st16(t_row + C::kPT + cc * 16, pp);
        const uint32_t atom = sds + (uint32_t)((cc >> 1) * C::kAtomBytes) + (uint32_t)row * 128u;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t chunk = (uint32_t)((cc & 1) * 4 + q4);
          const uint32_t addr = atom + ((chunk ^ (uint32_t)(row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dp[4 * q4]),
                       "r"(dp[4 * q4 + 1]), "r"(dp[4 * q4 + 2]), "r"(dp[4 * q4 + 3])
                       : "memory");
        }
      }
      if (!ok) break;
      ptx::tmem_wait_st();
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive_a(BAR(kPPFull));
      ++n;
    }
    // dK (times scale) and dV: 32 columns of d per half
    if (ok) {
      ok = ptx::mbar_wait_a(BAR(kPAcc), 0, abort_flag, err, kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
    }
    ptx::tc_fence_after();
    const long long base = (((long long)b * p.Hkv + hkv) * p.Lk + key) * 64 + half * 32;
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(which ? p.dv : p.dk) + base;
      const float f = which ? 1.0f : p.scale;
      uint32_t r[32];
      if (ok && n > 0) {  // warp-uniform
        ptx::tmem_ld32(t_row + (which ? C::kDV : C::kDK) + (uint32_t)(half * 32), r);
        ptx::tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      if (key < p.Lk) {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint4 v4;
          v4.x = ptx::pack_bf16x2(__uint_as_float(r[i]) * f, __uint_as_float(r[i + 1]) * f);
          v4.y = ptx::pack_bf16x2(__uint_as_float(r[i + 2]) * f, __uint_as_float(r[i + 3]) * f);
          v4.z = ptx::pack_bf16x2(__uint_as_float(r[i + 4]) * f, __uint_as_float(r[i + 5]) * f);
          v4.w = ptx::pack_bf16x2(__uint_as_float(r[i + 6]) * f, __uint_as_float(r[i + 7]) * f);
          *reinterpret_cast<uint4*>(out + i) = v4;
        }
      }
    }
  } else {
    // ----------------------------------------------------------------- dQ
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query of the tile (TMEM lane)
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    int n = 0;
    for (int it = next_live(0); it < n_iter && ok; it = next_live(it + 1)) {
      const int q0 = iter_q0(it);
      const long long bh = (long long)b * p.Hq + iter_hq(it);
      ok = ptx::mbar_wait_a(BAR(kPGradDone), (uint32_t)n & 1u, abort_flag, err,
                            kDevErrTimeoutSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      if (n > 0) {  // the staging tile has been read by the previous reduce
        if (threadIdx.x == kPipeDqIssuer) {
          ptx::bulk_wait_group_read0();
          ptx::mbar_arrive_a(BAR(kPStageFree));
        }
        ok = ptx::mbar_wait_a(BAR(kPStageFree), (uint32_t)(n - 1) & 1u, abort_flag, err,
                              kDevErrTimeoutSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      uint32_t r[2][32];
      ptx::tmem_ld32(t_row + C::kDQ, r[0]);
      ptx::tmem_ld32(t_row + C::kDQ + 32, r[1]);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive_a(BAR(kPDqFree));
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        const uint32_t rowp = sstage + (uint32_t)(c2 * C::kStageBoxBytes) + (uint32_t)row * 128u;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t addr = rowp + (((uint32_t)ch ^ (uint32_t)(row & 7)) << 4);
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                       "f"(__uint_as_float(r[c2][4 * ch]) * p.scale),
                       "f"(__uint_as_float(r[c2][4 * ch + 1]) * p.scale),
                       "f"(__uint_as_float(r[c2][4 * ch + 2]) * p.scale),
                       "f"(__uint_as_float(r[c2][4 * ch + 3]) * p.scale)
                       : "memory");
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive_a(BAR(kPStageFull));
      if (threadIdx.x == kPipeDqIssuer) {
        ok = ptx::mbar_wait_a(BAR(kPStageFull), (uint32_t)n & 1u, abort_flag, err,
                              kDevErrTimeoutSoftmax);
        if (ok) {
          ptx::tma_reduce_add_3d(&tm_dq, sstage, 0, q0, (int)bh);
          ptx::tma_reduce_add_3d(&tm_dq, sstage + C::kStageBoxBytes, 32, q0, (int)bh);
          ptx::bulk_commit_group();
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      ++n;
    }
    if (threadIdx.x == kPipeDqIssuer) ptx::bulk_wait_group0();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kBwdTmemCols);
  }
}

// The three launches of the backward: D_i, the main kernel, dQ to bf16.  The
// caller zeroes dq_acc before (on the same stream).
template <int D>
cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdParams& p,
                            cudaStream_t stream) {
  const long long nrows = (long long)p.B * p.Hq * p.Lq;
  attn_bwd_dsum_kernel<D><<<(unsigned)((nrows + 7) / 8), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)(p.B * p.Hkv), (unsigned)((p.Lk + 127) / 128), 1);
  if constexpr (D == 64) {
    constexpr int smem = PipeCfg::kSmemAlloc;
    static PerContextOnce once;
    e = once_per_context(once, [&](int) {
      return cudaFuncSetAttribute(attn_bwd64_pipe_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (e != cudaSuccess) return e;
    attn_bwd64_pipe_kernel<<<grid, kPipeThreads, smem, stream>>>(tq, tk, tv, tdo, tdq, p);
  } else {
    auto kern = attn_bwd_kernel<D>;
    constexpr int smem = BwdCfg<D>::kSmemAlloc;
    static PerContextOnce once;
    e = once_per_context(once, [&](int) {
      return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (e != cudaSuccess) return e;
    kern<<<grid, kBwdThreads, smem, stream>>>(tq, tk, tv, tdo, tdq, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long n4 = nrows * D / 4;
  attn_bwd_dq_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, stream>>>(p, n4);
  return cudaGetLastError();
}

template cudaError_t launch_backward<64>(const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const BwdParams&, cudaStream_t);
template cudaError_t launch_backward<128>(const CUtensorMap&, const CUtensorMap&,
                                          const CUtensorMap&, const CUtensorMap&,
                                          const CUtensorMap&, const BwdParams&, cudaStream_t);

}  // namespace attn
