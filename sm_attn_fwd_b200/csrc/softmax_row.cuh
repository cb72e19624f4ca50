// Row-wise softmax pieces shared by the split-KV decode and the short-query
// kernel: one thread owns one query row (its tensor-memory lane) of a 128-key
// tile of S, as in the online softmax of "FlashAttention 2 原理与 PyTorch 实战"
// (sections 3.1, 3.2): load the row's scores, apply the score modifier, and
// turn them into P = 2^(s*c - m) as packed bf16 pairs with their fp32 sum.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace attn {
namespace row {

// Score modifiers ("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 1:
// score_mod(score, b, h, q_idx, kv_idx), with ALiBi, a position bias and a
// learnable bias as examples); p is the query row's absolute position.
enum ScoreMod : int {
  kModNone = 0,
  kModAlibi = 1,    // S_ij += slope_h * (j - p)
  kModRelBias = 2,  // S_ij += table_h[clamp(j - p, -R, R) + R]
};

constexpr float kLog2e = 1.44269504088896340736f;

// The 128 fp32 columns [taddr, taddr + 128) of this thread's tensor-memory lane
// (32x32b shape): all four 32-column loads in flight, one wait.
__device__ __forceinline__ void tmem_ld_row128(uint32_t taddr, float (&s)[128]) {
  uint32_t r0[32], r1[32], r2[32], r3[32];
  ptx::tmem_ld32(taddr + 0, r0);
  ptx::tmem_ld32(taddr + 32, r1);
  ptx::tmem_ld32(taddr + 64, r2);
  ptx::tmem_ld32(taddr + 96, r3);
  ptx::tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    s[i] = __uint_as_float(r0[i]);
    s[32 + i] = __uint_as_float(r1[i]);
    s[64 + i] = __uint_as_float(r2[i]);
    s[96 + i] = __uint_as_float(r3[i]);
  }
}

// The raw scores of one 128-key tile (keys j = k0 + i) to the base-2 domain
// with the score modifier: s_i <- s_i * c + bias(j - p) * log2(e), given
// dj0 = k0 - p.  Masked scores (-inf) stay -inf.
//   ALiBi (alibi2 = slope * log2(e)): the bias of key pair i comes from one of
//   eight chains of packed fp32x2 adds that step 16 keys, each starting from
//   alibi2 * dj0 (exact in fp32 while |dj0| < 2^24): one packed add and one
//   packed FMA per pair.
//   Relative-position table (rel_row points at the head's entry for j - p = 0):
//   a tile whose keys all lie R or more from p on one side takes one clamped
//   value; only tiles within R of p look each key up.
template <int kMod>
__device__ __forceinline__ void score_mod128(float (&s)[128], float c, int dj0, float alibi2,
                                             const float* rel_row, int R) {
  if constexpr (kMod == kModAlibi) {
    const float base = alibi2 * (float)dj0;
    const float step = alibi2 * 16.0f;
    float b0[8], b1[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      b0[k] = fmaf(alibi2, (float)(2 * k), base);
      b1[k] = fmaf(alibi2, (float)(2 * k + 1), base);
    }
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const int k = i & 7;
      ptx::fma2_bv(s[2 * i], s[2 * i + 1], s[2 * i], s[2 * i + 1], c, b0[k], b1[k]);
      if (i + 8 < 64) ptx::add2_acc(b0[k], b1[k], step, step);
    }
  } else if constexpr (kMod == kModRelBias) {
    if (dj0 + 127 <= -R || dj0 >= R) {
      const float bias = __ldg(rel_row + (dj0 >= R ? R : -R)) * kLog2e;
#pragma unroll
      for (int i = 0; i < 64; ++i)
        ptx::fma2_bc(s[2 * i], s[2 * i + 1], s[2 * i], s[2 * i + 1], c, bias);
    } else {
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        const int delta = min(max(dj0 + i, -R), R);
        s[i] = fmaf(__ldg(rel_row + delta), kLog2e, s[i] * c);
      }
    }
  }
}

// One row of P = 2^(s_i * c - m), i = 0..127, as 64 packed bf16 pairs (key 2i in
// the low half; pairs 0..31 in lo, 32..63 in hi); returns the fp32 sum of the
// unrounded values.  s * c - m is one packed fp32x2 FMA per pair; each pair's
// exponentials are issued four pairs before the sum and packing that read them,
// so the MUFU results are ready when needed; the sum runs in four packed chains.
__device__ __forceinline__ float exp2_pack128(const float (&s)[128], float c, float m,
                                              uint32_t (&lo)[32], uint32_t (&hi)[32]) {
  constexpr int kAhead = 4;
  float e0[kAhead], e1[kAhead];
  float sum8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) sum8[k] = 0.0f;
#pragma unroll
  for (int i = 0; i < 64 + kAhead; ++i) {
    if (i >= kAhead) {
      const int j = i - kAhead;
      const float p0 = e0[j % kAhead], p1 = e1[j % kAhead];
      ptx::add2_acc(sum8[(j & 3) * 2], sum8[(j & 3) * 2 + 1], p0, p1);
      const uint32_t packed = ptx::pack_bf16x2(p0, p1);
      if (j < 32) lo[j] = packed;
      else hi[j - 32] = packed;
    }
    if (i < 64) {
      float a0, a1;
      ptx::fma2_bc(a0, a1, s[2 * i], s[2 * i + 1], c, -m);
      e0[i % kAhead] = ptx::ex2(a0);
      e1[i % kAhead] = ptx::ex2(a1);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) sum8[k] += sum8[k + 4];
  return (sum8[0] + sum8[1]) + (sum8[2] + sum8[3]);
}

}  // namespace row
}  // namespace attn
