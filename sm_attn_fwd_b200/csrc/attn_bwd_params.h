// Launch parameters of the backward pass, shared by the host code and the kernels.
#pragma once

#include <cstdint>

#include "attn_params.h"

namespace attn {

// Backward pass (dQ, dK, dV) of the prefill forward, [B, H, L, d] layout.
struct BwdParams {
  const void* o;        // bf16 [B, Hq, Lq, d], forward output
  const float* lse;     // fp32 [B, Hq, Lq], forward log-sum-exp (natural log)
  const void* dout;     // bf16 [B, Hq, Lq, d]
  void* dk;             // bf16 [B, Hkv, Lk, d], written
  void* dv;             // bf16 [B, Hkv, Lk, d], written
  void* dq;             // bf16 [B, Hq, Lq, d], written by the last kernel
  float* dq_acc;        // fp32 [B, Hq, Lq, d] workspace (zeroed, then reduced into)
  float* dsum;          // fp32 [B, Hq, Lq] workspace: D_i = sum_c dO_ic O_ic
  const int32_t* doc_ids;  // [B, Lk] or null
  int B, Hq, Hkv, Lq, Lk, group;
  int mask_kind, window_l, window_r, draft_block;
  float scale;          // softmax scale
  float scale_log2;     // scale * log2(e)
  int q_tiles;          // ceil(Lq / 128)
  int* err;             // device error word
};

}  // namespace attn
