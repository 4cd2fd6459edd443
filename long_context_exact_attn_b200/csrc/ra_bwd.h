// Internal declarations of the backward pass (kept apart from ra_internal.h
// so that the forward kernel's sources do not change with the backward's).
#pragma once

#include "ra_internal.h"

namespace ra {

struct BwdLaunch {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* workspace;
  int64_t BH, N, d;
  int P;
  int striped, causal;
  float scale;
  int device, num_sms;
  void* stream;
  int zigzag = 0;                // zigzag layout (striped == 0)
  int tok = 0;                   // all tensors in token order
};

ra_status attn_bwd_launch(const BwdLaunch& a);

// Capacity (floats) of the fixed scratch used by ra_attn_bwd_noalloc.
constexpr long long kNoAllocScratchFloats = 1LL << 20;
ra_status attn_bwd_noalloc_launch(BwdLaunch a);

}  // namespace ra
