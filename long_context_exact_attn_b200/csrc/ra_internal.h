// Internal interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "../../include/ringattn.h"

namespace ra {

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, looked up once (NULL on failure).
PFN_encodeTiled get_encode_tiled();

struct AttnLaunch {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int64_t BH, N, d;
  int P;
  int striped, causal, sched_free;
  float scale;
  int device, num_sms;
  void* stream;
  int blk_j = -1, blk_kb = -1;   // single-block mode when blk_kb >= 0 (P = 1)
  int zigzag = 0;                // zigzag layout (striped == 0)
  int o_f32 = 0;                 // write O as float32
  int tok = 0;                   // q, k, v, o, lse in token order
  int pair = 0;                  // the CTA-pair (two-SM MMA) kernel where it applies
  int64_t main_limit_ns = 0;     // > 0: limit of the main-loop waits (abort self-test)
  int withhold_first_s = 0;      // abort self-test: first S-ready signal never sent
};

ra_status attn_fwd_launch(const AttnLaunch& a);

ra_status read_device_fault(int* code);
unsigned int* device_fault_word();

// Phase profile of the forward kernel (profiling build only): counters per
// CTA (the first kProfCtas), role slot (softmax warps 0-7, MMA warp 8, one
// spare) and phase (the last phase counts tiles).
constexpr int kProfCtas = 160, kProfSlots = 10, kProfPhases = 8;
ra_status fwd_profile_read(unsigned long long* host, int64_t capacity);
ra_status wait_selftest_launch(int64_t limit_ns, void* stream);

ra_status partition_launch(const void* src, void* dst, int64_t rows_outer, int64_t N, int64_t P,
                           int64_t row_bytes, int layout, int inverse, void* stream);

ra_status partition_rope_launch(const void* src, void* dst, int64_t BH, int64_t N, int64_t P,
                                int64_t d, int layout, int half, double log2_base, int num_sms,
                                void* stream);
ra_status lse_merge_acc_launch(float* o_acc, float* lse_acc, const void* o_b,
                               const float* lse_b, void* o_final, int64_t rows, int64_t d,
                               int first, int final_, int b_f32, void* stream);
ra_status fill_f32_launch(float* dst, int64_t n, float value, void* stream);
ra_status lse_merge_launch(const void* o_a, const float* lse_a, const void* o_b,
                           const float* lse_b, void* o_out, float* lse_out, int64_t rows,
                           int64_t d, int num_sms, void* stream);

ra_status tile_census_launch(int64_t N, int P, int striped, int causal, int64_t* out,
                             void* stream);

}  // namespace ra
