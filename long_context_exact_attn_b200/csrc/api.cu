// C-ABI entry points of libringattn.so: host-side validation, then a launch
// on the caller's stream.  Declarations and contracts: include/ringattn.h.
#include <cmath>
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "ra_internal.h"
#include "ra_bwd.h"

namespace ra {

PFN_encodeTiled get_encode_tiled() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

namespace {

struct DevInfo {
  int ok;
  int num_sms;
};

// Current device, checked to be sm_100 (B200 class); SM count cached.
ra_status current_device(int* dev, DevInfo* info) {
  static DevInfo cache[64];
  static int cached[64] = {0};
  static std::mutex mu;
  if (cudaGetDevice(dev) != cudaSuccess) return RA_ERR_CUDA;
  if (*dev < 0 || *dev >= 64) return RA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[*dev]) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
      return RA_ERR_CUDA;
    cache[*dev].ok = (major == 10 && minor == 0);
    cache[*dev].num_sms = sms;
    cached[*dev] = 1;
  }
  *info = cache[*dev];
  return info->ok ? RA_OK : RA_ERR_DEVICE;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// a * b * c < 2^31 for positive factors, decided without overflowing int64
// (each factor and the partial product are bounded before the next multiply).
bool rows_fit(int64_t a, int64_t b, int64_t c) {
  const int64_t lim = (int64_t)1 << 31;
  return a < lim && b < lim && c < lim && a * b < lim && a * b * c < lim;
}

bool overlap(const void* a, int64_t na, const void* b, int64_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + (uintptr_t)nb && y < x + (uintptr_t)na;
}

// ------------------------------------------------------------ host path
// Device staging of ra_attn_fwd_host: two slots, each holding a chunk of G
// heads: q, k, v, o and lse, all in token order (the attention applies the
// layout's permutation in its own addressing).
struct HostPlan {
  int64_t tok;      // bytes of one [N, d] bf16 head
  int64_t lsz;      // bytes of one [N] float32 head
  int64_t per_head; // staging bytes per head per slot (256-byte rounded parts)
};

int64_t round256(int64_t x) { return (x + 255) / 256 * 256; }

HostPlan host_plan(int64_t N, int64_t d) {
  HostPlan h;
  h.tok = N * d * 2;
  h.lsz = N * 4;
  h.per_head = 4 * round256(h.tok) + round256(h.lsz);
  return h;
}

struct HostStreams {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t entry = nullptr, end = nullptr, h2d[2] = {}, comp[2] = {}, d2h[2] = {};
  bool ready = false;
};

// Copy streams and events per device, created on first use (no device
// memory); every call on a device holds the device's lock while enqueuing.
ra_status host_streams(int dev, HostStreams** out, std::mutex** mu) {
  static HostStreams hs[64];
  static std::mutex mus[64];
  *mu = &mus[dev];
  std::lock_guard<std::mutex> lock(mus[dev]);
  HostStreams& h = hs[dev];
  if (!h.ready) {
    const unsigned ef = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&h.entry, ef) != cudaSuccess ||
        cudaEventCreateWithFlags(&h.end, ef) != cudaSuccess)
      return RA_ERR_CUDA;
    for (int s = 0; s < 2; ++s)
      if (cudaEventCreateWithFlags(&h.h2d[s], ef) != cudaSuccess ||
          cudaEventCreateWithFlags(&h.comp[s], ef) != cudaSuccess ||
          cudaEventCreateWithFlags(&h.d2h[s], ef) != cudaSuccess)
        return RA_ERR_CUDA;
    h.ready = true;
  }
  *out = &h;
  return RA_OK;
}

}  // namespace
}  // namespace ra

using namespace ra;

extern "C" {

const char* ra_status_string(ra_status s) {
  switch (s) {
    case RA_OK: return "ok";
    case RA_ERR_NULL: return "a required pointer is NULL";
    case RA_ERR_ALIGN: return "a pointer is not suitably aligned (16 bytes)";
    case RA_ERR_SHAPE: return "sizes out of range or N not a multiple of P";
    case RA_ERR_HEADDIM: return "head dimension must be 64 or 128";
    case RA_ERR_LAYOUT: return "unknown layout or flag bits";
    case RA_ERR_SCALE: return "scale must be finite and > 0";
    case RA_ERR_DTYPE: return "unknown dtype code";
    case RA_ERR_ALIAS: return "input and output buffers overlap";
    case RA_ERR_CUDA: return "a CUDA runtime/driver call failed";
    case RA_ERR_DEVICE: return "current device is not an sm_100 GPU";
    case RA_ERR_DEVICE_FAULT: return "a kernel gave up a bounded wait; outputs incomplete";
    case RA_ERR_ROPE: return "unknown RoPE pairing, or RoPE base not finite and > 1";
    case RA_ERR_WORKSPACE: return "device workspace too small (see ra_attn_fwd_host_workspace)";
    case RA_ERR_NOPROFILE: return "library built without the phase profile (RA_PROFILE)";
    case RA_ERR_SCRATCH:
      return "B*H*N exceeds the built-in scratch of ra_attn_bwd_noalloc (1048576 rows); "
             "use ra_attn_bwd with a workspace";
    default: return "unknown status";
  }
}

int ra_version(void) { return 200; }

ra_status ra_partition(const void* src, void* dst, int64_t B, int64_t H, int64_t N, int64_t d,
                       int P, int layout, int inverse, int dtype, void* stream) {
  if (!src || !dst) return RA_ERR_NULL;
  if (layout != RA_CONTIGUOUS && layout != RA_STRIPED && layout != RA_ZIGZAG) return RA_ERR_LAYOUT;
  int64_t esz;
  switch (dtype) {
    case RA_BF16: esz = 2; break;
    case RA_F32: case RA_I32: esz = 4; break;
    default: return RA_ERR_DTYPE;
  }
  if (B < 1 || H < 1 || N < 1 || d < 1 || P < 1 || N % P != 0) return RA_ERR_SHAPE;
  if (layout == RA_ZIGZAG && (N / P) % 2 != 0) return RA_ERR_SHAPE;
  if (!rows_fit(B, H, N) || d >= ((int64_t)1 << 30) / esz) return RA_ERR_SHAPE;
  const int64_t row_bytes = d * esz;
  const uintptr_t need = (row_bytes % 16 == 0) ? 16 : (esz == 2 ? 2 : 4);
  if (!aligned(src, need) || !aligned(dst, need)) return RA_ERR_ALIGN;
  const int64_t bytes = B * H * N * row_bytes;
  if (overlap(src, bytes, dst, bytes)) return RA_ERR_ALIAS;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  return partition_launch(src, dst, B * H, N, P, row_bytes, layout, inverse != 0, stream);
}

ra_status ra_partition_rope(const void* src, void* dst, int64_t B, int64_t H, int64_t N,
                            int64_t d, int P, int layout, int pairing, float base, void* stream) {
  if (!src || !dst) return RA_ERR_NULL;
  if (layout != RA_CONTIGUOUS && layout != RA_STRIPED && layout != RA_ZIGZAG) return RA_ERR_LAYOUT;
  if (d < 16 || d > 512 || d % 16 != 0) return RA_ERR_HEADDIM;
  if (B < 1 || H < 1 || N < 1 || P < 1 || N % P != 0) return RA_ERR_SHAPE;
  if (layout == RA_ZIGZAG && (N / P) % 2 != 0) return RA_ERR_SHAPE;
  if (!rows_fit(B, H, N)) return RA_ERR_SHAPE;
  if (pairing != RA_ROPE_INTERLEAVED && pairing != RA_ROPE_HALF) return RA_ERR_ROPE;
  if (!(base > 1.f) || !isfinite(base)) return RA_ERR_ROPE;
  if (!aligned(src, 16) || !aligned(dst, 16)) return RA_ERR_ALIGN;
  const int64_t bytes = B * H * N * d * 2;
  if (overlap(src, bytes, dst, bytes)) return RA_ERR_ALIAS;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  return partition_rope_launch(src, dst, B * H, N, P, d, layout,
                               pairing == RA_ROPE_HALF, std::log2((double)base), info.num_sms,
                               stream);
}

// Validates ra_attn_fwd's arguments and fills the launch description.
static ra_status fwd_prepare(const void* q, const void* k, const void* v, void* o, float* lse,
                             int64_t B, int64_t H, int64_t N, int64_t d, int P, int layout,
                             int causal, float scale, void* stream, AttnLaunch* out) {
  if (!q || !k || !v || !o || !lse) return RA_ERR_NULL;
  if (layout & ~(0xff | RA_SCHED_FREE | RA_O_F32 | RA_TOKEN_ORDER | RA_CTA_PAIR))
    return RA_ERR_LAYOUT;
  const int base = layout & 0xff;
  if (base != RA_CONTIGUOUS && base != RA_STRIPED && base != RA_ZIGZAG) return RA_ERR_LAYOUT;
  if (d != 64 && d != 128) return RA_ERR_HEADDIM;
  if (B < 1 || H < 1 || N < 1 || P < 1 || N % P != 0) return RA_ERR_SHAPE;
  if (base == RA_ZIGZAG && (N / P) % 512 != 0) return RA_ERR_SHAPE;
  if (!rows_fit(B, H, N)) return RA_ERR_SHAPE;
  if (N / P > ((int64_t)1 << 30) / 128) return RA_ERR_SHAPE;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_SCALE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 16))
    return RA_ERR_ALIGN;
  const bool o_f32 = (layout & RA_O_F32) != 0;
  const int64_t tb = B * H * N * d * 2, ob = o_f32 ? 2 * tb : tb, lb = B * H * N * 4;
  if (overlap(o, ob, q, tb) || overlap(o, ob, k, tb) || overlap(o, ob, v, tb) ||
      overlap(lse, lb, q, tb) || overlap(lse, lb, k, tb) || overlap(lse, lb, v, tb) ||
      overlap(lse, lb, o, ob))
    return RA_ERR_ALIAS;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  AttnLaunch a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.BH = B * H; a.N = N; a.d = d; a.P = P;
  a.striped = base == RA_STRIPED;
  a.zigzag = base == RA_ZIGZAG;
  a.causal = causal != 0;
  a.sched_free = (layout & RA_SCHED_FREE) != 0;
  a.o_f32 = o_f32;
  a.tok = (layout & RA_TOKEN_ORDER) != 0;
  a.pair = (layout & RA_CTA_PAIR) != 0;
  a.scale = scale;
  a.device = dev;
  a.num_sms = info.num_sms;
  a.stream = stream;
  *out = a;
  return RA_OK;
}

ra_status ra_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                      int64_t B, int64_t H, int64_t N, int64_t d, int P, int layout, int causal,
                      float scale, void* stream) {
  AttnLaunch a;
  const ra_status st = fwd_prepare(q, k, v, o, lse, B, H, N, d, P, layout, causal, scale, stream,
                                   &a);
  return st ? st : attn_fwd_launch(a);
}

ra_status ra_attn_abort_selftest(const void* q, const void* k, const void* v, void* o,
                                 float* lse, int64_t B, int64_t H, int64_t N, int64_t d, int P,
                                 int layout, int causal, float scale, int64_t limit_ns,
                                 void* stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return RA_ERR_SHAPE;
  AttnLaunch a;
  const ra_status st = fwd_prepare(q, k, v, o, lse, B, H, N, d, P, layout, causal, scale, stream,
                                   &a);
  if (st) return st;
  a.main_limit_ns = limit_ns;
  a.withhold_first_s = 1;
  return attn_fwd_launch(a);
}

ra_status ra_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      float* workspace, int64_t B, int64_t H, int64_t N, int64_t d, int P,
                      int layout, int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return RA_ERR_NULL;
  const int tok = (layout & RA_TOKEN_ORDER) != 0;
  layout &= ~RA_TOKEN_ORDER;
  if (layout != RA_CONTIGUOUS && layout != RA_STRIPED && layout != RA_ZIGZAG) return RA_ERR_LAYOUT;
  if (d != 64 && d != 128) return RA_ERR_HEADDIM;
  if (B < 1 || H < 1 || N < 1 || P < 1 || N % P != 0) return RA_ERR_SHAPE;
  if (layout == RA_ZIGZAG && (N / P) % 512 != 0) return RA_ERR_SHAPE;
  if (!rows_fit(B, H, N) || N / P > ((int64_t)1 << 30) / 128) return RA_ERR_SHAPE;
  if (B * H * P * ((N / P + 127) / 128) >= ((int64_t)1 << 31)) return RA_ERR_SHAPE;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_SCALE;
  const void* all[] = {q, k, v, o, dout, lse, dq, dk, dv, workspace};
  for (const void* ptr : all)
    if (!aligned(ptr, 16)) return RA_ERR_ALIGN;
  const int64_t tb = B * H * N * d * 2, lb = B * H * N * 4;
  const void* ins[] = {q, k, v, o, dout};
  void* outs[] = {dq, dk, dv};
  for (void* out : outs) {
    for (const void* in : ins)
      if (overlap(out, tb, in, tb)) return RA_ERR_ALIAS;
    if (overlap(out, tb, lse, lb) || overlap(out, tb, workspace, lb)) return RA_ERR_ALIAS;
  }
  if (overlap(dq, tb, dk, tb) || overlap(dq, tb, dv, tb) || overlap(dk, tb, dv, tb))
    return RA_ERR_ALIAS;
  for (const void* in : ins)
    if (overlap(workspace, lb, in, tb)) return RA_ERR_ALIAS;
  if (overlap(workspace, lb, lse, lb)) return RA_ERR_ALIAS;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  BwdLaunch a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv; a.workspace = workspace;
  a.BH = B * H; a.N = N; a.d = d; a.P = P;
  a.striped = layout == RA_STRIPED;
  a.zigzag = layout == RA_ZIGZAG;
  a.tok = tok;
  a.causal = causal != 0;
  a.scale = scale;
  a.device = dev;
  a.num_sms = info.num_sms;
  a.stream = stream;
  return attn_bwd_launch(a);
}

ra_status ra_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int64_t B, int64_t H, int64_t N, int64_t d, int P, int layout,
                              int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return RA_ERR_NULL;
  const int tok = (layout & RA_TOKEN_ORDER) != 0;
  layout &= ~RA_TOKEN_ORDER;
  if (layout != RA_CONTIGUOUS && layout != RA_STRIPED && layout != RA_ZIGZAG) return RA_ERR_LAYOUT;
  if (d != 64 && d != 128) return RA_ERR_HEADDIM;
  if (B < 1 || H < 1 || N < 1 || P < 1 || N % P != 0) return RA_ERR_SHAPE;
  if (layout == RA_ZIGZAG && (N / P) % 512 != 0) return RA_ERR_SHAPE;
  if (!rows_fit(B, H, N) || N / P > ((int64_t)1 << 30) / 128) return RA_ERR_SHAPE;
  if (B * H * N > kNoAllocScratchFloats) return RA_ERR_SCRATCH;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_SCALE;
  const void* all[] = {q, k, v, o, dout, lse, dq, dk, dv};
  for (const void* ptr : all)
    if (!aligned(ptr, 16)) return RA_ERR_ALIGN;
  const int64_t tb = B * H * N * d * 2, lb = B * H * N * 4;
  const void* ins[] = {q, k, v, o, dout};
  void* outs[] = {dq, dk, dv};
  for (void* out : outs) {
    for (const void* in : ins)
      if (overlap(out, tb, in, tb)) return RA_ERR_ALIAS;
    if (overlap(out, tb, lse, lb)) return RA_ERR_ALIAS;
  }
  if (overlap(dq, tb, dk, tb) || overlap(dq, tb, dv, tb) || overlap(dk, tb, dv, tb))
    return RA_ERR_ALIAS;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  BwdLaunch a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv; a.workspace = nullptr;
  a.BH = B * H; a.N = N; a.d = d; a.P = P;
  a.striped = layout == RA_STRIPED;
  a.zigzag = layout == RA_ZIGZAG;
  a.tok = tok;
  a.causal = causal != 0;
  a.scale = scale;
  a.device = dev;
  a.num_sms = info.num_sms;
  a.stream = stream;
  return attn_bwd_noalloc_launch(a);
}

ra_status ra_attn_fwd_block(const void* q, const void* k, const void* v, void* o, float* lse,
                            int64_t B, int64_t H, int64_t c, int64_t d, int j, int kb, int P,
                            int layout, int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !lse) return RA_ERR_NULL;
  const bool o_f32 = (layout & RA_O_F32) != 0;
  layout &= ~RA_O_F32;
  if (layout != RA_CONTIGUOUS && layout != RA_STRIPED) return RA_ERR_LAYOUT;
  if (d != 64 && d != 128) return RA_ERR_HEADDIM;
  if (B < 1 || H < 1 || c < 1 || P < 1 || j < 0 || j >= P || kb < 0 || kb >= P)
    return RA_ERR_SHAPE;
  if (!rows_fit(B, H, c) || c > ((int64_t)1 << 30) / 128 || c * (int64_t)P >= ((int64_t)1 << 31))
    return RA_ERR_SHAPE;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_SCALE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 16))
    return RA_ERR_ALIGN;
  const int64_t tb = B * H * c * d * 2, ob = o_f32 ? 2 * tb : tb, lb = B * H * c * 4;
  if (overlap(o, ob, q, tb) || overlap(o, ob, k, tb) || overlap(o, ob, v, tb) ||
      overlap(lse, lb, q, tb) || overlap(lse, lb, k, tb) || overlap(lse, lb, v, tb) ||
      overlap(o, ob, lse, lb))
    return RA_ERR_ALIAS;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  // A block that GetMask hides completely (contiguous causal, kb > j): no
  // query row sees a key of it.
  if (causal && layout == RA_CONTIGUOUS && kb > j) {
    if (cudaMemsetAsync(o, 0, (size_t)ob, (cudaStream_t)stream) != cudaSuccess) return RA_ERR_CUDA;
    return fill_f32_launch(lse, B * H * c, -INFINITY, stream);
  }
  AttnLaunch a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.BH = B * H; a.N = c; a.d = d; a.P = 1;
  a.o_f32 = o_f32;
  a.striped = layout == RA_STRIPED;
  a.causal = causal != 0;
  a.sched_free = 1;
  a.scale = scale;
  a.device = dev;
  a.num_sms = info.num_sms;
  a.stream = stream;
  a.blk_j = j;
  a.blk_kb = kb;
  return attn_fwd_launch(a);
}

ra_status ra_lse_merge_acc(float* o_acc, float* lse_acc, const void* o_b, const float* lse_b,
                           void* o_final, int64_t rows, int64_t d, int mode, void* stream) {
  if (!o_acc || !lse_acc || !o_b || !lse_b) return RA_ERR_NULL;
  if ((mode & ~7) != 0) return RA_ERR_LAYOUT;
  const int first = mode & RA_MERGE_FIRST, final_ = (mode & RA_MERGE_FINAL) != 0;
  const int b_f32 = (mode & RA_MERGE_F32_PARTIAL) != 0;
  if (final_ && !o_final) return RA_ERR_NULL;
  if (rows < 0 || d < 8 || d % 8 != 0 || d > (1 << 20) || rows >= ((int64_t)1 << 31))
    return RA_ERR_SHAPE;
  if (!aligned(o_acc, 16) || !aligned(o_b, 16) || !aligned(lse_acc, 4) || !aligned(lse_b, 4) ||
      (final_ && !aligned(o_final, 16)))
    return RA_ERR_ALIGN;
  const int64_t ab = rows * d * 4, fb = rows * d * 2, bb = b_f32 ? ab : fb, lb = rows * 4;
  if (overlap(o_acc, ab, o_b, bb) || overlap(o_acc, ab, lse_acc, lb) ||
      overlap(o_acc, ab, lse_b, lb) || overlap(lse_acc, lb, o_b, bb) ||
      overlap(lse_acc, lb, lse_b, lb))
    return RA_ERR_ALIAS;
  if (final_ && (overlap(o_final, fb, o_acc, ab) || overlap(o_final, fb, o_b, bb) ||
                 overlap(o_final, fb, lse_acc, lb) || overlap(o_final, fb, lse_b, lb)))
    return RA_ERR_ALIAS;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  return lse_merge_acc_launch(o_acc, lse_acc, o_b, lse_b, o_final, rows, d, first, final_, b_f32,
                              stream);
}

int64_t ra_attn_fwd_host_workspace(int64_t N, int64_t d, int layout, int64_t heads_per_chunk) {
  if (N < 1 || d < 1 || heads_per_chunk < 1) return -1;
  if (N >= ((int64_t)1 << 31) || d > 1024) return -1;
  (void)layout;
  const HostPlan h = host_plan(N, d);
  if (heads_per_chunk > INT64_MAX / (2 * h.per_head)) return -1;
  return 2 * heads_per_chunk * h.per_head;
}

ra_status ra_attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                           int64_t B, int64_t H, int64_t N, int64_t d, int P, int layout,
                           int causal, float scale, void* workspace, int64_t workspace_bytes,
                           void* stream) {
  if (!q || !k || !v || !o || !lse || !workspace) return RA_ERR_NULL;
  if (layout & ~(0xff | RA_SCHED_FREE)) return RA_ERR_LAYOUT;
  const int base = layout & 0xff;
  if (base != RA_CONTIGUOUS && base != RA_STRIPED && base != RA_ZIGZAG) return RA_ERR_LAYOUT;
  if (d != 64 && d != 128) return RA_ERR_HEADDIM;
  if (B < 1 || H < 1 || N < 1 || P < 1 || N % P != 0) return RA_ERR_SHAPE;
  if (base == RA_ZIGZAG && (N / P) % 512 != 0) return RA_ERR_SHAPE;
  if (!rows_fit(B, H, N) || N / P > ((int64_t)1 << 30) / 128) return RA_ERR_SHAPE;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_SCALE;
  if (!aligned(workspace, 256)) return RA_ERR_ALIGN;
  const HostPlan hp = host_plan(N, d);
  const int64_t BH = B * H;
  int64_t G = workspace_bytes / (2 * hp.per_head);
  if (G < 1) return RA_ERR_WORKSPACE;
  // at least four chunks when there are enough heads, so that copies overlap
  const int64_t want = (BH + 3) / 4;
  if (G > want) G = want;
  if (G > BH) G = BH;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  HostStreams* hs;
  std::mutex* mu;
  if ((st = host_streams(dev, &hs, &mu))) return st;
  std::lock_guard<std::mutex> lock(*mu);
  cudaStream_t cs = (cudaStream_t)stream;
  auto chk = [](cudaError_t e) { return e == cudaSuccess; };
  if (!chk(cudaEventRecord(hs->entry, cs)) || !chk(cudaStreamWaitEvent(hs->in, hs->entry, 0)) ||
      !chk(cudaStreamWaitEvent(hs->out, hs->entry, 0)))
    return RA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t T = round256(hp.tok) * G;
  // Chunk sizes: the first chunk's copy in and the last chunk's copy out
  // overlap no compute, so both take half a chunk (when there are heads to
  // spare); the chunks between take G heads.
  std::vector<int64_t> sizes;
  {
    const int64_t half = G > 1 ? G / 2 : 1;
    int64_t rem = BH;
    int64_t last = 0;
    if (rem > 2 * half) {
      sizes.push_back(half);
      rem -= half;
      last = half;
      rem -= last;
    }
    while (rem > 0) {
      const int64_t g = rem < G ? rem : G;
      sizes.push_back(g);
      rem -= g;
    }
    if (last) sizes.push_back(last);
  }
  const int64_t nch = (int64_t)sizes.size();
  int64_t h0 = 0;
  for (int64_t i = 0; i < nch; h0 += sizes[i], ++i) {
    const int s = (int)(i & 1);
    const int64_t g = sizes[i];
    const int64_t tb = g * hp.tok, lb = g * hp.lsz;
    uint8_t* slot = ws + s * G * hp.per_head;
    uint8_t *dq = slot, *dk = dq + T, *dv = dk + T, *dout = dv + T;
    float* dl = reinterpret_cast<float*>(dout + T);
    // inputs of chunk i (the slot's previous chunk has been read back)
    if (i >= 2 && !chk(cudaStreamWaitEvent(hs->in, hs->d2h[s], 0))) return RA_ERR_CUDA;
    const uint8_t* hq = static_cast<const uint8_t*>(q) + h0 * hp.tok;
    const uint8_t* hk = static_cast<const uint8_t*>(k) + h0 * hp.tok;
    const uint8_t* hv = static_cast<const uint8_t*>(v) + h0 * hp.tok;
    if (!chk(cudaMemcpyAsync(dq, hq, tb, cudaMemcpyHostToDevice, hs->in)) ||
        !chk(cudaMemcpyAsync(dk, hk, tb, cudaMemcpyHostToDevice, hs->in)) ||
        !chk(cudaMemcpyAsync(dv, hv, tb, cudaMemcpyHostToDevice, hs->in)) ||
        !chk(cudaEventRecord(hs->h2d[s], hs->in)))
      return RA_ERR_CUDA;
    // compute on the caller's stream
    if (!chk(cudaStreamWaitEvent(cs, hs->h2d[s], 0))) return RA_ERR_CUDA;
    AttnLaunch a;
    a.BH = g; a.N = N; a.d = d; a.P = P;
    a.striped = base == RA_STRIPED;
    a.zigzag = base == RA_ZIGZAG;
    a.causal = causal != 0;
    a.sched_free = (layout & RA_SCHED_FREE) != 0;
    a.scale = scale;
    a.device = dev;
    a.num_sms = info.num_sms;
    a.stream = stream;
    a.q = dq; a.k = dk; a.v = dv; a.o = dout; a.lse = dl;
    a.tok = 1;
    if ((st = attn_fwd_launch(a))) return st;
    if (!chk(cudaEventRecord(hs->comp[s], cs))) return RA_ERR_CUDA;
    // results of chunk i back to the host
    if (!chk(cudaStreamWaitEvent(hs->out, hs->comp[s], 0)) ||
        !chk(cudaMemcpyAsync(static_cast<uint8_t*>(o) + h0 * hp.tok, dout, tb,
                             cudaMemcpyDeviceToHost, hs->out)) ||
        !chk(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(lse) + h0 * hp.lsz, dl, lb,
                             cudaMemcpyDeviceToHost, hs->out)) ||
        !chk(cudaEventRecord(hs->d2h[s], hs->out)))
      return RA_ERR_CUDA;
  }
  // the caller's stream continues once every result is on the host
  if (!chk(cudaEventRecord(hs->end, hs->out)) || !chk(cudaStreamWaitEvent(cs, hs->end, 0)))
    return RA_ERR_CUDA;
  return RA_OK;
}

ra_status ra_lse_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                       void* o_out, float* lse_out, int64_t rows, int64_t d, void* stream) {
  if (!o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out) return RA_ERR_NULL;
  if (rows < 0 || d < 1 || d % 8 != 0 || d > (1 << 20)) return RA_ERR_SHAPE;
  if (rows >= ((int64_t)1 << 40)) return RA_ERR_SHAPE;
  if (!aligned(o_a, 16) || !aligned(o_b, 16) || !aligned(o_out, 16) || !aligned(lse_a, 4) ||
      !aligned(lse_b, 4) || !aligned(lse_out, 4))
    return RA_ERR_ALIGN;
  const int64_t ob = rows * d * 2, lb = rows * 4;
  // o_out may coincide with o_a exactly; any other overlap is refused.
  if ((o_out != o_a && overlap(o_out, ob, o_a, ob)) || overlap(o_out, ob, o_b, ob) ||
      (lse_out != lse_a && overlap(lse_out, lb, lse_a, lb)) ||
      (lse_out != lse_b && overlap(lse_out, lb, lse_b, lb)) || overlap(o_out, ob, lse_out, lb))
    return RA_ERR_ALIAS;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  return lse_merge_launch(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d, info.num_sms, stream);
}

ra_status ra_tile_census(int64_t N, int P, int layout, int causal, int64_t* out, void* stream) {
  if (!out) return RA_ERR_NULL;
  if (layout != RA_CONTIGUOUS && layout != RA_STRIPED) return RA_ERR_LAYOUT;
  if (N < 1 || P < 1 || N % P != 0 || N >= ((int64_t)1 << 31) || P > 65536) return RA_ERR_SHAPE;
  if (!aligned(out, 8)) return RA_ERR_ALIGN;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  return tile_census_launch(N, P, layout == RA_STRIPED, causal != 0, out, stream);
}

ra_status ra_wait_selftest(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return RA_ERR_SHAPE;
  int dev;
  DevInfo info;
  ra_status st = current_device(&dev, &info);
  if (st) return st;
  return wait_selftest_launch(limit_ns, stream);
}

ra_status ra_device_fault(int* code) {
  if (!code) return RA_ERR_NULL;
  return read_device_fault(code);
}

ra_status ra_fwd_phase_profile(uint64_t* out, int64_t capacity) {
  if (!out) return RA_ERR_NULL;
  return fwd_profile_read(reinterpret_cast<unsigned long long*>(out), capacity);
}

}  // extern "C"
