// Memory-bound helpers of the ring: layout permutation (ra_partition), the
// (O, lse) merge (ra_lse_merge) and the tile census (ra_tile_census).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ra_internal.h"
#include "ra_tiles.cuh"

namespace ra {

// ------------------------------------------------------------- partition
// Row n of the destination (within one (b, h)) comes from source row
//   forward (token -> layout): slot n holds token (n % c) * P + n / c
//   inverse (layout -> token): token n sits in slot (n % P) * c + n / P
// (striped placement of the Striped Attention review, 分区策略对比), or, for
// the zigzag layout (zz; chunks j and 2P-1-j of h = c/2 tokens on shard j)
//   forward: slot n = (j, l) holds token j*h + l (l < h), (2P-1-j)*h + l-h
//   inverse: token n in chunk a = n / h sits in shard a (a < P) or 2P-1-a.
__device__ __forceinline__ int zz_token_of_slot(int n, int c, int P) {
  const int h = c >> 1, j = n / c, l = n - j * c;
  return l < h ? j * h + l : (2 * P - 1 - j) * h + (l - h);
}
__device__ __forceinline__ int zz_slot_of_token(int n, int c, int P) {
  const int h = c >> 1, a = n / h, l = n - a * h;
  return a < P ? a * c + l : (2 * P - 1 - a) * c + h + l;
}

template <typename U>
__global__ void partition_kernel(const U* __restrict__ src, U* __restrict__ dst, int rows_total,
                                 int N, int P, int c, int upr, int rows_per_block, int inverse,
                                 int zz) {
  const int row0 = blockIdx.x * rows_per_block;
  int nrows = rows_total - row0;
  if (nrows > rows_per_block) nrows = rows_per_block;
  const int units = nrows * upr;
  for (int u = threadIdx.x; u < units; u += blockDim.x) {
    const int rl = u / upr;
    const int e = u - rl * upr;
    const int row = row0 + rl;
    const int bh = row / N;
    const int n = row - bh * N;
    int sn;
    if (zz) {
      sn = inverse ? zz_slot_of_token(n, c, P) : zz_token_of_slot(n, c, P);
    } else if (inverse) {
      const int sh = n % P;
      sn = sh * c + n / P;
    } else {
      const int sh = n / c;
      sn = (n - sh * c) * P + sh;
    }
    dst[(size_t)row * upr + e] = src[((size_t)bh * N + sn) * upr + e];
  }
}

template <typename U>
static ra_status launch_partition_t(const void* src, void* dst, int rows_total, int N, int P,
                                    int64_t row_bytes, int inverse, int zz, void* stream) {
  const int upr = (int)(row_bytes / (int64_t)sizeof(U));
  int rpb = 2048 / upr;
  if (rpb < 1) rpb = 1;
  const int blocks = (rows_total + rpb - 1) / rpb;
  partition_kernel<U><<<blocks, 256, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const U*>(src), reinterpret_cast<U*>(dst), rows_total, N, P, N / P, upr,
      rpb, inverse, zz);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status partition_launch(const void* src, void* dst, int64_t rows_outer, int64_t N, int64_t P,
                           int64_t row_bytes, int layout, int inverse, void* stream) {
  const int64_t total_bytes = rows_outer * N * row_bytes;
  if (total_bytes == 0) return RA_OK;
  if (layout == RA_CONTIGUOUS) {
    // the contiguous placement is the identity
    return cudaMemcpyAsync(dst, src, (size_t)total_bytes, cudaMemcpyDeviceToDevice,
                           (cudaStream_t)stream) == cudaSuccess
               ? RA_OK
               : RA_ERR_CUDA;
  }
  const int rows_total = (int)(rows_outer * N);
  const uintptr_t al = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst);
  if (row_bytes % 16 == 0 && al % 16 == 0)
    return launch_partition_t<uint4>(src, dst, rows_total, (int)N, (int)P, row_bytes, inverse,
                                     layout == RA_ZIGZAG, stream);
  if (row_bytes % 8 == 0 && al % 8 == 0)
    return launch_partition_t<uint2>(src, dst, rows_total, (int)N, (int)P, row_bytes, inverse,
                                     layout == RA_ZIGZAG, stream);
  if (row_bytes % 4 == 0 && al % 4 == 0)
    return launch_partition_t<uint32_t>(src, dst, rows_total, (int)N, (int)P, row_bytes,
                                        inverse, layout == RA_ZIGZAG, stream);
  if (row_bytes % 2 == 0 && al % 2 == 0)
    return launch_partition_t<uint16_t>(src, dst, rows_total, (int)N, (int)P, row_bytes,
                                        inverse, layout == RA_ZIGZAG, stream);
  return launch_partition_t<uint8_t>(src, dst, rows_total, (int)N, (int)P, row_bytes, inverse,
                                     layout == RA_ZIGZAG, stream);
}

// --------------------------------------------------- partition with RoPE
// dst[bh, s(t), :] = RoPE(src[bh, t, :]) at position t, in layout order
// (Striped review, 位置编码处理: the position encoding sees the same stripe as
// the tokens).  RoPE as in RoFormer: pair i turns by t * base^(-2i/d); the
// pairs are dimensions (2i, 2i+1) (interleaved) or (i, i + d/2) (half).
// One thread owns one chunk of one token row and walks all (b, h), so the
// angles are computed once per (token, pair): in double precision (the
// angle reaches N radians), rotated in fp32, rounded to bf16 once.
template <int HALF>
__global__ void partition_rope_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                      int BH, int N, int P, int c, int layout, int d,
                                      double log2_base) {
  constexpr int kPairs = HALF ? 8 : 4;       // rotation pairs per work chunk
  const int u16 = d / 8;                     // 16-byte units per row
  const int cpr = HALF ? d / 16 : d / 8;     // work chunks per row
  const long long total = (long long)N * cpr;
  for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(w / cpr), ch = (int)(w % cpr);
    const int s = layout == RA_STRIPED ? (t % P) * c + t / P
                  : layout == RA_ZIGZAG ? zz_slot_of_token(t, c, P) : t;
    float cs[kPairs], sn[kPairs];
#pragma unroll
    for (int k = 0; k < kPairs; ++k) {
      const int i = ch * kPairs + k;
      const double ang = (double)t * exp2(-(2.0 * i / d) * log2_base);
      double sd, cd;
      sincos(ang, &sd, &cd);
      cs[k] = (float)cd;
      sn[k] = (float)sd;
    }
#pragma unroll 4
    for (int bh = 0; bh < BH; ++bh) {
      const uint4* in = src + ((size_t)bh * N + t) * u16;
      uint4* out = dst + ((size_t)bh * N + s) * u16;
      if (HALF) {
        uint4 a = in[ch], b = in[ch + u16 / 2];
        __nv_bfloat162* a2 = reinterpret_cast<__nv_bfloat162*>(&a);
        __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&b);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 u = __bfloat1622float2(a2[j]), v = __bfloat1622float2(b2[j]);
          const float c0 = cs[2 * j], s0 = sn[2 * j], c1 = cs[2 * j + 1], s1 = sn[2 * j + 1];
          a2[j] = __floats2bfloat162_rn(fmaf(u.x, c0, -v.x * s0), fmaf(u.y, c1, -v.y * s1));
          b2[j] = __floats2bfloat162_rn(fmaf(u.x, s0, v.x * c0), fmaf(u.y, s1, v.y * c1));
        }
        out[ch] = a;
        out[ch + u16 / 2] = b;
      } else {
        uint4 a = in[ch];
        __nv_bfloat162* a2 = reinterpret_cast<__nv_bfloat162*>(&a);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 u = __bfloat1622float2(a2[j]);
          a2[j] = __floats2bfloat162_rn(fmaf(u.x, cs[j], -u.y * sn[j]),
                                        fmaf(u.x, sn[j], u.y * cs[j]));
        }
        out[ch] = a;
      }
    }
  }
}

ra_status partition_rope_launch(const void* src, void* dst, int64_t BH, int64_t N, int64_t P,
                                int64_t d, int layout, int half, double log2_base, int num_sms,
                                void* stream) {
  const long long cpr = half ? d / 16 : d / 8;
  const long long total = N * cpr;
  if (total == 0) return RA_OK;
  long long blocks = (total + 255) / 256;
  if (blocks > (long long)num_sms * 8) blocks = (long long)num_sms * 8;
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* t = reinterpret_cast<uint4*>(dst);
  cudaStream_t st = (cudaStream_t)stream;
  if (half)
    partition_rope_kernel<1><<<(int)blocks, 256, 0, st>>>(s, t, (int)BH, (int)N, (int)P,
                                                           (int)(N / P), layout, (int)d, log2_base);
  else
    partition_rope_kernel<0><<<(int)blocks, 256, 0, st>>>(s, t, (int)BH, (int)N, (int)P,
                                                           (int)(N / P), layout, (int)d, log2_base);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// -------------------------------------------------------------- lse merge
// One warp per row: every lane reads both lse values before lane 0 writes
// lse_out (which may alias lse_a); each 8-element chunk of o is read and
// written by the same lane (o_out may alias o_a).
__global__ void lse_merge_kernel(const uint4* oa, const float* lse_a,
                                 const uint4* __restrict__ ob, const float* lse_b, uint4* oo,
                                 float* lse_o, long long rows, int chunks) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const float la = lse_a[r];
    const float lb = lse_b[r];
    const float mx = fmaxf(la, lb);
    float wa = 0.f, wb = 0.f, lse = -INFINITY;
    if (mx != -INFINITY) {
      const float ea = __expf(la - mx);
      const float eb = __expf(lb - mx);
      const float s = ea + eb;
      wa = ea / s;
      wb = eb / s;
      lse = mx + __logf(s);
    }
    __syncwarp();
    for (int ch = lane; ch < chunks; ch += 32) {
      const size_t idx = (size_t)r * chunks + ch;
      const uint4 a = oa[idx];
      const uint4 b = ob[idx];
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
      uint4 out;
      __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fa = __bfloat1622float2(a2[i]);
        const float2 fb = __bfloat1622float2(b2[i]);
        o2[i] = __floats2bfloat162_rn(wa * fa.x + wb * fb.x, wa * fa.y + wb * fb.y);
      }
      oo[idx] = out;
    }
    if (lane == 0) lse_o[r] = lse;
    __syncwarp();
  }
}

ra_status lse_merge_launch(const void* o_a, const float* lse_a, const void* o_b,
                           const float* lse_b, void* o_out, float* lse_out, int64_t rows,
                           int64_t d, int num_sms, void* stream) {
  if (rows == 0) return RA_OK;
  const int chunks = (int)(d / 8);
  long long blocks = (rows + 7) / 8;
  const long long cap = (long long)num_sms * 16;
  if (blocks > cap) blocks = cap;
  lse_merge_kernel<<<(int)blocks, 256, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint4*>(o_a), lse_a, reinterpret_cast<const uint4*>(o_b), lse_b,
      reinterpret_cast<uint4*>(o_out), lse_out, (long long)rows, chunks);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// ------------------------------------------------ merge into an accumulator
// (O_acc, lse_acc) <- merge of (O_acc, lse_acc) and a bf16 partial (O_b,
// lse_b) through their normalisers (1cademy page "Computing Attention
// Weights in Sequence Parallelism"), with O_acc kept in fp32 so that P
// rounds round to bf16 only once.  first: the accumulator is not yet set
// (it becomes the partial).  final: also write O_acc as bf16 to o_final.
// Both sides empty (lse = -inf) give O = 0, lse = -inf.
template <bool F32B>
__global__ void lse_merge_acc_kernel(float* __restrict__ oacc, float* __restrict__ lacc,
                                     const void* __restrict__ ob_, const float* __restrict__ lb_,
                                     uint4* __restrict__ ofin, long long rows, int chunks,
                                     int first, int final_) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const float lb = lb_[r];
    const float la = first ? -INFINITY : lacc[r];
    const float mx = fmaxf(la, lb);
    float wa = 0.f, wb = 0.f, lse = -INFINITY;
    if (mx != -INFINITY) {
      const float ea = expf(la - mx);
      const float eb = expf(lb - mx);
      const float sum = ea + eb;
      wa = ea / sum;
      wb = eb / sum;
      lse = mx + logf(sum);
    }
    __syncwarp();
    for (int ch = lane; ch < chunks; ch += 32) {
      const size_t idx = (size_t)r * chunks + ch;
      float2 b0, b1, b2v, b3;   // the partial's 8 values of this chunk
      if (F32B) {
        const float4* f = reinterpret_cast<const float4*>(ob_) + idx * 2;
        const float4 u = f[0], w = f[1];
        b0 = make_float2(u.x, u.y);
        b1 = make_float2(u.z, u.w);
        b2v = make_float2(w.x, w.y);
        b3 = make_float2(w.z, w.w);
      } else {
        const uint4 b = reinterpret_cast<const uint4*>(ob_)[idx];
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
        b0 = __bfloat1622float2(b2[0]);
        b1 = __bfloat1622float2(b2[1]);
        b2v = __bfloat1622float2(b2[2]);
        b3 = __bfloat1622float2(b2[3]);
      }
      float4* a4 = reinterpret_cast<float4*>(oacc) + idx * 2;
      float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
      if (!first) {
        a0 = a4[0];
        a1 = a4[1];
      }
      a0 = make_float4(wa * a0.x + wb * b0.x, wa * a0.y + wb * b0.y, wa * a0.z + wb * b1.x,
                       wa * a0.w + wb * b1.y);
      a1 = make_float4(wa * a1.x + wb * b2v.x, wa * a1.y + wb * b2v.y, wa * a1.z + wb * b3.x,
                       wa * a1.w + wb * b3.y);
      a4[0] = a0;
      a4[1] = a1;
      if (final_) {
        uint4 out;
        __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&out);
        o2[0] = __floats2bfloat162_rn(a0.x, a0.y);
        o2[1] = __floats2bfloat162_rn(a0.z, a0.w);
        o2[2] = __floats2bfloat162_rn(a1.x, a1.y);
        o2[3] = __floats2bfloat162_rn(a1.z, a1.w);
        ofin[idx] = out;
      }
    }
    if (lane == 0) lacc[r] = lse;
    __syncwarp();
  }
}

ra_status lse_merge_acc_launch(float* o_acc, float* lse_acc, const void* o_b,
                               const float* lse_b, void* o_final, int64_t rows, int64_t d,
                               int first, int final_, int b_f32, void* stream) {
  if (rows == 0) return RA_OK;
  const int chunks = (int)(d / 8);
  long long blocks = (rows + 7) / 8;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  if (b_f32)
    lse_merge_acc_kernel<true><<<(int)blocks, 256, 0, (cudaStream_t)stream>>>(
        o_acc, lse_acc, o_b, lse_b, reinterpret_cast<uint4*>(o_final), (long long)rows, chunks,
        first, final_);
  else
    lse_merge_acc_kernel<false><<<(int)blocks, 256, 0, (cudaStream_t)stream>>>(
        o_acc, lse_acc, o_b, lse_b, reinterpret_cast<uint4*>(o_final), (long long)rows, chunks,
        first, final_);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

__global__ void fill_f32_kernel(float* __restrict__ dst, long long n, float value) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    dst[i] = value;
}

ra_status fill_f32_launch(float* dst, int64_t n, float value, void* stream) {
  if (n == 0) return RA_OK;
  long long blocks = (n + 255) / 256;
  if (blocks > 148LL * 8) blocks = 148LL * 8;
  fill_f32_kernel<<<(int)blocks, 256, 0, (cudaStream_t)stream>>>(dst, (long long)n, value);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// ------------------------------------------------------------ tile census
// One thread per (query shard j, round r, query tile qt); classification and
// per-row limits are the attention kernel's own (ra_tiles.cuh).
__global__ void tile_census_kernel(int c, int P, int T, int striped, int causal,
                                   unsigned long long* out) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= (long long)P * P * T) return;
  const int qt = (int)(tid % T);
  const int jr = (int)(tid / T);
  const int j = jr / P;
  const int r = jr % P;
  const int kb = key_block(j, r, P);
  const BlockMask bm = block_mask(j, kb, striped, causal);
  const int x0 = qt * kBM;
  const int rows = tile_rows(x0, c);
  unsigned long long cnt[3] = {0, 0, 0};
  unsigned long long pairs = 0;
  for (int kt = 0; kt < T; ++kt) {
    const int y0 = kt * kBN;
    const int kind = tile_kind(bm, x0, y0, c);
    ++cnt[kind];
    if (kind == TILE_FULL) {
      pairs += (unsigned long long)rows * kBN;
    } else if (kind == TILE_PARTIAL) {
      for (int i = 0; i < rows; ++i) {
        int lim = row_limit(bm, x0 + i, y0, c);
        lim = lim < 0 ? 0 : (lim > kBN ? kBN : lim);
        pairs += (unsigned long long)lim;
      }
    }
  }
  unsigned long long* o = out + (size_t)(j * P + r) * 4;
  atomicAdd(o + 0, cnt[0]);
  atomicAdd(o + 1, cnt[1]);
  atomicAdd(o + 2, cnt[2]);
  atomicAdd(o + 3, pairs);
}

ra_status tile_census_launch(int64_t N, int P, int striped, int causal, int64_t* out,
                             void* stream) {
  const int c = (int)(N / P);
  const int T = (c + kBM - 1) / kBM;
  if (cudaMemsetAsync(out, 0, sizeof(int64_t) * 4 * (size_t)P * P, (cudaStream_t)stream) !=
      cudaSuccess)
    return RA_ERR_CUDA;
  const long long threads = (long long)P * P * T;
  const int blocks = (int)((threads + 127) / 128);
  tile_census_kernel<<<blocks, 128, 0, (cudaStream_t)stream>>>(
      c, P, T, striped, causal, reinterpret_cast<unsigned long long*>(out));
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace ra
