// norm.cuh — the second pass over a compressed latent that spans several
// GEMM tiles: RMSNorm with its bottleneck scale factor, and the FP8 encoding
// of a cache row.
//
// RMSNorm (DeepSeek-V2 explainer, adg.csdn.net, section 3.1.1: an extra RMS
// norm after the compressed latent vectors and extra scale factors at these
// width bottlenecks):
//   y = scale * g * x / sqrt(mean(x^2) + eps)
// x is the fp32 output of the latent GEMM (c^KV = W^DKV h or c^Q = W^DQ h);
// y goes out in bf16, either to a plain [T][n] buffer (c^Q, read by the next
// GEMM) or into the token's paged-cache row (c^KV, next to the RoPE key the
// compress GEMM wrote there).  With an FP8 cache (explainer section 3.1.4:
// the KV cache is quantised for serving) the cache row takes y (or x when
// the layer has no norm) as E4M3 codes with one power-of-two scale per row.
// Both the norm and the row scale span all n features of a token, which the
// GEMM spreads over several 128-row tiles, hence their own pass.  The same
// encoding turns bf16 cache rows into FP8 rows (mla_cache_to_fp8_kernel).
#pragma once

#include "common.cuh"

namespace mla {

struct NormArgs {
  const float* x;             // [T][n] fp32
  int n;
  int do_norm;                // 0: y = x (FP8 encoding only)
  const __nv_bfloat16* gain;  // [n]
  float eps, scale;
  __nv_bfloat16* out;         // plain destination [T][out_t], or nullptr: the cache row
  long long out_t;
  uint8_t* pool;              // paged cache [num_blocks][block_size][row_bytes]
  const int32_t* table;
  const int32_t* seq_idx;
  const int32_t* pos;
  int num_blocks, max_blocks, block_size, row_bytes;
  int fp8;                    // cache rows are FP8 (codes at byte 0, scale at scale_off)
  int scale_off;
};

constexpr int NORM_THREADS = 128;

__device__ __forceinline__ float block_reduce_128(float v, float* part, bool is_max) {
  v = is_max ? warp_max(v) : warp_sum(v);
  __syncthreads();  // part may still be read from a previous reduction
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = part[0];
#pragma unroll
  for (int w = 1; w < NORM_THREADS / 32; ++w) r = is_max ? fmaxf(r, part[w]) : r + part[w];
  return r;
}

// One block per token.  n is a multiple of 4.
__global__ void __launch_bounds__(NORM_THREADS) mla_latent_norm_kernel(const NormArgs a) {
  __shared__ float part[NORM_THREADS / 32];
  pdl_trigger();
  pdl_wait();  // x comes from the GEMM just before
  const int t = blockIdx.x;
  const float4* x = reinterpret_cast<const float4*>(a.x + (long long)t * a.n);
  float f = 1.f;
  if (a.do_norm) {
    float acc = 0.f;
    for (int i = threadIdx.x; i < a.n / 4; i += NORM_THREADS) {
      const float4 v = x[i];
      acc = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, acc))));
    }
    f = a.scale / sqrtf(block_reduce_128(acc, part, false) / (float)a.n + a.eps);
  }
  auto value = [&](int i) -> float4 {
    float4 v = x[i];
    if (a.do_norm) {
      const float2 ga = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(a.gain + 4 * i));
      const float2 gb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(a.gain + 4 * i + 2));
      v = make_float4(ga.x * (v.x * f), ga.y * (v.y * f), gb.x * (v.z * f), gb.y * (v.w * f));
    }
    return v;
  };
  uint8_t* dst = reinterpret_cast<uint8_t*>(a.out);
  if (dst) {
    dst += (long long)t * a.out_t * 2;
  } else {
    const long long p = a.pos[t];
    const int page = (int)(p / a.block_size);
    const int blk = (page >= 0 && page < a.max_blocks) ? a.table[(long long)a.seq_idx[t] * a.max_blocks + page] : -1;
    if (blk < 0 || blk >= a.num_blocks) {
      if (threadIdx.x == 0) record_error(ERR_CAPACITY, 602);
      return;
    }
    dst = a.pool + ((long long)blk * a.block_size + p % a.block_size) * a.row_bytes;
  }
  if (!a.fp8) {
    for (int i = threadIdx.x; i < a.n / 4; i += NORM_THREADS) {
      const float4 v = value(i);
      *reinterpret_cast<uint2*>(dst + 8 * i) = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
    }
    return;
  }
  float amax = 0.f;
  for (int i = threadIdx.x; i < a.n / 4; i += NORM_THREADS) {
    const float4 v = value(i);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  const int e = fp8_scale_exponent(block_reduce_128(amax, part, true));
  const float inv = exp2_int(-e);
  for (int i = threadIdx.x; i < a.n / 4; i += NORM_THREADS) {
    const float4 v = value(i);
    const uint32_t lo = e4m3x2_from_f32(v.x * inv, v.y * inv), hi = e4m3x2_from_f32(v.z * inv, v.w * inv);
    *reinterpret_cast<uint32_t*>(dst + 4 * i) = lo | (hi << 16);
  }
  // the scale and the row's zero padding (the field is 16-byte aligned)
  if (threadIdx.x == 0) *reinterpret_cast<uint4*>(dst + a.scale_off) = make_uint4(__float_as_uint(exp2_int(e)), 0, 0, 0);
}

// bf16 cache rows [n][d_c + d_hr] -> FP8 rows [n][row_bytes]: E4M3 codes of
// c^KV with the row's power-of-two scale, k^R copied, padding zeroed.  One
// warp per row; d_c == 512, d_hr == 64.  A NaN element (an unwritten slot)
// becomes a NaN code and does not enter the row maximum.
constexpr int CVT_ROWS_PER_BLOCK = 8;
__global__ void __launch_bounds__(32 * CVT_ROWS_PER_BLOCK)
    mla_cache_to_fp8_kernel(const __nv_bfloat16* __restrict__ src, long long n, uint8_t* __restrict__ dst,
                            int row_bytes) {
  pdl_trigger();
  pdl_wait();
  const long long r = (long long)blockIdx.x * CVT_ROWS_PER_BLOCK + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= n) return;
  const __nv_bfloat16* s = src + r * 576;
  uint8_t* d = dst + r * row_bytes;
  // lane: latent elements 16 lane .. 16 lane + 15
  const uint4 raw0 = reinterpret_cast<const uint4*>(s)[2 * lane];
  const uint4 raw1 = reinterpret_cast<const uint4*>(s)[2 * lane + 1];
  float v[16];
  const uint32_t w[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = fp8_scale_exponent(warp_max(amax));
  const float inv = exp2_int(-e);
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    c[i] = (uint32_t)e4m3x2_from_f32(v[4 * i] * inv, v[4 * i + 1] * inv) |
           ((uint32_t)e4m3x2_from_f32(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
  reinterpret_cast<uint4*>(d)[lane] = make_uint4(c[0], c[1], c[2], c[3]);
  // k^R (128 bytes) and the scale with its padding (16 bytes)
  if (lane < 8) reinterpret_cast<uint4*>(d + 512)[lane] = reinterpret_cast<const uint4*>(s + 512)[lane];
  if (lane == 8) reinterpret_cast<uint4*>(d + 640)[0] = make_uint4(__float_as_uint(exp2_int(e)), 0, 0, 0);
}

}  // namespace mla
