// norm.cuh — RMSNorm of the compressed latents with their bottleneck scale
// factors (DeepSeek-V2 explainer, adg.csdn.net, section 3.1.1: an extra RMS
// norm after the compressed latent vectors and extra scale factors at these
// width bottlenecks):
//   y = scale * g * x / sqrt(mean(x^2) + eps)
// x is the fp32 output of the latent GEMM (c^KV = W^DKV h or c^Q = W^DQ h);
// y goes out in bf16, either to a plain [T][n] buffer (c^Q, read by the next
// GEMM) or into the token's paged-cache row (c^KV, next to the RoPE key the
// compress GEMM wrote there).  The norm spans all n features of a token,
// which the GEMM spreads over several 128-row tiles, hence its own pass.
#pragma once

#include "common.cuh"

namespace mla {

struct NormArgs {
  const float* x;             // [T][n] fp32
  int n;
  const __nv_bfloat16* gain;  // [n]
  float eps, scale;
  __nv_bfloat16* out;         // plain destination [T][out_t], or nullptr: the cache row
  long long out_t;
  __nv_bfloat16* pool;        // paged cache [num_blocks][block_size][row]
  const int32_t* table;
  const int32_t* seq_idx;
  const int32_t* pos;
  int num_blocks, max_blocks, block_size, row;
};

constexpr int NORM_THREADS = 128;

// One block per token.  n is a multiple of 4.
__global__ void __launch_bounds__(NORM_THREADS) mla_latent_norm_kernel(const NormArgs a) {
  __shared__ float part[NORM_THREADS / 32];
  pdl_trigger();
  pdl_wait();  // x comes from the GEMM just before
  const int t = blockIdx.x;
  const float4* x = reinterpret_cast<const float4*>(a.x + (long long)t * a.n);
  float acc = 0.f;
  for (int i = threadIdx.x; i < a.n / 4; i += NORM_THREADS) {
    const float4 v = x[i];
    acc = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, acc))));
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < NORM_THREADS / 32; ++w) tot += part[w];
  const float f = a.scale / sqrtf(tot / (float)a.n + a.eps);
  __nv_bfloat16* dst = a.out;
  if (dst) {
    dst += (long long)t * a.out_t;
  } else {
    const long long p = a.pos[t];
    const int page = (int)(p / a.block_size);
    const int blk = (page >= 0 && page < a.max_blocks) ? a.table[(long long)a.seq_idx[t] * a.max_blocks + page] : -1;
    if (blk < 0 || blk >= a.num_blocks) {
      if (threadIdx.x == 0) record_error(ERR_CAPACITY, 602);
      return;
    }
    dst = a.pool + ((long long)blk * a.block_size + p % a.block_size) * a.row;
  }
  for (int i = threadIdx.x; i < a.n / 4; i += NORM_THREADS) {
    const float4 v = x[i];
    const __nv_bfloat162 g01 = *reinterpret_cast<const __nv_bfloat162*>(a.gain + 4 * i);
    const __nv_bfloat162 g23 = *reinterpret_cast<const __nv_bfloat162*>(a.gain + 4 * i + 2);
    const float2 ga = __bfloat1622float2(g01), gb = __bfloat1622float2(g23);
    *reinterpret_cast<uint2*>(dst + 4 * i) =
        make_uint2(pack_bf16(ga.x * (v.x * f), ga.y * (v.y * f)), pack_bf16(gb.x * (v.z * f), gb.y * (v.w * f)));
  }
}

}  // namespace mla
