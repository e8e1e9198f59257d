// simt_f32.cuh — exact fp32 kernels of the MLA layer (CUDA cores).
//
// Used for MLA_F32 layers (the tiny validation layer: d = 64, n_h = 4,
// d_h = 16, d_c = 32, d_h^R = 8), where a 1e-4 relative tolerance rules out
// tf32 tensor-core arithmetic.  Plain FMA in fp32; RoPE angles in fp64.
#pragma once

#include "common.cuh"
#include "rope.cuh"

namespace mla {

struct F32Layer {
  int d, n_h, d_h, d_c, d_cq, d_hr, block_size;
  RopeParams rope;
  float scale_log2;  // softmax scale * log2(e)
  int latent_norm;   // RMSNorm + scale factor on c^KV and c^Q
  float norm_eps, scale_kv, scale_q;
};

// v[0..n) <- scale * g * v / sqrt(mean(v^2) + eps) over the block (the
// latent RMSNorm with its bottleneck scale factor, DeepSeek-V2 explainer,
// adg.csdn.net, section 3.1.1).  All threads of the block call it.
__device__ void f32_rmsnorm_inplace(float* v, int n, const float* __restrict__ g, float eps, float scale) {
  __shared__ float part[32];
  __shared__ float inv;
  float acc = 0.f;
  for (int k = threadIdx.x; k < n; k += blockDim.x) acc = fmaf(v[k], v[k], acc);
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += part[w];
    inv = 1.f / sqrtf(tot / (float)n + eps);
  }
  __syncthreads();
  for (int k = threadIdx.x; k < n; k += blockDim.x) v[k] = scale * g[k] * (v[k] * inv);
  __syncthreads();
}

// y[r] = sum_k W[r, k] x[k] for r in [0, rows), one warp per row.
__device__ __forceinline__ void f32_matvec_warp(const float* __restrict__ W, const float* x, float* y, int rows,
                                                int cols) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = warp; r < rows; r += nw) {
    const float* w = W + (size_t)r * cols;
    float acc = 0.f;
    for (int k = lane; k < cols; k += 32) acc = fmaf(w[k], x[k], acc);
    acc = warp_sum(acc);
    if (lane == 0) y[r] = acc;
  }
}

// Rotate interleaved pairs of v[0..d_hr) in place by pos * theta_k.
__device__ __forceinline__ void f32_rope_inplace(float* v, int d_hr, long long pos, const RopeParams& rp) {
  for (int k = threadIdx.x; k < d_hr / 2; k += blockDim.x) {
    float c, s;
    rope_cos_sin(rp, d_hr, k, pos, &c, &s);
    const float a = v[2 * k], b = v[2 * k + 1];
    v[2 * k] = a * c - b * s;
    v[2 * k + 1] = a * s + b * c;
  }
}

// One block per new token: [c^KV ; RoPE(W^KR h)] -> its cache slot.
__global__ void f32_compress_append_kernel(F32Layer L, const float* __restrict__ h, const float* __restrict__ w_dkv,
                                           const float* __restrict__ w_kr, const float* __restrict__ g_kv,
                                           const int32_t* __restrict__ seq_idx,
                                           const int32_t* __restrict__ pos, float* __restrict__ pool, int num_blocks,
                                           const int32_t* __restrict__ table, int max_blocks) {
  extern __shared__ float sm[];
  const int t = blockIdx.x;
  const int row = L.d_c + L.d_hr;
  float* x = sm;       // [d]
  float* y = sm + L.d; // [row]
  for (int k = threadIdx.x; k < L.d; k += blockDim.x) x[k] = h[(size_t)t * L.d + k];
  __syncthreads();
  f32_matvec_warp(w_dkv, x, y, L.d_c, L.d);
  f32_matvec_warp(w_kr, x, y + L.d_c, L.d_hr, L.d);
  __syncthreads();
  if (L.latent_norm) f32_rmsnorm_inplace(y, L.d_c, g_kv, L.norm_eps, L.scale_kv);
  const long long p = pos[t];
  f32_rope_inplace(y + L.d_c, L.d_hr, p, L.rope);
  __syncthreads();
  const int s = seq_idx[t];
  const int page = (int)(p / L.block_size);
  const int blk = (page >= 0 && page < max_blocks) ? table[(size_t)s * max_blocks + page] : -1;
  if (blk < 0 || blk >= num_blocks) {
    if (threadIdx.x == 0) record_error(ERR_CAPACITY, 101);
    return;
  }
  float* dst = pool + ((size_t)blk * L.block_size + (size_t)(p % L.block_size)) * row;
  for (int k = threadIdx.x; k < row; k += blockDim.x) dst[k] = y[k];
}

// One block per token: q_lat = (W^UK_i)^T W^UQ_i c^Q and q_rope = RoPE(W^QR_i c^Q).
__global__ void f32_absorb_q_kernel(F32Layer L, const float* __restrict__ h, const float* __restrict__ w_dq,
                                    const float* __restrict__ g_q, const float* __restrict__ w_uq,
                                    const float* __restrict__ w_qr,
                                    const float* __restrict__ w_uk, const int32_t* __restrict__ pos,
                                    float* __restrict__ q_lat, float* __restrict__ q_rope) {
  extern __shared__ float sm[];
  const int t = blockIdx.x;
  const int q_in = L.d_cq ? L.d_cq : L.d;
  float* x = sm;                      // [d]
  float* cq = x + L.d;                // [q_in]
  float* qc = cq + q_in;              // [n_h*d_h]
  float* qr = qc + L.n_h * L.d_h;     // [n_h*d_hr]
  for (int k = threadIdx.x; k < L.d; k += blockDim.x) x[k] = h[(size_t)t * L.d + k];
  __syncthreads();
  if (L.d_cq) {
    f32_matvec_warp(w_dq, x, cq, L.d_cq, L.d);
  } else {
    for (int k = threadIdx.x; k < L.d; k += blockDim.x) cq[k] = x[k];
  }
  __syncthreads();
  if (L.d_cq && L.latent_norm) f32_rmsnorm_inplace(cq, L.d_cq, g_q, L.norm_eps, L.scale_q);
  f32_matvec_warp(w_uq, cq, qc, L.n_h * L.d_h, q_in);
  f32_matvec_warp(w_qr, cq, qr, L.n_h * L.d_hr, q_in);
  __syncthreads();
  const long long p = pos[t];
  for (int i = 0; i < L.n_h; ++i) f32_rope_inplace(qr + i * L.d_hr, L.d_hr, p, L.rope);
  __syncthreads();
  for (int e = threadIdx.x; e < L.n_h * L.d_c; e += blockDim.x) {
    const int i = e / L.d_c, c = e % L.d_c;
    const float* wk = w_uk + (size_t)i * L.d_h * L.d_c + c;
    const float* q = qc + i * L.d_h;
    float acc = 0.f;
    for (int j = 0; j < L.d_h; ++j) acc = fmaf(wk[(size_t)j * L.d_c], q[j], acc);
    q_lat[(size_t)t * L.n_h * L.d_c + e] = acc;
  }
  for (int e = threadIdx.x; e < L.n_h * L.d_hr; e += blockDim.x) q_rope[(size_t)t * L.n_h * L.d_hr + e] = qr[e];
}

// One block per (query row, head): scores into scratch, softmax, o_lat.
// Row r belongs to sequence r / q_per_seq; its key count is kv_len[r]
// (decode) or q_start[seq] + r % q_per_seq + 1 (causal prefill).
__global__ void f32_attn_kernel(F32Layer L, const float* __restrict__ q_lat, const float* __restrict__ q_rope,
                                const float* __restrict__ pool, int num_blocks, const int32_t* __restrict__ table,
                                int max_blocks, const int32_t* __restrict__ kv_len, const int32_t* __restrict__ q_start,
                                int q_per_seq, float* __restrict__ scores, int max_len, float* __restrict__ o_lat,
                                float* __restrict__ lse) {
  __shared__ float red[32];
  __shared__ int bad;
  const int r = blockIdx.x, i = blockIdx.y;
  const int seq = r / q_per_seq;
  const int n = kv_len ? kv_len[r] : q_start[seq] + (r % q_per_seq) + 1;
  const int row = L.d_c + L.d_hr;
  const float* ql = q_lat + ((size_t)r * L.n_h + i) * L.d_c;
  const float* qr = q_rope + ((size_t)r * L.n_h + i) * L.d_hr;
  float* sc = scores + ((size_t)r * L.n_h + i) * max_len;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  if (n < 1 || n > max_len) {
    if (threadIdx.x == 0) record_error(ERR_CAPACITY, 102);
    return;
  }
  float m = -INFINITY;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const int blk = table[(size_t)seq * max_blocks + j / L.block_size];
    if (blk < 0 || blk >= num_blocks) {
      bad = 1;
      sc[j] = -INFINITY;
      continue;
    }
    const float* kv = pool + ((size_t)blk * L.block_size + j % L.block_size) * row;
    float acc = 0.f;
    for (int c = 0; c < L.d_c; ++c) acc = fmaf(ql[c], kv[c], acc);
    for (int c = 0; c < L.d_hr; ++c) acc = fmaf(qr[c], kv[L.d_c + c], acc);
    const float z = acc * L.scale_log2;  // log2-domain logit
    sc[j] = z;
    m = fmaxf(m, z);
  }
  // block max
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) record_error(ERR_CAPACITY, 103);
    return;
  }
  m = -INFINITY;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  float l = 0.f;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const float p = exp2f(sc[j] - m);
    sc[j] = p;
    l += p;
  }
  l = warp_sum(l);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = l;
  __syncthreads();
  l = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) l += red[w];
  const float inv_l = 1.f / l;
  for (int c = threadIdx.x; c < L.d_c; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < n; ++j) {
      const int blk = table[(size_t)seq * max_blocks + j / L.block_size];
      acc = fmaf(sc[j], pool[((size_t)blk * L.block_size + j % L.block_size) * row + c], acc);
    }
    o_lat[((size_t)r * L.n_h + i) * L.d_c + c] = acc * inv_l;
  }
  if (lse && threadIdx.x == 0) lse[(size_t)r * L.n_h + i] = (m + log2f(l)) * 0.69314718055994531f;
}

// One block per token: o_i = W^UV_i o_lat_i, u = W^O [o_1; ...; o_nh].
__global__ void f32_out_proj_kernel(F32Layer L, const float* __restrict__ o_lat, const float* __restrict__ w_uv,
                                    const float* __restrict__ w_o, float* __restrict__ u) {
  extern __shared__ float sm[];
  const int t = blockIdx.x;
  float* ol = sm;                         // [n_h*d_c]
  float* o = sm + L.n_h * L.d_c;          // [n_h*d_h]
  for (int k = threadIdx.x; k < L.n_h * L.d_c; k += blockDim.x) ol[k] = o_lat[(size_t)t * L.n_h * L.d_c + k];
  __syncthreads();
  for (int i = 0; i < L.n_h; ++i) f32_matvec_warp(w_uv + (size_t)i * L.d_h * L.d_c, ol + i * L.d_c, o + i * L.d_h, L.d_h, L.d_c);
  __syncthreads();
  f32_matvec_warp(w_o, o, u + (size_t)t * L.d, L.d, L.n_h * L.d_h);
}

}  // namespace mla
