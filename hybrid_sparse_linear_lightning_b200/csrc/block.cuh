// Element-wise kernels of the decoder block around the attention: the two
// pre-norms (RMSNorm of the fp32 residual stream into bf16 GEMM operands)
// and the SwiGLU gate of the feed-forward network.  Every attention block is
// followed by an FFN block (MiniCPM-SALA paper, section 2.1).  The GEMMs of
// the block are plain dense products and run in cuBLASLt.
#pragma once

#include "common.cuh"

namespace sala {

constexpr int kBlkNormThreads = 256;

// y[m, :] = bf16(x[m, :] / sqrt(mean(x[m, :]^2) + eps) * w), one CTA per row,
// fp32 math.  hidden must be a multiple of 8.
__global__ void __launch_bounds__(kBlkNormThreads)
block_rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ w,
                     __nv_bfloat16* __restrict__ y, int hidden, float eps) {
  __shared__ float red[kBlkNormThreads / 32];
  __shared__ float s_r;
  const long long row = blockIdx.x;
  const float* xr = x + row * hidden;
  float ss = 0.f;
  for (int e = threadIdx.x * 8; e < hidden; e += kBlkNormThreads * 8) {
    float v[8];
    load8(xr + e, v);
#pragma unroll
    for (int u = 0; u < 8; ++u) ss = fmaf(v[u], v[u], ss);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < kBlkNormThreads / 32 ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) s_r = rsqrtf(t / hidden + eps);
  }
  __syncthreads();
  const float r = s_r;
  for (int e = threadIdx.x * 8; e < hidden; e += kBlkNormThreads * 8) {
    float v[8], wv[8];
    load8(xr + e, v);
    load8(w + e, wv);
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = v[u] * r * wv[u];
    store8(y + row * hidden + e, v);
  }
}

// s[m, j] = bf16(silu(u[m, j]) * u[m, ffn + j]) for the fused W1 | W3
// product u [M, 2 ffn]; 8 columns per thread.  ffn must be a multiple of 8.
__global__ void __launch_bounds__(256)
block_swiglu_kernel(const __nv_bfloat16* __restrict__ u, __nv_bfloat16* __restrict__ s,
                    long long rows, int ffn) {
  const long long per_row = ffn / 8;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * per_row) return;
  const long long m = i / per_row;
  const int j = (int)(i % per_row) * 8;
  float a[8], b[8];
  load8(u + m * 2 * ffn + j, a);
  load8(u + m * 2 * ffn + ffn + j, b);
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] = a[e] * __fdividef(1.f, 1.f + __expf(-a[e])) * b[e];
  store8(s + m * ffn + j, a);
}

}  // namespace sala
