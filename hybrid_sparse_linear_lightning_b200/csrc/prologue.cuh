// QK-RMSNorm + RoPE prologue kernels (CUDA cores, HBM-bound).
//
// QK normalisation is applied in every layer (MiniCPM-SALA paper, summary);
// HyPE keeps RoPE in the linear layers and drops it (NoPE) in the sparse
// layers (acgfav.com "SALA 混合架构"; intelliparadigm.com section 2.2).
// RMSNorm: x / sqrt(mean(x^2) + eps) * w over head_dim, fp32 math.
// RoPE: rotate-half, dims (i, i + D/2) turned by (pos0 + t) * base^(-2i/D).
#pragma once

#include "common.cuh"

namespace sala {

constexpr int kPrologueThreads = 256;

// RoPE inverse frequencies base^(-2i/D), i < D/2, formed in fp64 on the host.
struct RopeFreq {
  double inv[64];
};
constexpr int kRopeTokens = 4;   // tokens per CTA of the linear prologue

// Thread layout: a "row" is one (token, head) vector of D elements, handled by
// TPR = D/16 threads; thread c of the row owns elements [8c, 8c+8) of the
// first half and [D/2 + 8c, D/2 + 8c + 8) of the second (a RoPE pair each).
template <int D>
struct RowLayout {
  static constexpr int TPR = D / 16;
  static constexpr int kRowsPerPass = kPrologueThreads / TPR;
};

// Normalise (and optionally rotate) one row held as two 8-element halves.
template <int D>
__device__ __forceinline__ void norm_row(float* lo, float* hi, const float* w_lo,
                                         const float* w_hi, float eps) {
  constexpr int TPR = D / 16;
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss += lo[e] * lo[e] + hi[e] * hi[e];
#pragma unroll
  for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o, TPR);
  const float r = rsqrtf(ss * (1.0f / D) + eps);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    lo[e] = lo[e] * r * w_lo[e];
    hi[e] = hi[e] * r * w_hi[e];
  }
}

__device__ __forceinline__ void rope_pair8(float* lo, float* hi, const float* c, const float* s) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float x1 = lo[e], x2 = hi[e];
    lo[e] = x1 * c[e] - x2 * s[e];
    hi[e] = x2 * c[e] + x1 * s[e];
  }
}

// cos / sin of (pos0 + t) * theta_i for `ntok` tokens starting at token t0 of
// a sequence of length N (flattened index over batch * N): the argument is
// formed and reduced modulo 2 pi in fp64 (|p| < 2^53), then evaluated in fp32
// on [-pi, pi].
template <int D>
__device__ __forceinline__ void rope_table(float* cs, float* sn, long long tok0, int ntok,
                                           int N, long long pos0, const RopeFreq& rf) {
  for (int e = threadIdx.x; e < ntok * (D / 2); e += blockDim.x) {
    const int tt = e / (D / 2), i = e % (D / 2);
    const long long p = pos0 + (tok0 + tt) % N;
    const double a = (double)p * rf.inv[i];
    const double two_pi = 6.283185307179586476925286766559;
    sincosf((float)(a - rint(a / two_pi) * two_pi), &sn[e], &cs[e]);
  }
}

// Linear-layer prologue: q, k [B*N, H, D] of T -> qn, kn [B*N, H, D] bf16,
// RMSNorm then RoPE.
template <typename T, int D>
__global__ void __launch_bounds__(kPrologueThreads)
linear_prologue_kernel(const T* __restrict__ q, const T* __restrict__ k,
                       const float* __restrict__ wq, const float* __restrict__ wk,
                       __nv_bfloat16* __restrict__ qn, __nv_bfloat16* __restrict__ kn,
                       long long total_tokens, int N, int H, long long pos0,
                       const RopeFreq rf, float eps) {
  constexpr int TPR = D / 16;
  __shared__ float cs[kRopeTokens * D / 2];
  __shared__ float sn[kRopeTokens * D / 2];
  const long long tok0 = (long long)blockIdx.x * kRopeTokens;
  const int ntok = (int)(total_tokens - tok0 < kRopeTokens ? total_tokens - tok0 : kRopeTokens);
  rope_table<D>(cs, sn, tok0, ntok, N, pos0, rf);
  __syncthreads();

  const int c = threadIdx.x % TPR;
  const int rg = threadIdx.x / TPR;
  float wq_lo[8], wq_hi[8], wk_lo[8], wk_hi[8];
  load8(wq + 8 * c, wq_lo);
  load8(wq + D / 2 + 8 * c, wq_hi);
  load8(wk + 8 * c, wk_lo);
  load8(wk + D / 2 + 8 * c, wk_hi);

  // Every thread runs the same number of passes (the row-norm shuffles need
  // whole warps); rows past the end are computed on zeros and not stored.
  const int rows = ntok * H * 2;
  for (int base = 0; base < rows; base += RowLayout<D>::kRowsPerPass) {
    const int r = base + rg;
    const bool active = r < rows;
    const int rc = active ? r : 0;
    const int which = rc / (ntok * H);          // 0: q, 1: k
    const int rr = rc % (ntok * H);
    const int tt = rr / H, h = rr % H;
    const long long off = ((tok0 + tt) * H + h) * (long long)D;
    const T* src = which ? k : q;
    __nv_bfloat16* dst = which ? kn : qn;
    float lo[8], hi[8];
    load8(src + off + 8 * c, lo);
    load8(src + off + D / 2 + 8 * c, hi);
    norm_row<D>(lo, hi, which ? wk_lo : wq_lo, which ? wk_hi : wq_hi, eps);
    rope_pair8(lo, hi, cs + tt * (D / 2) + 8 * c, sn + tt * (D / 2) + 8 * c);
    if (active) {
      store8(dst + off + 8 * c, lo);
      store8(dst + off + D / 2 + 8 * c, hi);
    }
  }
}

// Sparse-layer prologue (NoPE).  One CTA per (batch, block of BLK tokens, kv
// head g): normalises the block's q rows of the group's G heads and its k
// rows of head g, writes them as bf16, and writes the fp32 block sums
//   qbar_sum[b, blk, g] = sum_{h in G(g)} mean_t q^_t^h,  kbar[b, blk, g] = mean_t k^_t^g
// from the normalised values before rounding.  The reduction order is fixed
// (deterministic).
template <typename T, int D>
__global__ void __launch_bounds__(kPrologueThreads)
sparse_prologue_kernel(const T* __restrict__ q, const T* __restrict__ k,
                       const float* __restrict__ wq, const float* __restrict__ wk,
                       __nv_bfloat16* __restrict__ qn, __nv_bfloat16* __restrict__ kn,
                       float* __restrict__ qbar_sum, float* __restrict__ kbar,
                       int N, int Hq, int Hkv, int BLK, float eps) {
  constexpr int TPR = D / 16;
  constexpr int NRG = RowLayout<D>::kRowsPerPass;
  __shared__ float red[NRG][D];

  const int g = blockIdx.x % Hkv;
  const int blk = (blockIdx.x / Hkv);
  const int nb = N / BLK;
  const int b = blk / nb;
  const int jb = blk % nb;
  const int G = Hq / Hkv;
  const int c = threadIdx.x % TPR;
  const int rg = threadIdx.x / TPR;
  const long long tok0 = (long long)b * N + (long long)jb * BLK;

  float w_lo[8], w_hi[8];
  float acc_lo[8], acc_hi[8];
  for (int pass = 0; pass < 2; ++pass) {
    const bool isq = pass == 0;
    load8((isq ? wq : wk) + 8 * c, w_lo);
    load8((isq ? wq : wk) + D / 2 + 8 * c, w_hi);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc_lo[e] = acc_hi[e] = 0.f;
    const int rows = isq ? BLK * G : BLK;
    for (int base = 0; base < rows; base += NRG) {
      const int r0 = base + rg;
      const bool active = r0 < rows;
      const int r = active ? r0 : 0;
      int t, h, H;
      if (isq) { t = r / G; h = g * G + r % G; H = Hq; }
      else { t = r; h = g; H = Hkv; }
      const long long off = ((tok0 + t) * H + h) * (long long)D;
      const T* src = isq ? q : k;
      float lo[8], hi[8];
      load8(src + off + 8 * c, lo);
      load8(src + off + D / 2 + 8 * c, hi);
      norm_row<D>(lo, hi, w_lo, w_hi, eps);
      if (active) {
#pragma unroll
        for (int e = 0; e < 8; ++e) { acc_lo[e] += lo[e]; acc_hi[e] += hi[e]; }
        store8((isq ? qn : kn) + off + 8 * c, lo);
        store8((isq ? qn : kn) + off + D / 2 + 8 * c, hi);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red[rg][8 * c + e] = acc_lo[e];
      red[rg][D / 2 + 8 * c + e] = acc_hi[e];
    }
    __syncthreads();
    if (threadIdx.x < D) {
      float s = 0.f;
      for (int i = 0; i < NRG; ++i) s += red[i][threadIdx.x];
      float* dst = isq ? qbar_sum : kbar;
      dst[(((long long)b * nb + jb) * Hkv + g) * D + threadIdx.x] = s / (float)BLK;
    }
    __syncthreads();
  }
}

}  // namespace sala
