// Decode step: one new token through n_linear linear layers and one sparse
// layer.
//
// Linear layers keep a constant-size state (MiniCPM-SALA paper, section 2.1):
//   S <- lam S + k^T v,   o = scale * q^ S,   out = sigmoid(g) * o
// with q^, k^ RMSNorm'd and RoPE'd at the token's position.
// The sparse layer (NoPE, so cached keys carry no position: acgfav.com
// "SALA 混合架构") appends the normalised key and the value to its cache,
// closes a block mean when a block completes, scores the complete candidate
// blocks against the group-summed normalised query, keeps the top-k plus the
// initial and local blocks (the block holding the token is local), and runs
// exact softmax attention over them (split over blocks, then combined).
#pragma once

#include "common.cuh"
#include "prologue.cuh"
#include "select.cuh"

namespace sala {

struct DecodeLinearArgs {
  const void* q[8];
  const void* k[8];
  const void* v[8];
  const void* gate[8];
  const float* wq[8];
  const float* wk[8];
  const float* lambda[8];
  float* state[8];
  void* out[8];
};

// One CTA per (layer, batch, head, 64-column slice); 256 threads = 64 columns
// x 4 row groups.  Reads and rewrites its slice of S once (HBM-bound).
template <typename T, int D>
__global__ void __launch_bounds__(256)
decode_linear_kernel(DecodeLinearArgs a, int B, int H, long long pos, double log2_base,
                     float eps, float scale) {
  constexpr int NSL = D / 64;
  __shared__ float qh[D], kh[D], vv[D];
  __shared__ float part[4][64];
  const int slice = blockIdx.x % NSL;
  const int h = (blockIdx.x / NSL) % H;
  const int b = (blockIdx.x / (NSL * H)) % B;
  const int layer = blockIdx.x / (NSL * H * B);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long voff = ((long long)b * H + h) * D;
  const T* q = static_cast<const T*>(a.q[layer]);
  const T* k = static_cast<const T*>(a.k[layer]);
  const T* v = static_cast<const T*>(a.v[layer]);
  // warps 0 / 1 normalise + rotate q / k (one lane per element pair)
  if (warp < 2) {
    const T* src = warp == 0 ? q : k;
    const float* w = warp == 0 ? a.wq[layer] : a.wk[layer];
    float* dst = warp == 0 ? qh : kh;
    float ss = 0.f;
    for (int e = lane; e < D; e += 32) { const float x = to_f32(src[voff + e]); ss += x * x; }
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / D + eps);
    for (int i = lane; i < D / 2; i += 32) {
      const float x1 = to_f32(src[voff + i]) * r * w[i];
      const float x2 = to_f32(src[voff + i + D / 2]) * r * w[i + D / 2];
      double sv, cv;
      sincos((double)pos * exp2(-2.0 * i / D * log2_base), &sv, &cv);
      const float c = (float)cv, s = (float)sv;
      dst[i] = x1 * c - x2 * s;
      dst[i + D / 2] = x2 * c + x1 * s;
    }
  } else if (warp == 2) {
    for (int e = lane; e < D; e += 32) vv[e] = to_f32(v[voff + e]);
  }
  __syncthreads();
  const int col = slice * 64 + (tid & 63);
  const int rg = tid >> 6;
  const float lam = a.lambda[layer][h];
  float* S = a.state[layer] + ((long long)b * H + h) * D * D;
  const float vc = vv[col];
  float acc = 0.f;
  for (int r = rg * (D / 4); r < (rg + 1) * (D / 4); ++r) {
    const float sn = lam * S[(long long)r * D + col] + kh[r] * vc;
    S[(long long)r * D + col] = sn;
    acc = fmaf(qh[r], sn, acc);
  }
  part[rg][tid & 63] = acc;
  __syncthreads();
  if (tid < 64) {
    const float o = scale * (part[0][tid] + part[1][tid] + part[2][tid] + part[3][tid]);
    const T* g = static_cast<const T*>(a.gate[layer]);
    T* out = static_cast<T*>(a.out[layer]);
    out[voff + col] = from_f32<T>(sigmoidf_(to_f32(g[voff + col])) * o);
  }
}

// Sparse layer, step 1 (one CTA per batch): normalise k (append to the cache,
// update the running block sum / block mean), copy v, normalise q and form
// the group sums.
template <typename T, int D>
__global__ void __launch_bounds__(256)
decode_sparse_prep_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                          const float* __restrict__ wq, const float* __restrict__ wk,
                          __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache,
                          float* __restrict__ kbar, float* __restrict__ ksum,
                          float* __restrict__ qhat, float* __restrict__ qgrp,
                          int Hq, int Hkv, long long cap, long long pos, int BLK, float eps) {
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = Hq / Hkv;
  const bool closes = ((pos + 1) % BLK) == 0;
  // rows: Hkv key rows, then Hq query rows; one warp per row
  for (int r = warp; r < Hkv + Hq; r += 8) {
    const bool isk = r < Hkv;
    const int h = isk ? r : r - Hkv;
    const T* src = isk ? k + ((long long)b * Hkv + h) * D : q + ((long long)b * Hq + h) * D;
    const float* w = isk ? wk : wq;
    float x[D / 32];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) { x[e] = to_f32(src[lane + 32 * e]); ss += x[e] * x[e]; }
    ss = warp_sum(ss);
    const float rn = rsqrtf(ss / D + eps);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) x[e] = x[e] * rn * w[lane + 32 * e];
    if (isk) {
      const long long crow = (((long long)b * cap + pos) * Hkv + h) * D;
      float* ks = ksum + ((long long)b * Hkv + h) * D;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) {
        const int d = lane + 32 * e;
        k_cache[crow + d] = __float2bfloat16_rn(x[e]);
        v_cache[crow + d] = __float2bfloat16_rn(to_f32(v[((long long)b * Hkv + h) * D + d]));
        const float s = ks[d] + x[e];
        if (closes) {
          kbar[(((long long)b * (cap / BLK) + pos / BLK) * Hkv + h) * D + d] = s / (float)BLK;
          ks[d] = 0.f;
        } else {
          ks[d] = s;
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < D / 32; ++e) qhat[((long long)b * Hq + h) * D + lane + 32 * e] = x[e];
    }
  }
  __syncthreads();
  // group sums of the normalised queries (fixed order)
  for (int e = tid; e < Hkv * D; e += 256) {
    const int g = e / D, d = e % D;
    float s = 0.f;
    for (int hh = 0; hh < G; ++hh) s += qhat[((long long)b * Hq + g * G + hh) * D + d];
    qgrp[((long long)b * Hkv + g) * D + d] = s;
  }
}

// Sparse layer, step 2: candidate scores, one warp per candidate block.
template <int D>
__global__ void __launch_bounds__(256)
decode_scores_kernel(const float* __restrict__ qgrp, const float* __restrict__ kbar,
                     uint32_t* __restrict__ keys, int Hkv, long long cap_blocks, int n_init,
                     int n_cand, long long total_warps) {
  const int lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (gw >= total_warps) return;
  const int c = (int)(gw % n_cand);
  const int g = (int)((gw / n_cand) % Hkv);
  const int b = (int)(gw / ((long long)n_cand * Hkv));
  const float* kr = kbar + (((long long)b * cap_blocks + n_init + c) * Hkv + g) * D;
  const float* qg = qgrp + ((long long)b * Hkv + g) * D;
  float p = 0.f;
#pragma unroll
  for (int e = lane; e < D; e += 32) p = fmaf(qg[e], kr[e], p);
  p = warp_sum(p);
  if (lane == 0) keys[((long long)b * Hkv + g) * cap_blocks + c] = score_key(p * rsqrtf((float)D));
}

// Sparse layer, step 3: selection, one CTA per (batch, kv head).  Dynamic smem:
// n_cand uint32 keys.
__global__ void __launch_bounds__(kSelectThreads)
decode_topk_kernel(const uint32_t* __restrict__ keys_g, int32_t* __restrict__ idx, int Hkv,
                   long long cap_blocks, int bcur, int topk, int n_init, int n_local, int width) {
  extern __shared__ uint32_t keys[];
  __shared__ int hist[256];
  __shared__ int scan_scratch[kSelectThreads / 32 + 1];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  const int g = blockIdx.x % Hkv, b = blockIdx.x / Hkv;
  const int tid = threadIdx.x;
  int32_t* row = idx + ((long long)b * Hkv + g) * width;
  const int n_cand = max(0, bcur - n_local + 1 - n_init);
  const int k = min(topk, n_cand);
  const int n_first = min(n_init, bcur + 1);
  for (int e = tid; e < n_first; e += kSelectThreads) row[e] = e;
  const int local_lo = max(n_init, bcur - n_local + 1);
  const int n_loc = max(0, bcur - local_lo + 1);
  for (int e = tid; e < n_loc; e += kSelectThreads) row[n_first + k + e] = local_lo + e;
  for (int e = n_first + k + n_loc + tid; e < width; e += kSelectThreads) row[e] = -1;
  if (k == 0) return;
  if (k == n_cand) {
    for (int e = tid; e < n_cand; e += kSelectThreads) row[n_first + e] = n_init + e;
    return;
  }
  const uint32_t* src = keys_g + ((long long)b * Hkv + g) * cap_blocks;
  for (int c = tid; c < n_cand; c += kSelectThreads) keys[c] = src[c];
  __syncthreads();
  topk_emit_sorted(keys, n_cand, k, row + n_first, n_init, hist, scan_scratch, &s_prefix, &s_need);
}

// Sparse layer, step 4: partial attention of the group's G heads over one
// selected block.  One CTA per (batch, kv head, index slot); one warp per head
// (heads strided over 8 warps).  Writes (m, l, o[D]) per head, in base-2
// logits, or m = -inf for an empty slot.
template <int D>
__global__ void __launch_bounds__(256)
decode_attn_kernel(const float* __restrict__ qhat, const __nv_bfloat16* __restrict__ k_cache,
                   const __nv_bfloat16* __restrict__ v_cache, const int32_t* __restrict__ idx,
                   float* __restrict__ part, int Hq, int Hkv, long long cap, long long pos,
                   int BLK, int width, float scale) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float (*ks)[D + 1] = reinterpret_cast<float (*)[D + 1]>(smem_raw);
  float (*vs)[D] = reinterpret_cast<float (*)[D]>(smem_raw + sizeof(float) * 64 * (D + 1));
  const int slot = blockIdx.x % width;
  const int g = (blockIdx.x / width) % Hkv;
  const int b = blockIdx.x / (width * Hkv);
  const int G = Hq / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = idx[((long long)b * Hkv + g) * width + slot];
  float* pbase = part + (((long long)b * Hkv + g) * width + slot) * G * (D + 2);
  if (j < 0 || (long long)j * BLK > pos) {
    if (j >= 0) set_status(kStatusBounds);
    for (int e = tid; e < G; e += 256) pbase[e * (D + 2)] = -INFINITY;
    return;
  }
  const long long kend = ((long long)(j + 1) * BLK < pos + 1) ? (long long)(j + 1) * BLK : pos + 1;
  const int nk = (int)(kend - (long long)j * BLK);
  for (int e = tid; e < 64 * D; e += 256) {
    const int r = e / D, d = e % D;
    float kv = 0.f, vv2 = 0.f;
    if (r < nk) {
      const long long off = (((long long)b * cap + (long long)j * BLK + r) * Hkv + g) * D + d;
      kv = __bfloat162float(k_cache[off]);
      vv2 = __bfloat162float(v_cache[off]);
    }
    ks[r][d] = kv;
    vs[r][d] = vv2;
  }
  __syncthreads();
  const float sl2 = scale * 1.4426950408889634f;
  for (int hh = warp; hh < G; hh += 8) {
    const float* qv = qhat + ((long long)b * Hq + g * G + hh) * D;
    float s0 = 0.f, s1 = 0.f;
    for (int d = 0; d < D; ++d) {
      const float x = qv[d];
      s0 = fmaf(x, ks[lane][d], s0);
      s1 = fmaf(x, ks[lane + 32][d], s1);
    }
    s0 = lane < nk ? s0 * sl2 : -INFINITY;
    s1 = lane + 32 < nk ? s1 * sl2 : -INFINITY;
    const float m = warp_max(fmaxf(s0, s1));
    const float p0 = exp2f(s0 - m), p1 = exp2f(s1 - m);
    const float l = warp_sum(p0 + p1);
    float* pr = pbase + hh * (D + 2);
    for (int d = lane; d < D; d += 32) {
      float o = 0.f;
      for (int kk = 0; kk < 32; ++kk) {
        o = fmaf(__shfl_sync(0xffffffffu, p0, kk), vs[kk][d], o);
        o = fmaf(__shfl_sync(0xffffffffu, p1, kk), vs[kk + 32][d], o);
      }
      pr[2 + d] = o;
    }
    if (lane == 0) { pr[0] = m; pr[1] = l; }
  }
}

// Sparse layer, step 5: combine the per-block partials of each head and gate.
template <typename T, int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const float* __restrict__ part, const T* __restrict__ gate,
                      T* __restrict__ out, int Hq, int Hkv, int width) {
  const int h = blockIdx.x % Hq, b = blockIdx.x / Hq;
  const int G = Hq / Hkv, g = h / G, hh = h % G;
  const int d = threadIdx.x;
  const float* pb = part + (((long long)b * Hkv + g) * width) * G * (D + 2) + hh * (D + 2);
  float m = -INFINITY;
  for (int s = 0; s < width; ++s) m = fmaxf(m, pb[(long long)s * G * (D + 2)]);
  float l = 0.f, o = 0.f;
  for (int s = 0; s < width; ++s) {
    const float* pr = pb + (long long)s * G * (D + 2);
    if (pr[0] == -INFINITY) continue;
    const float c = exp2f(pr[0] - m);
    l = fmaf(c, pr[1], l);
    o = fmaf(c, pr[2 + d], o);
  }
  const long long off = ((long long)b * Hq + h) * D + d;
  out[off] = from_f32<T>(sigmoidf_(to_f32(gate[off])) * o / l);
}

}  // namespace sala
