// Token-level block selection of the sparse layer (selection variant 1).
//
// Reading of the InfLLM-V2 block selection the pages name (MiniCPM-SALA
// paper, summary and section 2.1; acgfav.com "SALA 混合架构": a fine-grained
// block selection lets each query attend to a small set of key blocks):
// every query token t of query block i and every q head h of kv group g
// scores each candidate key block j in [n_init, i - n_local] against the
// block's mean normalised key, z = <q^_t^h, kbar_j> / sqrt(d); a softmax over
// the candidates turns one (token, head)'s scores into a distribution, and
// the importance of block j is the mass all 64 tokens and all G heads give
// it.  The top-k blocks by importance (ties to the lower block) join the
// initial and local blocks, emitted ascending and -1 padded.
//
// One CTA per (batch, kv head, query block), fp32 on CUDA cores: the ranking
// must agree with an fp64 evaluation to well within a relative 1e-3.  The
// 64 G rows are taken 128 at a time (normalised from the raw queries into
// shared memory, transposed); per row chunk, pass 1 forms each row's
// log-sum-exp over all candidates and pass 2 adds the normalised
// probabilities into the per-candidate importance.  Every reduction has a
// fixed order, so the result is deterministic.
#pragma once

#include "common.cuh"
#include "select.cuh"

namespace sala {

constexpr int kTsThreads = 256;
constexpr int kTsRows = 128;           // query rows per chunk
constexpr int kTsCands = 64;           // candidate blocks per tile
constexpr int kTsMaxCand = 8192;       // importance accumulators held in shared memory

template <int D>
struct TsLayout {
  static constexpr int kQT = 0;                                   // float [D][kTsRows]
  static constexpr int kKT = kQT + D * kTsRows * 4;               // float [kTsCands][D]
  static constexpr int kML = kKT + D * kTsCands * 4;              // float [8][kTsRows][2]
  static constexpr int kLse = kML + 8 * kTsRows * 2 * 4;          // float [kTsRows]
  static constexpr int kImp = kLse + kTsRows * 4;                 // float / key [n_cand]
  static size_t bytes(int n_cand) { return (size_t)kImp + (size_t)n_cand * 4; }
};

// 4 rows x 8 candidates of dot products for one thread: rows r0..r0+3 of the
// transposed query chunk qT [D][kTsRows] (one 16-byte load per d, consecutive
// across the warp's lanes) and candidates c0..c0+7 of the key tile
// kT [kTsCands][D] (16-byte loads, the same address for the whole warp).
template <int D>
__device__ __forceinline__ void ts_dots(const float* qT, const float* kT, int r0, int c0,
                                        float acc[4][8]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;
#pragma unroll 2
  for (int d = 0; d < D; d += 4) {
    float qa[4][4], kc[8][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 v = *reinterpret_cast<const float4*>(qT + (d + u) * kTsRows + r0);
      qa[u][0] = v.x; qa[u][1] = v.y; qa[u][2] = v.z; qa[u][3] = v.w;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 v = *reinterpret_cast<const float4*>(kT + (c0 + c) * D + d);
      kc[c][0] = v.x; kc[c][1] = v.y; kc[c][2] = v.z; kc[c][3] = v.w;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(qa[u][a], kc[c][u], acc[a][c]);
  }
}

// Candidate tile [ct, ct + kTsCands) of (b, g) into kT [kTsCands][D] (zeros
// past the last candidate).
template <int D>
__device__ __forceinline__ void ts_stage_keys(float* kT, const float* __restrict__ kbar, int b,
                                              int g, int nb, int Hkv, int n_init, int ct,
                                              int n_cand) {
  constexpr int V = D / 4;
  for (int e = threadIdx.x; e < kTsCands * V; e += kTsThreads) {
    const int cc = e / V, d4 = e % V;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ct + cc < n_cand)
      v = reinterpret_cast<const float4*>(kbar + (((long long)b * nb + n_init + ct + cc) * Hkv + g) * D)[d4];
    reinterpret_cast<float4*>(kT + cc * D)[d4] = v;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kTsThreads)
select_token_softmax_kernel(const T* __restrict__ q, const float* __restrict__ wq,
                            const float* __restrict__ kbar, int32_t* __restrict__ idx, int nb,
                            int Hq, int Hkv, int topk, int n_init, int n_local, int width,
                            float eps) {
  using L = TsLayout<D>;
  extern __shared__ __align__(16) unsigned char ts_smem[];
  float* qT = reinterpret_cast<float*>(ts_smem + L::kQT);
  float* kT = reinterpret_cast<float*>(ts_smem + L::kKT);
  float* ml = reinterpret_cast<float*>(ts_smem + L::kML);
  float* lse = reinterpret_cast<float*>(ts_smem + L::kLse);
  float* imp = reinterpret_cast<float*>(ts_smem + L::kImp);
  __shared__ int hist[256];
  __shared__ int scan_scratch[kTsThreads / 32 + 1];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;

  const int i = blockIdx.x % nb;
  const int g = (blockIdx.x / nb) % Hkv;
  const int b = blockIdx.x / (nb * Hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = Hq / Hkv;
  const int N = nb * 64;
  int32_t* row = idx + (((long long)b * Hkv + g) * nb + i) * width;

  const int n_cand = max(0, i - n_local + 1 - n_init);
  const int k = min(topk, n_cand);
  const int n_first = min(n_init, i + 1);
  const int local_lo = max(n_init, i - n_local + 1);
  const int n_loc = max(0, i - local_lo + 1);
  for (int e = tid; e < n_first; e += kTsThreads) row[e] = e;
  for (int e = tid; e < n_loc; e += kTsThreads) row[n_first + k + e] = local_lo + e;
  for (int e = n_first + k + n_loc + tid; e < width; e += kTsThreads) row[e] = -1;
  if (k == 0) return;
  if (k == n_cand) {
    for (int e = tid; e < n_cand; e += kTsThreads) row[n_first + e] = n_init + e;
    return;
  }

  for (int c = tid; c < n_cand; c += kTsThreads) imp[c] = 0.f;
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);   // base-2 logits
  const int n_rows = 64 * G;
  const int r0 = lane * 4, c0 = warp * 8;
  for (int rc = 0; rc < n_rows; rc += kTsRows) {
    // ---- normalised query rows of this chunk, transposed: row rr = (head
    // rc/64 + rr/64 of the group, token rr % 64); two threads per row
    __syncthreads();
    {
      const int rr = tid >> 1, half = tid & 1;
      const int rho = rc + rr;
      float x[D / 2];
      float ss = 0.f;
      if (rho < n_rows) {
        const int h = g * G + rho / 64, t = rho % 64;
        const T* src = q + (((long long)b * N + (long long)i * 64 + t) * Hq + h) * D + half * (D / 2);
#pragma unroll
        for (int e = 0; e < D / 2; e += 8) load8(src + e, x + e);
#pragma unroll
        for (int e = 0; e < D / 2; ++e) ss = fmaf(x[e], x[e], ss);
      } else {
#pragma unroll
        for (int e = 0; e < D / 2; ++e) x[e] = 0.f;
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      const float rn = rsqrtf(ss * (1.0f / D) + eps);
#pragma unroll
      for (int e = 0; e < D / 2; ++e)
        qT[(half * (D / 2) + e) * kTsRows + rr] = x[e] * rn * wq[half * (D / 2) + e];
    }
    // ---- pass 1: per-row log-sum-exp (base 2) over all candidates
    float m[4], l[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) { m[a] = -INFINITY; l[a] = 0.f; }
    for (int ct = 0; ct < n_cand; ct += kTsCands) {
      __syncthreads();
      ts_stage_keys<D>(kT, kbar, b, g, nb, Hkv, n_init, ct, n_cand);
      __syncthreads();
      float acc[4][8];
      ts_dots<D>(qT, kT, r0, c0, acc);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        float mx = m[a];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (ct + c0 + c < n_cand) mx = fmaxf(mx, acc[a][c] * sl2);
        float s = l[a] * exp2f(m[a] - mx);
        if (mx == -INFINITY) s = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (ct + c0 + c < n_cand) s += exp2f(acc[a][c] * sl2 - mx);
        m[a] = mx;
        l[a] = s;
      }
    }
    // combine the 8 warps' partial (m, l) of each row, in warp order
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      ml[(warp * kTsRows + r0 + a) * 2] = m[a];
      ml[(warp * kTsRows + r0 + a) * 2 + 1] = l[a];
    }
    __syncthreads();
    if (tid < kTsRows) {
      float M = -INFINITY;
      for (int w = 0; w < 8; ++w) M = fmaxf(M, ml[(w * kTsRows + tid) * 2]);
      float S = 0.f;
      for (int w = 0; w < 8; ++w) {
        const float mw = ml[(w * kTsRows + tid) * 2];
        if (mw != -INFINITY) S += ml[(w * kTsRows + tid) * 2 + 1] * exp2f(mw - M);
      }
      lse[tid] = M + log2f(S);
    }
    __syncthreads();
    float ls[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) ls[a] = lse[r0 + a];
    // ---- pass 2: importance += sum over this chunk's rows of 2^(z - lse)
    for (int ct = 0; ct < n_cand; ct += kTsCands) {
      __syncthreads();
      ts_stage_keys<D>(kT, kbar, b, g, nb, Hkv, n_init, ct, n_cand);
      __syncthreads();
      float acc[4][8];
      ts_dots<D>(qT, kT, r0, c0, acc);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float s = 0.f;
#pragma unroll
        for (int a = 0; a < 4; ++a)
          if (rc + r0 + a < n_rows) s += exp2f(acc[a][c] * sl2 - ls[a]);
        s = warp_sum(s);                      // the warp's 128 rows, fixed tree
        if (lane == 0 && ct + c0 + c < n_cand) imp[ct + c0 + c] += s;
      }
    }
  }
  __syncthreads();
  // ---- top-k by importance (exact, ties to the lower block)
  uint32_t* keys = reinterpret_cast<uint32_t*>(imp);
  for (int c = tid; c < n_cand; c += kTsThreads) keys[c] = score_key(imp[c]);
  __syncthreads();
  topk_emit_sorted<kTsThreads>(keys, n_cand, k, row + n_first, n_init, hist, scan_scratch,
                               &s_prefix, &s_need);
}

}  // namespace sala
