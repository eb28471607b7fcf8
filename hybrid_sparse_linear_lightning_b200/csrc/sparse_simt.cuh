// Gathered block-sparse attention on CUDA cores (fp32).  Cross-check of the
// tensor-core kernel and fallback for shapes it does not cover.
//
// Each query token t of block i and q head h attends, with exact softmax of
// logits * scale, to every key s <= t in the blocks listed for (kv head
// h / G, block i); the output is sigmoid(gate) * attention (output gate after
// each block: MiniCPM-SALA paper, summary).  NoPE: no rotation here.
#pragma once

#include "common.cuh"

namespace sala {

constexpr int kSpSimtThreads = 256;
constexpr int kSpSimtRowsPerWarp = 8;

template <int D>
struct SpSimtSmem {
  float k[64][D + 1];
  float v[64][D];
  float q[kSpSimtThreads / 32][kSpSimtRowsPerWarp][D];
  int sel[1024];
};

// One CTA per (batch, query block i, kv head g); rows are (token, head) pairs
// of the block's BLK=64 tokens and the group's G heads.
template <typename T, int D>
__global__ void __launch_bounds__(kSpSimtThreads)
sparse_attn_simt_kernel(const __nv_bfloat16* __restrict__ qn, const __nv_bfloat16* __restrict__ kn,
                        const T* __restrict__ v, const T* __restrict__ gate,
                        const int32_t* __restrict__ idx, T* __restrict__ out,
                        int N, int Hq, int Hkv, int width, float scale) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SpSimtSmem<D>& sm = *reinterpret_cast<SpSimtSmem<D>*>(smem_raw);
  constexpr int BLK = 64;
  constexpr int DL = D / 32;                 // output dims per lane
  const int nb = N / BLK;
  const int g = blockIdx.x % Hkv;
  const int i = (blockIdx.x / Hkv) % nb;
  const int b = blockIdx.x / (Hkv * nb);
  const int G = Hq / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float sl2 = scale * 1.4426950408889634f;   // logits in base 2

  const int32_t* row = idx + (((long long)b * Hkv + g) * nb + i) * width;
  int nsel = 0;
  for (int e = 0; e < width; ++e) {
    const int j = row[e];
    if (j < 0) break;
    if (tid == 0) sm.sel[e] = (j <= i) ? j : -1;
    if (j > i) set_status(kStatusBounds);
    ++nsel;
  }
  // a valid row lists at least the query's own block; rows with no visible
  // key get a zero output and the bounds bit
  if (nsel == 0 && tid == 0) set_status(kStatusBounds);
  __syncthreads();

  const int rows = BLK * G;
  const int rows_per_pass = (kSpSimtThreads / 32) * kSpSimtRowsPerWarp;
  for (int r0 = 0; r0 < rows; r0 += rows_per_pass) {
    // this warp's rows: r = r0 + warp * 8 + rr -> token r / G, head g*G + r % G
    for (int rr = 0; rr < kSpSimtRowsPerWarp; ++rr) {
      const int r = min(rows - 1, r0 + warp * kSpSimtRowsPerWarp + rr);
      const int t = r / G, h = g * G + r % G;
      const long long off = (((long long)b * N + (long long)i * BLK + t) * Hq + h) * D;
      for (int e = lane; e < D; e += 32) sm.q[warp][rr][e] = __bfloat162float(qn[off + e]);
    }
    float m[kSpSimtRowsPerWarp], l[kSpSimtRowsPerWarp], o[kSpSimtRowsPerWarp][DL];
#pragma unroll
    for (int rr = 0; rr < kSpSimtRowsPerWarp; ++rr) {
      m[rr] = -INFINITY;
      l[rr] = 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) o[rr][e] = 0.f;
    }
    for (int s = 0; s < nsel; ++s) {
      const int j = sm.sel[s];
      __syncthreads();
      if (j >= 0) {
        for (int e = tid; e < BLK * D; e += kSpSimtThreads) {
          const int kr = e / D, d = e % D;
          const long long off = (((long long)b * N + (long long)j * BLK + kr) * Hkv + g) * D + d;
          sm.k[kr][d] = __bfloat162float(kn[off]);
          sm.v[kr][d] = to_f32(v[off]);
        }
      }
      __syncthreads();
      if (j < 0) continue;
#pragma unroll
      for (int rr = 0; rr < kSpSimtRowsPerWarp; ++rr) {
        const int r = r0 + warp * kSpSimtRowsPerWarp + rr;
        const int t = min(rows - 1, r) / G;
        float s0 = 0.f, s1 = 0.f;
        for (int d = 0; d < D; ++d) {
          const float qv = sm.q[warp][rr][d];
          s0 = fmaf(qv, sm.k[lane][d], s0);
          s1 = fmaf(qv, sm.k[lane + 32][d], s1);
        }
        s0 *= sl2;
        s1 *= sl2;
        if (j == i) {                        // causal mask inside the diagonal block
          if (lane > t) s0 = -INFINITY;
          if (lane + 32 > t) s1 = -INFINITY;
        }
        const float mx = warp_max(fmaxf(s0, s1));
        const float mnew = fmaxf(m[rr], mx);
        const float corr = exp2f(m[rr] - mnew);
        const float p0 = exp2f(s0 - mnew), p1 = exp2f(s1 - mnew);
        l[rr] = l[rr] * corr + warp_sum(p0 + p1);
        m[rr] = mnew;
#pragma unroll
        for (int e = 0; e < DL; ++e) o[rr][e] *= corr;
        for (int kk = 0; kk < 32; ++kk) {
          const float pa = __shfl_sync(0xffffffffu, p0, kk);
          const float pb = __shfl_sync(0xffffffffu, p1, kk);
#pragma unroll
          for (int e = 0; e < DL; ++e)
            o[rr][e] = fmaf(pa, sm.v[kk][lane + 32 * e], fmaf(pb, sm.v[kk + 32][lane + 32 * e], o[rr][e]));
        }
      }
    }
#pragma unroll
    for (int rr = 0; rr < kSpSimtRowsPerWarp; ++rr) {
      const int r = r0 + warp * kSpSimtRowsPerWarp + rr;
      if (r >= rows) continue;
      const int t = r / G, h = g * G + r % G;
      const long long off = (((long long)b * N + (long long)i * BLK + t) * Hq + h) * D;
      const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) {
        const int d = lane + 32 * e;
        out[off + d] = from_f32<T>(sigmoidf_(to_f32(gate[off + d])) * o[rr][e] * inv);
      }
    }
    __syncthreads();
  }
}

}  // namespace sala
