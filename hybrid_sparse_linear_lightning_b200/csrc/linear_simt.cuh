// Chunked linear attention on CUDA cores (fp32 FMA).  Used as an independent
// cross-check of the tensor-core kernel and for shapes it does not cover.
//
// Lightning attention, chunk-wise (acgfav.com "SALA 混合架构": linear layers
// at O(N); paper section 2.1: constant-size state).  Per chunk of C tokens:
//   O_intra = (Q_c K_c^T . D) V_c,          D_ij = lam^(i-j) (j <= i), else 0
//   O_inter = diag(lam^(i+1)) Q_c S_prev
//   S_new   = lam^C S_prev + (diag(lam^(C-1-j)) K_c)^T V_c
//   out     = sigmoid(G) . scale (O_intra + O_inter)
// One CTA owns (batch, head, 32 value columns); the fp32 state slice
// S[:, cols] stays in shared memory for the whole sequence.
#pragma once

#include "common.cuh"

namespace sala {

constexpr int kSimtChunk = 64;
constexpr int kSimtCols = 32;
constexpr int kSimtThreads = 256;

template <int D>
struct SimtSmem {
  float qt[D][kSimtChunk];          // Q^T of the chunk
  float kt[D][kSimtChunk];          // K^T of the chunk
  float v[kSimtChunk][kSimtCols];   // V slice
  float at[kSimtChunk][kSimtChunk + 1];  // (Q K^T . D)^T, padded
  float s[D][kSimtCols];            // state slice
  float pw[kSimtChunk + 1];         // lam^m, m = 0..C
};

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads)
linear_chunk_simt_kernel(const __nv_bfloat16* __restrict__ qn, const __nv_bfloat16* __restrict__ kn,
                         const T* __restrict__ v, const T* __restrict__ gate,
                         const float* __restrict__ lambda, const float* __restrict__ state_in,
                         float* __restrict__ state_out, T* __restrict__ out,
                         int N, int H, float scale) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem<D>& sm = *reinterpret_cast<SimtSmem<D>*>(smem_raw);
  constexpr int C = kSimtChunk;
  constexpr int NS = D / kSimtCols;        // column slices per head
  const int slice = blockIdx.x % NS;
  const int h = (blockIdx.x / NS) % H;
  const int b = blockIdx.x / (NS * H);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col0 = slice * kSimtCols;
  const float lam = lambda[h];

  if (tid <= C) sm.pw[tid] = (float)pow((double)lam, (double)tid);
  const long long sbase = ((long long)b * H + h) * D * D;
  for (int e = tid; e < D * kSimtCols; e += kSimtThreads) {
    const int r = e / kSimtCols, c = e % kSimtCols;
    sm.s[r][c] = state_in ? state_in[sbase + (long long)r * D + col0 + c] : 0.f;
  }
  __syncthreads();
  const float lamC = sm.pw[C];

  for (int c0 = 0; c0 < N; c0 += C) {
    const long long tok0 = (long long)b * N + c0;
    // 1. load Q^T, K^T (bf16 -> fp32) and the V slice
    for (int item = tid; item < C * (D / 8); item += kSimtThreads) {
      const int i = item % C, kg = item / C;
      const long long off = ((tok0 + i) * H + h) * (long long)D + 8 * kg;
      float fq[8], fk[8];
      load8(qn + off, fq);
      load8(kn + off, fk);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sm.qt[8 * kg + e][i] = fq[e];
        sm.kt[8 * kg + e][i] = fk[e];
      }
    }
    for (int item = tid; item < C * (kSimtCols / 8); item += kSimtThreads) {
      const int j = item / (kSimtCols / 8), cg = item % (kSimtCols / 8);
      float fv[8];
      load8(v + ((tok0 + j) * H + h) * (long long)D + col0 + 8 * cg, fv);
#pragma unroll
      for (int e = 0; e < 8; ++e) sm.v[j][8 * cg + e] = fv[e];
    }
    __syncthreads();

    // 2. A = Q K^T with the decay mask; warp w owns rows [8w, 8w+8), lane owns cols l, l+32
    {
      float acc[8][2];
#pragma unroll
      for (int r = 0; r < 8; ++r) acc[r][0] = acc[r][1] = 0.f;
      for (int kk = 0; kk < D; ++kk) {
        const float k0 = sm.kt[kk][lane], k1 = sm.kt[kk][lane + 32];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float qv = sm.qt[kk][8 * warp + r];
          acc[r][0] = fmaf(qv, k0, acc[r][0]);
          acc[r][1] = fmaf(qv, k1, acc[r][1]);
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = 8 * warp + r;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int j = lane + 32 * u;
          sm.at[j][i] = (j <= i) ? acc[r][u] * sm.pw[i - j] : 0.f;
        }
      }
    }
    __syncthreads();

    // 3. O = A V + diag(lam^(i+1)) Q S; warp w owns rows [8w, 8w+8), lane = column
    {
      float oi[8], oe[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) oi[r] = oe[r] = 0.f;
      for (int j = 0; j < C; ++j) {
        const float vv = sm.v[j][lane];
#pragma unroll
        for (int r = 0; r < 8; ++r) oi[r] = fmaf(sm.at[j][8 * warp + r], vv, oi[r]);
      }
      for (int kk = 0; kk < D; ++kk) {
        const float sv = sm.s[kk][lane];
#pragma unroll
        for (int r = 0; r < 8; ++r) oe[r] = fmaf(sm.qt[kk][8 * warp + r], sv, oe[r]);
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = 8 * warp + r;
        const long long off = ((tok0 + i) * H + h) * (long long)D + col0 + lane;
        const float o = scale * (oi[r] + sm.pw[i + 1] * oe[r]);
        out[off] = from_f32<T>(sigmoidf_(to_f32(gate[off])) * o);
      }
    }
    __syncthreads();

    // 4. S = lam^C S + (diag(lam^(C-1-j)) K)^T V; warp w owns rows [D/8 w, D/8 (w+1)), lane = column
    {
      constexpr int RW = D / 8;
      float acc[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) acc[r] = 0.f;
      for (int j = 0; j < C; ++j) {
        const float vv = sm.v[j][lane] * sm.pw[C - 1 - j];
#pragma unroll
        for (int r = 0; r < RW; ++r) acc[r] = fmaf(sm.kt[RW * warp + r][j], vv, acc[r]);
      }
#pragma unroll
      for (int r = 0; r < RW; ++r) sm.s[RW * warp + r][lane] = lamC * sm.s[RW * warp + r][lane] + acc[r];
    }
    __syncthreads();
  }

  if (state_out) {
    for (int e = tid; e < D * kSimtCols; e += kSimtThreads) {
      const int r = e / kSimtCols, c = e % kSimtCols;
      state_out[sbase + (long long)r * D + col0 + c] = sm.s[r][c];
    }
  }
}

}  // namespace sala
