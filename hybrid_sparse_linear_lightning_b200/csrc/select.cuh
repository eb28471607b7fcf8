// Block scoring and top-k selection of the sparse layer.
//
// InfLLM-V2-style selection (acgfav.com "SALA 混合架构": a fine-grained block
// selection lets each query attend to only a small set of key blocks).
// Query block i of kv head g scores each causal candidate block
// j in [n_init, i - n_local] by <qsum_i^g, kbar_j^g> / sqrt(d), where qsum is
// the sum over the group's q heads of the block-mean normalised query and
// kbar the block-mean normalised key.  It keeps the initial blocks
// [0, n_init), the local blocks [i-n_local+1, i] and the top-k candidates
// (ties to the lower block index), written in ascending order, -1 padded.
//
// The k-th largest score is found exactly by a 4-pass radix select over the
// order-preserving uint32 image of the fp32 scores; the selected set is then
// emitted in index order by a block-wide ordered compaction, so the output is
// deterministic and matches the tie rule exactly.
#pragma once

#include "common.cuh"

namespace sala {

constexpr int kSelectThreads = 256;

// Exclusive prefix sum of one int per thread over a CTA of NT threads
// (NT / 32 <= 32); *total gets the sum.  scratch: >= NT/32 + 1 ints.
template <int NT = kSelectThreads>
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  static_assert(NT % 32 == 0 && NT / 32 <= 32, "one warp scans the warp totals");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / 32) scratch[lane] = w;   // inclusive per warp
  }
  __syncthreads();
  const int before = (warp ? scratch[warp - 1] : 0) + x - v;
  *total = scratch[NT / 32 - 1];
  __syncthreads();
  return before;
}

// Top-k of n_cand keys held in shared memory (k < n_cand): writes the chosen
// candidate numbers c (ascending) to out[0..k) as base + c.  Whole CTA of
// NT threads; hist [256] / scan_scratch / s_prefix / s_need in smem.
template <int NT = kSelectThreads>
__device__ __forceinline__ void topk_emit_sorted(const uint32_t* keys, int n_cand, int k,
                                                 int32_t* out, int base, int* hist,
                                                 int* scan_scratch, uint32_t* s_prefix,
                                                 int* s_need) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, mask = 0;
  int need = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int e = tid; e < 256; e += NT) hist[e] = 0;
    __syncthreads();
    for (int c = tid; c < n_cand; c += NT) {
      const uint32_t key = keys[c];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // bins from the top: lane l owns bins 255 - 8l .. 248 - 8l; find the bin
      // where the count of larger-or-equal keys first reaches `need`
      const int lane = tid;
      int cnt[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) { cnt[u] = hist[255 - 8 * lane - u]; tot += cnt[u]; }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int before = incl - tot;
      const unsigned hit = __ballot_sync(0xffffffffu, before < need && incl >= need);
      if (lane == __ffs(hit) - 1) {
        int cum = before, u = 0;
        for (; u < 8; ++u) {
          if (cum + cnt[u] >= need) break;
          cum += cnt[u];
        }
        *s_prefix = prefix | ((uint32_t)(255 - 8 * lane - u) << shift);
        *s_need = need - cum;
      }
    }
    __syncthreads();
    prefix = *s_prefix;
    need = *s_need;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;   // key of the k-th largest score; `need` ties at T are taken

  // ordered compaction: each thread owns a contiguous range of candidates
  const int per = (n_cand + NT - 1) / NT;
  const int lo = min(n_cand, tid * per), hi = min(n_cand, lo + per);
  int n_gt = 0, n_eq = 0;
  for (int c = lo; c < hi; ++c) {
    const uint32_t key = keys[c];
    n_gt += key > T;
    n_eq += key == T;
  }
  int tot;
  const int eq_before = block_exclusive_scan<NT>(n_eq, scan_scratch, &tot);
  const int take_eq = max(0, min(n_eq, need - eq_before));
  const int out_before = block_exclusive_scan<NT>(n_gt + take_eq, scan_scratch, &tot);
  int pos = out_before, eq_seen = 0;
  for (int c = lo; c < hi; ++c) {
    const uint32_t key = keys[c];
    bool sel = key > T;
    if (key == T) { sel = eq_seen < take_eq; ++eq_seen; }
    if (sel) {
      if (pos < k) out[pos++] = base + c;
      else set_status(kStatusBounds);
    }
  }
}

// One CTA per (batch, kv head g, TQ consecutive query blocks i0..i0+TQ-1).
// Each candidate block mean is read once per CTA and scored against the TQ
// group queries (one warp per candidate; every score is the same lane-strided
// fmaf chain and butterfly sum whatever TQ is, so the keys do not depend on
// the tiling).  Then the rows' top-k are taken one after the other.
// Dynamic smem: TQ * nb uint32 keys.
template <int D>
__global__ void __launch_bounds__(kSelectThreads)
select_topk_kernel(const float* __restrict__ qsum, const float* __restrict__ kbar,
                   int32_t* __restrict__ idx, int nb, int Hkv, int topk, int n_init,
                   int n_local, int width, int TQ) {
  extern __shared__ uint32_t keys[];
  __shared__ float qv[8][D];
  __shared__ int hist[256];
  __shared__ int scan_scratch[kSelectThreads / 32 + 1];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;

  const int n_tiles = (nb + TQ - 1) / TQ;
  const int i0 = (blockIdx.x % n_tiles) * TQ;
  const int g = (blockIdx.x / n_tiles) % Hkv;
  const int b = blockIdx.x / (n_tiles * Hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nq = min(TQ, nb - i0);

  // rows that rank (fewer slots than candidates) and the largest candidate count
  int n_cand_max = 0;
  for (int t = 0; t < nq; ++t) {
    const int i = i0 + t;
    int32_t* row = idx + (((long long)b * Hkv + g) * nb + i) * width;
    const int n_cand = max(0, i - n_local + 1 - n_init);
    const int k = min(topk, n_cand);
    const int n_first = min(n_init, i + 1);
    const int local_lo = max(n_init, i - n_local + 1);
    const int n_loc = max(0, i - local_lo + 1);
    for (int e = tid; e < n_first; e += kSelectThreads) row[e] = e;
    for (int e = tid; e < n_loc; e += kSelectThreads) row[n_first + k + e] = local_lo + e;
    for (int e = n_first + k + n_loc + tid; e < width; e += kSelectThreads) row[e] = -1;
    if (k == n_cand)
      for (int e = tid; e < n_cand; e += kSelectThreads) row[n_first + e] = n_init + e;
    if (k > 0 && k < n_cand) n_cand_max = n_cand;
  }
  if (n_cand_max == 0) return;

  // scores: one warp per candidate, TQ queries (coalesced over d)
  for (int e = tid; e < nq * D; e += kSelectThreads) {
    const int t = e / D, d = e % D;
    qv[t][d] = qsum[(((long long)b * nb + i0 + t) * Hkv + g) * D + d];
  }
  __syncthreads();
  const float inv_sqrt_d = rsqrtf((float)D);
  for (int c = warp; c < n_cand_max; c += kSelectThreads / 32) {
    const float* kr = kbar + (((long long)b * nb + n_init + c) * Hkv + g) * D;
    float kk[D / 32];
#pragma unroll
    for (int u = 0; u < D / 32; ++u) kk[u] = kr[lane + 32 * u];
    for (int t = 0; t < nq; ++t) {
      float p = 0.f;
#pragma unroll
      for (int u = 0; u < D / 32; ++u) p = fmaf(qv[t][lane + 32 * u], kk[u], p);
      p = warp_sum(p);
      if (lane == 0) keys[t * nb + c] = score_key(p * inv_sqrt_d);
    }
  }
  __syncthreads();

  for (int t = 0; t < nq; ++t) {
    const int i = i0 + t;
    const int n_cand = max(0, i - n_local + 1 - n_init);
    const int k = min(topk, n_cand);
    if (k == 0 || k == n_cand) continue;           // uniform across the CTA
    int32_t* row = idx + (((long long)b * Hkv + g) * nb + i) * width;
    const int n_first = min(n_init, i + 1);
    topk_emit_sorted(keys + t * nb, n_cand, k, row + n_first, n_init, hist, scan_scratch,
                     &s_prefix, &s_need);
    __syncthreads();
  }
}

// Query blocks per selection CTA: as many as fit 200 KB of keys, at most 8.
inline int select_rows_per_cta(int nb) {
  const int fit = (int)((200u << 10) / ((unsigned)nb * 4u));
  return fit < 1 ? 1 : (fit > 8 ? 8 : fit);
}

}  // namespace sala
