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
// Scores are compared through the order-preserving uint32 image of their
// fp32 value.  The k-th largest of a key set is found exactly by a 4-pass
// radix select (8 bits a pass); the selection is therefore deterministic
// and follows the tie rule exactly.
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

// The k-th largest of n keys (1 <= k <= n) by a 4-pass radix select over
// their bytes, high byte first: returns T, and in *need_out how many keys
// equal to T belong to the top k (the number greater than T is k - need).
// Whole CTA of NT threads; keys(c) gives key c.  hist [256], s_prefix and
// s_need in shared memory.
template <int NT, typename KeyAt>
__device__ __forceinline__ uint32_t radix_kth(KeyAt keys, int n, int k, int* hist,
                                              uint32_t* s_prefix, int* s_need, int* need_out) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, mask = 0;
  int need = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int e = tid; e < 256; e += NT) hist[e] = 0;
    __syncthreads();
    for (int c = tid; c < n; c += NT) {
      const uint32_t key = keys(c);
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
  *need_out = need;
  return prefix;
}

// Top-k of n_cand keys held in shared memory in candidate order (k < n_cand):
// writes the chosen candidate numbers c (ascending) to out[0..k) as base + c.
// Whole CTA of NT threads; hist [256] / scan_scratch / s_prefix / s_need in smem.
template <int NT = kSelectThreads>
__device__ __forceinline__ void topk_emit_sorted(const uint32_t* keys, int n_cand, int k,
                                                 int32_t* out, int base, int* hist,
                                                 int* scan_scratch, uint32_t* s_prefix,
                                                 int* s_need) {
  const int tid = threadIdx.x;
  int need;
  const uint32_t T = radix_kth<NT>([&](int c) { return keys[c]; }, n_cand, k, hist, s_prefix,
                                   s_need, &need);
  // ordered compaction: each thread owns a contiguous range of candidates;
  // `need` ties at T are taken, the lowest candidates first
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

// ---------------------------------------------------------------- prefill

constexpr int kSelTQMax = 8;                       // query blocks per CTA at most
constexpr int kSelBatch = kSelectThreads / 4;      // candidates scored per pass, 4 threads each

// Running top-k of one query block: a buffer of (key, candidate) pairs that
// holds every candidate seen so far that can still be among the top k.
struct SelRowState {
  int cnt;          // entries in the buffer
  uint32_t thr;     // admission threshold on the key
  int strict;       // 0: admit key >= thr; 1: admit key > thr
  int n_cand;       // candidates of the row
  int k;            // slots of the row
};

// Cuts the buffer of row state `rs` (n > k entries) down to its exact top k
// by (key descending, candidate ascending), in place.  Afterwards only keys
// above the k-th are admitted: candidates arrive in increasing order, so a
// later candidate equal to the k-th key loses the tie.  Whole CTA.
template <int PER>
__device__ void sel_compact(uint32_t* key, int32_t* cid, SelRowState* rs, int* hist,
                            int* scan_scratch, uint32_t* s_prefix, int* s_need) {
  const int tid = threadIdx.x;
  const int n = rs->cnt, k = rs->k;
  int need;
  const uint32_t T = radix_kth<kSelectThreads>([&](int c) { return key[c]; }, n, k, hist,
                                               s_prefix, s_need, &need);
  uint32_t kv[PER];
  int32_t cv[PER];
  int n_eq = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = tid + j * kSelectThreads;
    kv[j] = e < n ? key[e] : 0u;
    cv[j] = e < n ? cid[e] : -1;
    n_eq += e < n && kv[j] == T;
  }
  int n_eq_all;
  block_exclusive_scan<kSelectThreads>(n_eq, scan_scratch, &n_eq_all);
  int keep = 0;
  bool take[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = tid + j * kSelectThreads;
    take[j] = e < n && kv[j] > T;
    if (e < n && kv[j] == T) {
      if (n_eq_all <= need) {
        take[j] = true;
      } else {
        // rank among the ties by candidate number (candidates are distinct)
        int r = 0;
        for (int f = 0; f < n; ++f) r += key[f] == T && cid[f] < cv[j];
        take[j] = r < need;
      }
    }
    keep += take[j];
  }
  int total;
  int pos = block_exclusive_scan<kSelectThreads>(keep, scan_scratch, &total);   // all reads done
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (take[j]) {
      key[pos] = kv[j];
      cid[pos] = cv[j];
      ++pos;
    }
  }
  if (tid == 0) {
    if (total != k) set_status(kStatusBounds);
    rs->cnt = min(total, k);
    rs->thr = T;
    rs->strict = 1;
  }
  __syncthreads();
}

// One CTA per (batch, kv head g, tile of tq consecutive query blocks).  The
// candidates stream through in increasing order, kSelBatch at a time: four
// threads share a candidate (each a quarter of its block mean, read as
// contiguous 64-byte pieces) and score it against every query of the tile,
// so each block mean is read once per tile.  Each score is the same fmaf
// chain over the thread's quarter plus a two-step butterfly, whatever tq is.
// A candidate enters a row's buffer when its key passes the row's
// threshold; a buffer that could overflow on the next batch is cut to its
// exact top k (sel_compact), which raises the threshold.  At the end the
// row's top k are written in ascending order.  Tiles are taken from the last
// (largest candidate count) down.  Dynamic smem: tq * cap keys + tq * cap
// candidate numbers, cap = PER * kSelectThreads.
template <int D, int PER>
__global__ void __launch_bounds__(kSelectThreads)
select_topk_kernel(const float* __restrict__ qsum, const float* __restrict__ kbar,
                   int32_t* __restrict__ idx, int nb, int Hkv, int topk, int n_init,
                   int n_local, int width, int tq) {
  constexpr int cap = PER * kSelectThreads;
  extern __shared__ __align__(16) uint32_t sel_dyn[];
  __shared__ __align__(16) float qv[kSelTQMax][D];
  __shared__ SelRowState rows[kSelTQMax];
  __shared__ int hist[256];
  __shared__ int scan_scratch[kSelectThreads / 32 + 1];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;

  const int n_tiles = (nb + tq - 1) / tq;
  const int i0 = (n_tiles - 1 - (int)(blockIdx.x % n_tiles)) * tq;
  const int g = (blockIdx.x / n_tiles) % Hkv;
  const int b = blockIdx.x / (n_tiles * Hkv);
  const int tid = threadIdx.x;
  const int nq = min(tq, nb - i0);
  uint32_t* keyb = sel_dyn;                                         // [tq][cap]
  int32_t* cidb = reinterpret_cast<int32_t*>(sel_dyn + tq * cap);   // [tq][cap]

  // fixed parts of every row; rows that rank (fewer slots than candidates)
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
    const bool ranks = k > 0 && k < n_cand;
    if (ranks) n_cand_max = n_cand;
    if (tid == 0) rows[t] = SelRowState{0, 0u, 0, ranks ? n_cand : 0, k};
  }
  if (n_cand_max == 0) return;
  for (int e = tid; e < nq * D; e += kSelectThreads) {
    const int t = e / D, d = e % D;
    qv[t][d] = qsum[(((long long)b * nb + i0 + t) * Hkv + g) * D + d];
  }
  __syncthreads();

  const float inv_sqrt_d = rsqrtf((float)D);
  const int slot = tid >> 2, q4 = tid & 3;
  constexpr int NE = D / 16;                     // float4 pieces of a thread's quarter
  for (int c0 = 0; c0 < n_cand_max; c0 += kSelBatch) {
    const int c = c0 + slot;
    float4 kk[NE];
    if (c < n_cand_max) {
      const float4* kr = reinterpret_cast<const float4*>(
          kbar + (((long long)b * nb + n_init + c) * Hkv + g) * D);
#pragma unroll
      for (int e = 0; e < NE; ++e) kk[e] = __ldg(kr + 4 * e + q4);
    } else {
#pragma unroll
      for (int e = 0; e < NE; ++e) kk[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int t = 0; t < kSelTQMax; ++t) {
      if (t >= nq) break;                        // uniform across the CTA
      const float4* qq = reinterpret_cast<const float4*>(qv[t]);
      float p = 0.f;
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        const float4 a = qq[4 * e + q4];
        p = fmaf(a.x, kk[e].x, p);
        p = fmaf(a.y, kk[e].y, p);
        p = fmaf(a.z, kk[e].z, p);
        p = fmaf(a.w, kk[e].w, p);
      }
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      if (q4 == (t & 3) && c < rows[t].n_cand) {
        const uint32_t key = score_key(p * inv_sqrt_d);
        const uint32_t thr = rows[t].thr;
        if (rows[t].strict ? key > thr : key >= thr) {
          const int at = atomicAdd(&rows[t].cnt, 1);
          if (at < cap) {
            keyb[t * cap + at] = key;
            cidb[t * cap + at] = c;
          } else {
            set_status(kStatusBounds);
          }
        }
      }
    }
    __syncthreads();
    // cut the buffers that the next batch could overflow (the row states are
    // not written between the barrier above and the cut, so every thread
    // takes the same decision)
    if (c0 + kSelBatch < n_cand_max) {
      for (int t = 0; t < nq; ++t)
        if (rows[t].n_cand > 0 && rows[t].cnt > cap - kSelBatch)
          sel_compact<PER>(keyb + t * cap, cidb + t * cap, rows + t, hist, scan_scratch,
                           &s_prefix, &s_need);
    }
  }

  // final top k of every ranking row, written in ascending block order
  for (int t = 0; t < nq; ++t) {
    if (rows[t].n_cand == 0) continue;            // uniform
    if (rows[t].cnt > rows[t].k)
      sel_compact<PER>(keyb + t * cap, cidb + t * cap, rows + t, hist, scan_scratch, &s_prefix,
                       &s_need);
    const int i = i0 + t;
    const int k = rows[t].k, n = min(rows[t].cnt, k);
    const int n_first = min(n_init, i + 1);
    int32_t* out = idx + (((long long)b * Hkv + g) * nb + i) * width + n_first;
    const int32_t* cb = cidb + t * cap;
    for (int e = tid; e < n; e += kSelectThreads) {
      const int32_t me = cb[e];
      int r = 0;
      for (int f = 0; f < n; ++f) r += cb[f] < me;
      out[r] = n_init + me;
    }
    if (tid == 0 && n != k) set_status(kStatusBounds);
    __syncthreads();
  }
}

// Buffer size (entries per row = PER * kSelectThreads) for `topk` slots: room
// for the top k plus at least one batch, and twice the top k when that fits,
// so that a cut happens at most every k admissions.
inline int select_buffer_per(int topk) {
  for (int per = 2; per <= 8; per *= 2)
    if (per * kSelectThreads >= 2 * topk + kSelBatch) return per;
  return 8;
}

// Query blocks per selection CTA: enough CTAs for about four per SM, at most
// kSelTQMax, and the buffers within 64 KB.
inline int select_rows_per_cta(long long tiles_total, int per, int sms) {
  long long tq = tiles_total / (4LL * sms);
  const long long fit = 65536 / ((long long)per * kSelectThreads * 8);
  tq = std::min<long long>(tq, fit);
  tq = std::min<long long>(tq, kSelTQMax);
  return (int)std::max<long long>(tq, 1);
}

}  // namespace sala
