// Decode step: one new token through n_linear linear layers and one sparse
// layer, in ONE cooperative launch.
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
//
// The step is bound by HBM traffic (the linear states and the block-mean
// table) and by the latency of its dependent phases, so it runs as one
// persistent grid of one CTA per SM whose phases are separated by bounded
// grid barriers (the launch is cooperative, so every CTA is resident):
//
//   P0  the scores of all candidate blocks in chunks of 256, each score
//       also counted in a 4096-bin histogram of its top 12 key bits per
//       (batch, kv head); the sparse layer's cache append and query
//       normalisation; then every linear (layer, batch, head) state update
//       and output, which need nothing from the sparse layer and run while
//       the selections do.  The CTA that scores the last chunk of a (batch,
//       kv head) selects for it while the other CTAs take the remaining
//       units: the bin T holding
//       the k-th largest score, the candidates above T (certainly selected)
//       and those in T (the boundary), the remaining ones picked exactly from
//       the boundary (score descending, ties to the lower block), and the
//       ascending index row.  A boundary of more than 1024 entries
//       (degenerate score distributions) falls back to an exact radix
//       select over all scores.
//   B1  barrier.
//   P1  one unit per (batch, kv head, selected block): partial softmax sums
//       of the group's q heads over that block's keys.
//   B2  barrier.
//   P2  one unit per (batch, q head): combine of the partials, output gate.
//
// Every wait is bounded (about a second); a barrier that runs out sets the
// timeout bit of the status word and the CTAs return.
#pragma once

#include "common.cuh"
#include "prologue.cuh"
#include "select.cuh"

namespace sala {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecChunk = 256;          // candidate blocks per scoring unit (two threads each)
constexpr int kDecBinBits = 12;
constexpr int kDecBins = 1 << kDecBinBits;
constexpr int kDecBndMax = 1024;        // boundary entries resolved by rank counting
constexpr int kDecodeMaxQHeads = 64;    // largest sparse-layer q head count the step takes
constexpr int kDecMaxLayers = 8;

// Row stride (in keys) of the per-(batch, kv head) score keys: rows start on
// 16-byte boundaries so that the selection can stage a row with 16-byte
// asynchronous copies.
__host__ __device__ constexpr long long dec_key_stride(long long capb) { return (capb + 3) / 4 * 4; }

// Control words at the start of the workspace (zeroed by the host before
// each launch), each on its own 128-byte line: the barriers' arrival counts,
// the work counters of P0 and P1, and per (batch, kv head) the number of
// scored chunks.
constexpr int kDecCtlBarriers = 2;
constexpr int kDecLine = 32;            // words per 128-byte line
__host__ __device__ constexpr int dec_ctl_words(int bg) { return kDecLine * (kDecCtlBarriers + 2 + bg); }
__device__ __forceinline__ unsigned* dec_bar_count(unsigned* ctl, int i) { return ctl + kDecLine * i; }
// work counters of P0 (phase 0) and P1 (phase 1)
__device__ __forceinline__ unsigned* dec_work(unsigned* ctl, int phase) {
  return ctl + kDecLine * (kDecCtlBarriers + phase);
}
__device__ __forceinline__ unsigned* dec_bg_done(unsigned* ctl, int bg) {
  return ctl + kDecLine * (kDecCtlBarriers + 2 + bg);
}

// Persistent loop over `n` units in order: CTA x takes unit x first, and
// later units from a work counter once it is free.  (Asking for the next
// unit while the current one runs would let one CTA hold two units of the
// first round while another has none.)  f(u) runs with the whole CTA.
template <typename F>
__device__ __forceinline__ void dec_unit_loop(unsigned* counter, int n, F f) {
  __shared__ int s_unit;
  int u = blockIdx.x;
  while (u < n) {
    f(u);
    __syncthreads();
    if (threadIdx.x == 0) s_unit = (int)gridDim.x + (int)atomicAdd(counter, 1u);
    __syncthreads();
    u = s_unit;
  }
}

struct DecodeParams {
  // linear layers
  const void* lq[kDecMaxLayers];
  const void* lk[kDecMaxLayers];
  const void* lv[kDecMaxLayers];
  const void* lgate[kDecMaxLayers];
  const float* lwq[kDecMaxLayers];
  const float* lwk[kDecMaxLayers];
  const float* llam[kDecMaxLayers];
  float* lstate[kDecMaxLayers];
  void* lout[kDecMaxLayers];
  int n_linear, B, H;
  float eps_l, scale_l;
  // sparse layer
  const void* q;
  const void* k;
  const void* v;
  const void* gate;
  void* out;
  const float* wq;
  const float* wk;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  float* kbar;
  float* ksum;
  int Hq, Hkv, BLK, topk, n_init, n_local, width;
  long long cap, capb, pos;
  long long kstride;    // row stride of `keys`: capb rounded up to 16 bytes
  float eps_s, sl2;
  // selection shape of this step (the same for every batch and kv head)
  int bcur, n_cand, kk, n_chunks;
  // workspace
  unsigned* ctl;
  unsigned* hist;       // [B * Hkv][kDecBins]
  uint32_t* keys;       // [B * Hkv][kstride]
  int* idx;             // [B * Hkv][width]
  float* qhat;          // [B][Hq][D]
  float* part;          // [B * Hkv][width][G][D + 4]
  RopeFreq rf;
};

// cos / sin of p * base^(-2i/D): the argument is formed and reduced modulo
// 2 pi in fp64 (|p| < 2^53), then evaluated in fp32 on [-pi, pi].
__device__ __forceinline__ void rope_cs(long long p, double inv_freq, float& c, float& s) {
  const double a = (double)p * inv_freq;
  const double two_pi = 6.283185307179586476925286766559;
  const double r = a - rint(a / two_pi) * two_pi;
  sincosf((float)r, &s, &c);
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Atomic add with acquire-release semantics at GPU scope; returns the old value.
__device__ __forceinline__ unsigned atom_add_acq_rel_u32(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Grid barrier of a cooperative launch, bounded like every wait here.  Each
// CTA arrives with one acquire-release add (after a CTA barrier, so it
// releases everything the CTA wrote) and polls the count with acquire loads
// until every CTA has arrived; the count is zeroed before the launch.
// Returns false (and sets the timeout bit) if the others did not arrive.
__device__ __forceinline__ bool dec_grid_sync(unsigned* count) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    s_ok = 1;
    if (atom_add_acq_rel_u32(count, 1u) + 1u < gridDim.x) {
      const long long t0 = clock64();
      while (ld_acquire_u32(count) < gridDim.x) {
        if (clock64() - t0 > (1ll << 31)) {
          set_status(kStatusTimeout);
          s_ok = 0;
          break;
        }
      }
    }
  }
  __syncthreads();
  return s_ok != 0;
}

template <typename T>
__device__ __forceinline__ float ldf(const void* p, long long i) {
  return to_f32(static_cast<const T*>(p)[i]);
}

// ------------------------------------------------------------------ P0 units

template <int D>
__device__ void dec_select_bg(const DecodeParams& p, int bg, unsigned char* smem_raw);

// Normalised query of q head h of batch b (RMSNorm over D, no rotation):
// one warp, D/32 values per lane.
template <typename T, int D>
__device__ __forceinline__ void norm_query_warp(const DecodeParams& p, int b, int h, float* x) {
  const int lane = threadIdx.x & 31;
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) {
    x[e] = ldf<T>(p.q, ((long long)b * p.Hq + h) * D + lane + 32 * e);
    ss += x[e] * x[e];
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / D + p.eps_s);
#pragma unroll
  for (int e = 0; e < D / 32; ++e) x[e] = x[e] * r * p.wq[lane + 32 * e];
}

// Scores of candidate blocks [c0, c0 + nc) of (b, g) against the group's
// summed normalised query; each score's key goes to `keys` and to the
// (b, g) histogram.
template <typename T, int D>
__device__ void dec_score_unit(const DecodeParams& p, int u, float* sm) {
  const int ck = u % p.n_chunks;
  const int bg = u / p.n_chunks;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* qh = sm;              // [kDecWarps][D] per-warp partial group sums
  float* qv = sm + kDecWarps * D;
  unsigned* hs = reinterpret_cast<unsigned*>(qv + D);   // [kDecBins] this unit's histogram
  // this thread's half row of its candidate's block mean is loaded first, so
  // that the loads are in flight while the group query is formed
  const int c0 = ck * kDecChunk;
  const int nc = min(kDecChunk, p.n_cand - c0);
  const int c = tid >> 1, half = tid & 1;
  float4 kv[D / 8];
  if (c < nc) {
    const float4* kr = reinterpret_cast<const float4*>(
        p.kbar + (((long long)b * p.capb + p.n_init + c0 + c) * p.Hkv + g) * D + half * (D / 2));
#pragma unroll
    for (int e = 0; e < D / 8; ++e) kv[e] = kr[e];
  } else {
#pragma unroll
    for (int e = 0; e < D / 8; ++e) kv[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int e = tid; e < kDecBins; e += kDecThreads) hs[e] = 0u;
  float acc[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
  for (int h = warp; h < G; h += kDecWarps) {
    float x[D / 32];
    norm_query_warp<T, D>(p, b, g * G + h, x);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) acc[e] += x[e];
  }
#pragma unroll
  for (int e = 0; e < D / 32; ++e) qh[warp * D + lane + 32 * e] = acc[e];
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
    for (int w = 0; w < kDecWarps; ++w) s += qh[w * D + tid];
    qv[tid] = s;
  }
  __syncthreads();
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  {
    const float* qq = qv + half * (D / 2);
#pragma unroll
    for (int e = 0; e < D / 8; ++e) {
      s0 = fmaf(qq[4 * e], kv[e].x, s0);
      s1 = fmaf(qq[4 * e + 1], kv[e].y, s1);
      s2 = fmaf(qq[4 * e + 2], kv[e].z, s2);
      s3 = fmaf(qq[4 * e + 3], kv[e].w, s3);
    }
  }
  float s = (s0 + s1) + (s2 + s3);
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  if (c < nc && half == 0) {
    const uint32_t key = score_key(s * rsqrtf((float)D));
    p.keys[(long long)bg * p.kstride + c0 + c] = key;
    atomicAdd(hs + (key >> (32 - kDecBinBits)), 1u);
  }
  // the unit's histogram is added to the (b, g) one bin by bin, only where it
  // is not empty: scores crowd into few bins, and a global atomic per score
  // would queue on them
  __syncthreads();
  for (int e = tid; e < kDecBins; e += kDecThreads) {
    const unsigned n = hs[e];
    if (n) atomicAdd(p.hist + (long long)bg * kDecBins + e, n);
  }
  // the CTA that finishes the last chunk of (b, g) selects for it
  __shared__ int s_last_chunk;
  __syncthreads();
  if (tid == 0)   // releases this CTA's keys and bins; the last one acquires all the others'
    s_last_chunk = atom_add_acq_rel_u32(dec_bg_done(p.ctl, bg), 1u) == (unsigned)(p.n_chunks - 1);
  __syncthreads();
  if (s_last_chunk) dec_select_bg<D>(p, bg, reinterpret_cast<unsigned char*>(sm));
}

// One linear (layer, batch, head): S <- lam S + k^T v over the whole d x d
// state, out = sigmoid(g) * scale * q^ S.  Thread (row group rg of 32 rows,
// column col).
template <typename T, int D>
__device__ void dec_linear_unit(const DecodeParams& p, int u, float* sm) {
  const int h = u % p.H;
  const int b = (u / p.H) % p.B;
  const int layer = u / (p.H * p.B);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* qh = sm;
  float* kh = sm + D;
  float* vv = sm + 2 * D;
  float* part = sm + 3 * D;          // [4][D]
  const long long voff = ((long long)b * p.H + h) * D;
  const int col = tid & (D - 1);
  const int rg = tid / D;                       // D = 128: four groups of 32 rows; D = 64: eight of 8
  constexpr int NRG = kDecThreads / D;
  constexpr int RPT = D / NRG;
  float* S = p.lstate[layer] + ((long long)b * p.H + h) * D * D;
  // the state loads are issued before the token's norm and rotation
  float sv[RPT];
#pragma unroll
  for (int u2 = 0; u2 < RPT; ++u2) sv[u2] = S[(long long)(rg * RPT + u2) * D + col];
  if (warp < 2) {
    const void* src = warp == 0 ? p.lq[layer] : p.lk[layer];
    const float* w = warp == 0 ? p.lwq[layer] : p.lwk[layer];
    float* dst = warp == 0 ? qh : kh;
    float ss = 0.f;
    for (int e = lane; e < D; e += 32) { const float x = ldf<T>(src, voff + e); ss += x * x; }
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / D + p.eps_l);
    for (int i = lane; i < D / 2; i += 32) {
      const float x1 = ldf<T>(src, voff + i) * r * w[i];
      const float x2 = ldf<T>(src, voff + i + D / 2) * r * w[i + D / 2];
      float c, s;
      rope_cs(p.pos, p.rf.inv[i], c, s);
      dst[i] = x1 * c - x2 * s;
      dst[i + D / 2] = x2 * c + x1 * s;
    }
  } else if (warp == 2) {
    for (int e = lane; e < D; e += 32) vv[e] = ldf<T>(p.lv[layer], voff + e);
  }
  __syncthreads();
  const float lam = p.llam[layer][h];
  const float vc = vv[col];
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
  for (int u2 = 0; u2 < RPT; u2 += 2) {
    const int r = rg * RPT + u2;
    const float s0 = lam * sv[u2] + kh[r] * vc;
    const float s1 = lam * sv[u2 + 1] + kh[r + 1] * vc;
    S[(long long)r * D + col] = s0;
    S[(long long)(r + 1) * D + col] = s1;
    acc0 = fmaf(qh[r], s0, acc0);
    acc1 = fmaf(qh[r + 1], s1, acc1);
  }
  part[rg * D + col] = acc0 + acc1;
  __syncthreads();
  if (tid < D) {
    float o = 0.f;
#pragma unroll
    for (int r = 0; r < NRG; ++r) o += part[r * D + tid];
    o *= p.scale_l;
    T* out = static_cast<T*>(p.lout[layer]);
    out[voff + tid] = from_f32<T>(sigmoidf_(ldf<T>(p.lgate[layer], voff + tid)) * o);
  }
}

// The sparse layer's new token of batch b: normalise its key (append key and
// value to the caches, add to the running block sum, close the block mean
// when the block completes) and its queries (kept in fp32 for P2).  One warp
// per row.
template <typename T, int D>
__device__ void dec_sparse_prep_unit(const DecodeParams& p, int b) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool closes = ((p.pos + 1) % p.BLK) == 0;
  for (int r = warp; r < p.Hkv + p.Hq; r += kDecWarps) {
    float x[D / 32];
    if (r < p.Hkv) {
      const int h = r;
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) {
        x[e] = ldf<T>(p.k, ((long long)b * p.Hkv + h) * D + lane + 32 * e);
        ss += x[e] * x[e];
      }
      ss = warp_sum(ss);
      const float rn = rsqrtf(ss / D + p.eps_s);
      const long long crow = (((long long)b * p.cap + p.pos) * p.Hkv + h) * D;
      float* ks = p.ksum + ((long long)b * p.Hkv + h) * D;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) {
        const int d = lane + 32 * e;
        const float xn = x[e] * rn * p.wk[d];
        p.k_cache[crow + d] = __float2bfloat16_rn(xn);
        p.v_cache[crow + d] = __float2bfloat16_rn(ldf<T>(p.v, ((long long)b * p.Hkv + h) * D + d));
        const float s = ks[d] + xn;
        if (closes) {
          p.kbar[(((long long)b * p.capb + p.pos / p.BLK) * p.Hkv + h) * D + d] = s / (float)p.BLK;
          ks[d] = 0.f;
        } else {
          ks[d] = s;
        }
      }
    } else {
      const int h = r - p.Hkv;
      norm_query_warp<T, D>(p, b, h, x);
#pragma unroll
      for (int e = 0; e < D / 32; ++e) p.qhat[((long long)b * p.Hq + h) * D + lane + 32 * e] = x[e];
    }
  }
}

// ------------------------------------------------------------------ selection

// Index row when no ranking is needed (no candidates, or k covers them all).
__device__ void dec_direct_row(const DecodeParams& p, int bg) {
  const int tid = threadIdx.x;
  const int b_ = p.bcur;
  const int n_first = min(p.n_init, b_ + 1);
  const int local_lo = max(p.n_init, b_ - p.n_local + 1);
  const int n_loc = max(0, b_ - local_lo + 1);
  int32_t* row = p.idx + (long long)bg * p.width;
  for (int e = tid; e < n_first; e += kDecThreads) row[e] = e;
  for (int e = tid; e < p.kk; e += kDecThreads) row[n_first + e] = p.n_init + e;
  for (int e = tid; e < n_loc; e += kDecThreads) row[n_first + p.kk + e] = local_lo + e;
  for (int e = n_first + p.kk + n_loc + tid; e < p.width; e += kDecThreads) row[e] = -1;
}

// Selection of (b, g) once all its scores and histogram counts are in, by
// one CTA:
//  1. T = the bin holding the kk-th largest key: the 4096 bins are scanned
//     from the top (thread t owns bins 4095 - 8t - u, u = 0..7);
//  2. every key above bin T is selected; the keys in bin T (the boundary)
//     are collected with their candidate numbers;
//  3. the remaining kk - n_above are the boundary entries of rank < that by
//     (key descending, candidate ascending), found by counting;
//  4. the kk candidates are ordered by counting and written, after the
//     initial blocks and before the local ones.
// If the boundary holds more than kDecBndMax entries, the kk candidates are
// taken by an exact radix select over every key instead.
template <int D>
__device__ void dec_select_bg(const DecodeParams& p, int bg, unsigned char* smem_raw) {
  const int tid = threadIdx.x;
  __shared__ int scan_s[kDecThreads / 32 + 1];
  __shared__ int hist_s[256];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need, s_T, s_n_above, s_n_bnd;
  int32_t* chosen = reinterpret_cast<int32_t*>(smem_raw);          // [topk]
  int32_t* sorted = chosen + p.topk;                               // [topk]
  uint8_t* tail = reinterpret_cast<uint8_t*>(sorted + p.topk);
  tail = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tail) + 15) & ~uintptr_t(15));
  uint2* sb = reinterpret_cast<uint2*>(tail);                     // [kDecBndMax] boundary
  uint32_t* sk = reinterpret_cast<uint32_t*>(tail + kDecBndMax * 8);  // [kstride] all keys
  // 0. every key of (b, g) is copied into shared memory while the threshold
  // is found (L2 -> shared, 16 bytes a copy, rows 16-byte aligned)
  {
    const uint32_t* src = p.keys + (long long)bg * p.kstride;
    const uint32_t dst = (uint32_t)__cvta_generic_to_shared(sk);
    for (int e = tid; e < (p.n_cand + 3) / 4; e += kDecThreads)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst + 16 * e),
                   "l"(src + 4 * e)
                   : "memory");
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  }
  // 1. threshold bin
  {
    const unsigned* h = p.hist + (long long)bg * kDecBins;
    int cnt[8], tot = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) cnt[u] = 0;
    {
      // this thread's 8 bins kDecBins-1-8 tid .. kDecBins-8-8 tid as two 16-byte loads
      const uint4* hv = reinterpret_cast<const uint4*>(h + kDecBins - 8 - 8 * tid);
      const uint4 lo = __ldcg(hv), hi = __ldcg(hv + 1);
      const unsigned w[8] = {hi.w, hi.z, hi.y, hi.x, lo.w, lo.z, lo.y, lo.x};
#pragma unroll
      for (int u = 0; u < 8; ++u) { cnt[u] = (int)w[u]; tot += cnt[u]; }
    }
    if (tid == 0) { s_n_above = 0; s_n_bnd = 0; s_T = 0; }
    int all;
    const int before = block_exclusive_scan<kDecThreads>(tot, scan_s, &all);
    if (before < p.kk && before + tot >= p.kk) {
      int cum = before, u = 0;
      for (; u < 8; ++u) {
        if (cum + cnt[u] >= p.kk) break;
        cum += cnt[u];
      }
      s_T = kDecBins - 1 - 8 * tid - u;
    }
    __syncthreads();
  }
  // 2. above / boundary lists (slot order is arbitrary; the result is not)
  const unsigned T = (unsigned)s_T;
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();
  for (int c = tid; c < p.n_cand; c += kDecThreads) {
    const uint32_t key = sk[c];
    const unsigned bin = key >> (32 - kDecBinBits);
    if (bin > T) {
      const int slot = atomicAdd(&s_n_above, 1);
      if (slot < p.topk) chosen[slot] = c;
      else set_status(kStatusBounds);
    } else if (bin == T) {
      const int slot = atomicAdd(&s_n_bnd, 1);
      if (slot < kDecBndMax) sb[slot] = make_uint2(key, (unsigned)c);
    }
  }
  __syncthreads();
  const int n_above = min(s_n_above, p.topk);
  const int n_bnd = s_n_bnd;
  const int need = p.kk - n_above;
  bool in_order = false;
  if (n_bnd <= kDecBndMax && need >= 1 && need <= n_bnd) {
    // 3. ranks inside the boundary
    for (int e = tid; e < n_bnd; e += kDecThreads) {
      const uint2 me = sb[e];
      int rank = 0;
      for (int f = 0; f < n_bnd; ++f) {
        const uint2 o = sb[f];
        rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
      }
      if (rank < need) chosen[n_above + rank] = (int)me.y;
    }
  } else {
    // degenerate boundary: exact radix select over every key of (b, g)
    topk_emit_sorted<kDecThreads>(sk, p.n_cand, p.kk, sorted, 0, hist_s, scan_s, &s_prefix,
                                  &s_need);
    in_order = true;
  }
  __syncthreads();
  if (!in_order) {
    for (int e = tid; e < p.kk; e += kDecThreads) {
      const int me = chosen[e];
      int r = 0;
      for (int f = 0; f < p.kk; ++f) r += chosen[f] < me;
      sorted[r] = me;
    }
    __syncthreads();
  }
  // 4. the row
  const int b_ = p.bcur;
  const int n_first = min(p.n_init, b_ + 1);
  const int local_lo = max(p.n_init, b_ - p.n_local + 1);
  const int n_loc = max(0, b_ - local_lo + 1);
  int32_t* row = p.idx + (long long)bg * p.width;
  for (int e = tid; e < n_first; e += kDecThreads) row[e] = e;
  for (int e = tid; e < p.kk; e += kDecThreads) row[n_first + e] = p.n_init + sorted[e];
  for (int e = tid; e < n_loc; e += kDecThreads) row[n_first + p.kk + e] = local_lo + e;
  for (int e = n_first + p.kk + n_loc + tid; e < p.width; e += kDecThreads) row[e] = -1;
}

// ------------------------------------------------------------------ P1, P2

// Partial softmax sums of the G q heads of (b, g) over selected block `slot`:
// [G][D + 4] = (m, l, -, -, o[D]) with logits in base 2.  Keys and values are
// staged as bf16 with 16-byte chunks XOR-swizzled by row.
template <int D>
__device__ void dec_attn_unit(const DecodeParams& p, int u, unsigned char* smem_raw) {
  constexpr int NC = D / 8;
  constexpr int DP = D + 4;
  const int slot = u % p.width;
  const int bg = u / p.width;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint4* ks = reinterpret_cast<uint4*>(smem_raw);                 // [64][NC]
  uint4* vs = ks + 64 * NC;                                       // [64][NC]
  float* qs = reinterpret_cast<float*>(vs + 64 * NC);             // [G][D]
  float* lg = qs + G * D;                                         // [G][64]
  float* red = lg + G * 64;                                       // [2][G][D]
  float* ml = red + 2 * G * D;                                    // [G][2]
  float* pb = p.part + ((long long)bg * p.width + slot) * G * DP;
  int j = __ldcg(p.idx + (long long)bg * p.width + slot);
  if (j >= 0 && (long long)j * p.BLK > p.pos) {
    set_status(kStatusBounds);
    j = -1;
  }
  if (j < 0) {
    for (int e = tid; e < G * DP; e += kDecThreads) pb[e] = (e % DP) == 0 ? -INFINITY : 0.f;
    return;
  }
  const long long kend = min((long long)(j + 1) * p.BLK, p.pos + 1);
  const int nk = (int)(kend - (long long)j * p.BLK);
  {
    // every load of the unit is issued before the first shared-memory store
    constexpr int PER = (64 * NC + kDecThreads - 1) / kDecThreads;
    constexpr int QPER = 1;     // one query float4 per thread in flight (G * D / 4 <= 512 at G = 16)
    uint4 kv[PER], vv[PER];
    float4 qv[QPER];
    const float4* qsrc = reinterpret_cast<const float4*>(p.qhat + ((long long)b * p.Hq + g * G) * D);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + u * kDecThreads, sr = e / NC, c = e % NC;
      kv[u] = vv[u] = make_uint4(0, 0, 0, 0);
      if (e < 64 * NC && sr < nk) {
        const long long off = (((long long)b * p.cap + (long long)j * p.BLK + sr) * p.Hkv + g) * D + 8 * c;
        kv[u] = __ldcg(reinterpret_cast<const uint4*>(p.k_cache + off));
        vv[u] = __ldcg(reinterpret_cast<const uint4*>(p.v_cache + off));
      }
    }
#pragma unroll
    for (int u = 0; u < QPER; ++u) {
      const int e = tid + u * kDecThreads;
      if (e < G * D / 4) qv[u] = __ldcg(qsrc + e);
    }
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + u * kDecThreads, sr = e / NC, c = e % NC;
      if (e < 64 * NC) {
        ks[sr * NC + (c ^ (sr & (NC - 1)))] = kv[u];
        vs[sr * NC + (c ^ (sr & (NC - 1)))] = vv[u];
      }
    }
#pragma unroll
    for (int u = 0; u < QPER; ++u) {
      const int e = tid + u * kDecThreads;
      if (e < G * D / 4) reinterpret_cast<float4*>(qs)[e] = qv[u];
    }
    for (int e = tid + QPER * kDecThreads; e < G * D / 4; e += kDecThreads)
      reinterpret_cast<float4*>(qs)[e] = __ldcg(qsrc + e);
  }
  __syncthreads();
  // logits: thread (key sr, heads hq0 + 8 m)
  {
    const int sr = tid & 63;
    for (int h = tid >> 6; h < G; h += kDecThreads / 64) {
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      const float* qr = qs + h * D;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        float kf[8];
        load8(reinterpret_cast<const __nv_bfloat16*>(&ks[sr * NC + (c ^ (sr & (NC - 1)))]), kf);
        a0 = fmaf(kf[0], qr[8 * c + 0], a0); a1 = fmaf(kf[1], qr[8 * c + 1], a1);
        a2 = fmaf(kf[2], qr[8 * c + 2], a2); a3 = fmaf(kf[3], qr[8 * c + 3], a3);
        a0 = fmaf(kf[4], qr[8 * c + 4], a0); a1 = fmaf(kf[5], qr[8 * c + 5], a1);
        a2 = fmaf(kf[6], qr[8 * c + 6], a2); a3 = fmaf(kf[7], qr[8 * c + 7], a3);
      }
      lg[h * 64 + sr] = sr < nk ? ((a0 + a1) + (a2 + a3)) * p.sl2 : -INFINITY;
    }
  }
  __syncthreads();
  // softmax of one block per head: one warp per head, two logits per lane
  for (int h = warp; h < G; h += kDecWarps) {
    const float x0 = lg[h * 64 + lane], x1 = lg[h * 64 + lane + 32];
    const float m = warp_max(fmaxf(x0, x1));
    const float p0 = exp2f(x0 - m), p1 = exp2f(x1 - m);
    const float l = warp_sum(p0 + p1);
    lg[h * 64 + lane] = p0;
    lg[h * 64 + lane + 32] = p1;
    if (lane == 0) { ml[2 * h] = m; ml[2 * h + 1] = l; }
  }
  __syncthreads();
  // P V: item (head, 8-column chunk, key half)
  for (int e = tid; e < G * NC * 2; e += kDecThreads) {
    const int half = e & 1, c = (e >> 1) % NC, h = (e >> 1) / NC;
    float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int s0 = half * 32, s1 = min(nk, s0 + 32);
    for (int sr = s0; sr < s1; ++sr) {
      float vf[8];
      load8(reinterpret_cast<const __nv_bfloat16*>(&vs[sr * NC + (c ^ (sr & (NC - 1)))]), vf);
      const float pr = lg[h * 64 + sr];
#pragma unroll
      for (int w = 0; w < 8; ++w) o[w] = fmaf(pr, vf[w], o[w]);
    }
#pragma unroll
    for (int w = 0; w < 8; ++w) red[(half * G + h) * D + 8 * c + w] = o[w];
  }
  __syncthreads();
  for (int e = tid; e < G * DP; e += kDecThreads) {
    const int h = e / DP, c = e % DP;
    pb[e] = c == 0 ? ml[2 * h]
                   : (c == 1 ? ml[2 * h + 1]
                             : (c < 4 ? 0.f : red[h * D + c - 4] + red[(G + h) * D + c - 4]));
  }
}

// The same partial sums on the tensor cores with warp-level MMAs
// (m16n8k16, bf16 operands, fp32 accumulation), for groups of at most 16 q
// heads: the group's queries (rows past G zero) against the block's 64 keys,
// logits Q K^T by warps 0..7 (8 keys each), the softmax per head, then
// P V by warps 0..D/8-1 (8 value columns each).  A 16-row tile is below the
// smallest tcgen05 tile and the step is bound by latency, not by MMA
// throughput.  Queries and P are rounded to bf16 for the products, as in the
// prefill kernel.
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__device__ void dec_attn_unit_mma(const DecodeParams& p, int u, unsigned char* smem_raw) {
  constexpr int NC = D / 8;
  constexpr int DP = D + 4;
  constexpr int QS = D + 8;            // bf16 row stride of Q (conflict-free fragment loads)
  constexpr int PS = 64 + 8;           // bf16 row stride of P
  const int slot = u % p.width;
  const int bg = u / p.width;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint4* ks = reinterpret_cast<uint4*>(smem_raw);                 // [64][NC]
  uint4* vs = ks + 64 * NC;                                       // [64][NC]
  __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(vs + 64 * NC);   // [16][QS]
  float* lg = reinterpret_cast<float*>(qb + 16 * QS);             // [16][64]
  __nv_bfloat16* pbs = reinterpret_cast<__nv_bfloat16*>(lg + 16 * 64);  // [16][PS]
  float* pb = p.part + ((long long)bg * p.width + slot) * G * DP;
  int j = __ldcg(p.idx + (long long)bg * p.width + slot);
  if (j >= 0 && (long long)j * p.BLK > p.pos) {
    set_status(kStatusBounds);
    j = -1;
  }
  if (j < 0) {
    for (int e = tid; e < G * DP; e += kDecThreads) pb[e] = (e % DP) == 0 ? -INFINITY : 0.f;
    return;
  }
  const long long kend = min((long long)(j + 1) * p.BLK, p.pos + 1);
  const int nk = (int)(kend - (long long)j * p.BLK);
  {
    // every load of the unit is issued before the first shared-memory store
    constexpr int PER = (64 * NC + kDecThreads - 1) / kDecThreads;
    uint4 kv[PER], vv[PER];
#pragma unroll
    for (int w = 0; w < PER; ++w) {
      const int e = tid + w * kDecThreads, sr = e / NC, c = e % NC;
      kv[w] = vv[w] = make_uint4(0, 0, 0, 0);
      if (e < 64 * NC && sr < nk) {
        const long long off = (((long long)b * p.cap + (long long)j * p.BLK + sr) * p.Hkv + g) * D + 8 * c;
        kv[w] = __ldcg(reinterpret_cast<const uint4*>(p.k_cache + off));
        vv[w] = __ldcg(reinterpret_cast<const uint4*>(p.v_cache + off));
      }
    }
    // one query float4 per thread (16 x D / 4 <= 512)
    const int qh = tid / (D / 4), qc = tid % (D / 4);
    float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid < 16 * D / 4 && qh < G)
      qv = __ldcg(reinterpret_cast<const float4*>(p.qhat + ((long long)b * p.Hq + g * G + qh) * D) + qc);
#pragma unroll
    for (int w = 0; w < PER; ++w) {
      const int e = tid + w * kDecThreads, sr = e / NC, c = e % NC;
      if (e < 64 * NC) {
        ks[sr * NC + (c ^ (sr & (NC - 1)))] = kv[w];
        vs[sr * NC + (c ^ (sr & (NC - 1)))] = vv[w];
      }
    }
    if (tid < 16 * D / 4) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(qv.x, qv.y), hi = __floats2bfloat162_rn(qv.z, qv.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(qb + qh * QS + 4 * qc) = pk;
    }
  }
  __syncthreads();
  const int fr = lane >> 2, fc = (lane & 3) * 2;     // fragment row / column pair
  // logits: warp w < 8 takes keys [8w, 8w + 8)
  if (warp < 8) {
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    const int sr = 8 * warp + fr;                      // this lane's key row (B operand)
    const uint8_t* krow = reinterpret_cast<const uint8_t*>(ks + sr * NC);
#pragma unroll
    for (int kq = 0; kq < D / 16; ++kq) {
      uint32_t a[4];
      a[0] = *reinterpret_cast<const uint32_t*>(qb + fr * QS + 16 * kq + fc);
      a[1] = *reinterpret_cast<const uint32_t*>(qb + (fr + 8) * QS + 16 * kq + fc);
      a[2] = *reinterpret_cast<const uint32_t*>(qb + fr * QS + 16 * kq + 8 + fc);
      a[3] = *reinterpret_cast<const uint32_t*>(qb + (fr + 8) * QS + 16 * kq + 8 + fc);
      const uint32_t b0 = *reinterpret_cast<const uint32_t*>(
          krow + (((2 * kq) ^ (sr & (NC - 1))) << 4) + 2 * fc);
      const uint32_t b1 = *reinterpret_cast<const uint32_t*>(
          krow + (((2 * kq + 1) ^ (sr & (NC - 1))) << 4) + 2 * fc);
      mma_bf16_16816(c, a, b0, b1);
    }
    const int key = 8 * warp + fc;
    lg[fr * 64 + key] = key < nk ? c[0] * p.sl2 : -INFINITY;
    lg[fr * 64 + key + 1] = key + 1 < nk ? c[1] * p.sl2 : -INFINITY;
    lg[(fr + 8) * 64 + key] = key < nk ? c[2] * p.sl2 : -INFINITY;
    lg[(fr + 8) * 64 + key + 1] = key + 1 < nk ? c[3] * p.sl2 : -INFINITY;
  }
  __syncthreads();
  // softmax of the block per head (one warp per row of the tile; rows past
  // G get P = 0)
  if (warp < 16) {
    const int h = warp;
    float p0 = 0.f, p1 = 0.f;
    if (h < G) {
      const float x0 = lg[h * 64 + lane], x1 = lg[h * 64 + lane + 32];
      const float m = warp_max(fmaxf(x0, x1));      // key 0 is always valid: m is finite
      p0 = exp2f(x0 - m);
      p1 = exp2f(x1 - m);
      const float l = warp_sum(p0 + p1);
      if (lane < 4) pb[h * DP + lane] = lane == 0 ? m : (lane == 1 ? l : 0.f);
    }
    pbs[h * PS + lane] = __float2bfloat16_rn(p0);
    pbs[h * PS + lane + 32] = __float2bfloat16_rn(p1);
  }
  __syncthreads();
  // P V: warp w < D / 8 takes value columns [8w, 8w + 8)
  if (warp < D / 8) {
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t vbase = (uint32_t)__cvta_generic_to_shared(vs);
#pragma unroll
    for (int kq = 0; kq < 4; ++kq) {
      uint32_t a[4];
      a[0] = *reinterpret_cast<const uint32_t*>(pbs + fr * PS + 16 * kq + fc);
      a[1] = *reinterpret_cast<const uint32_t*>(pbs + (fr + 8) * PS + 16 * kq + fc);
      a[2] = *reinterpret_cast<const uint32_t*>(pbs + fr * PS + 16 * kq + 8 + fc);
      a[3] = *reinterpret_cast<const uint32_t*>(pbs + (fr + 8) * PS + 16 * kq + 8 + fc);
      // rows (keys) 16 kq + 0..15 of value chunk `warp`, transposed into the
      // B fragment: lanes 0-7 address keys 16kq+0..7, lanes 8-15 keys 16kq+8..15
      const int key = 16 * kq + (lane & 15);
      const uint32_t addr = vbase + (uint32_t)((key * NC + (warp ^ (key & (NC - 1)))) * 16);
      uint32_t b0, b1;
      asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
                   : "=r"(b0), "=r"(b1)
                   : "r"(addr));
      mma_bf16_16816(c, a, b0, b1);
    }
    const int col = 8 * warp + fc;
    if (fr < G) {
      pb[fr * DP + 4 + col] = c[0];
      pb[fr * DP + 4 + col + 1] = c[1];
    }
    if (fr + 8 < G) {
      pb[(fr + 8) * DP + 4 + col] = c[2];
      pb[(fr + 8) * DP + 4 + col + 1] = c[3];
    }
  }
}

// Combine of the `width` partials of q head hq of batch b and the output
// gate, for value columns [32 cu, 32 cu + 32) (a head is split over D / 32
// units so that more CTAs share the reads).  Warp w takes partials w, w + 16,
// ...; lane l column 32 cu + l.
constexpr int kDecCombCols = 32;
template <typename T, int D>
__device__ void dec_combine_unit(const DecodeParams& p, int u, float* sm) {
  constexpr int DP = D + 4;
  constexpr int NCU = D / kDecCombCols;          // units per head
  constexpr int NG = kDecThreads / kDecCombCols; // partial groups (one per warp)
  constexpr int kBatch = 8;                      // partials in flight per thread
  const int cu = u % NCU, hq = (u / NCU) % p.Hq, b = u / (NCU * p.Hq);
  const int G = p.Hq / p.Hkv, g = hq / G, h = hq % G;
  const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
  float* wts = sm;                       // [width] weights, then [width] sums
  float* lsum = sm + p.width;
  float* red = sm + 2 * p.width;         // [NG][32]
  __shared__ float s_l;
  const float* pb = p.part + (((long long)b * p.Hkv + g) * p.width * G + h) * DP;
  const long long pstride = (long long)G * DP;
  const int col = cu * kDecCombCols + lane;
  // this thread's first batch of partial columns and the gate are loaded
  // before the weights are formed (every thread runs this block: it holds
  // the CTA barriers)
  float pv[kBatch];
#pragma unroll
  for (int v = 0; v < kBatch; ++v) {
    const int e = grp + v * NG;
    pv[v] = e < p.width ? __ldcg(pb + e * pstride + 4 + col) : 0.f;
  }
  const long long off = ((long long)b * p.Hq + hq) * D + col;
  const float gt = tid < kDecCombCols ? ldf<T>(p.gate, off) : 0.f;
  for (int e = tid; e < p.width; e += kDecThreads) {
    wts[e] = __ldcg(pb + e * pstride);
    lsum[e] = __ldcg(pb + e * pstride + 1);
  }
  __syncthreads();
  if (tid < 32) {
    float M = -INFINITY;
    for (int e = tid; e < p.width; e += 32) M = fmaxf(M, wts[e]);
    M = warp_max(M);
    float L = 0.f;
    for (int e = tid; e < p.width; e += 32) {
      const float m = wts[e];
      const float f = m == -INFINITY ? 0.f : exp2f(m - M);
      L = fmaf(f, lsum[e], L);
      wts[e] = f;
    }
    L = warp_sum(L);
    if (tid == 0) s_l = L;
  }
  __syncthreads();
  float o = 0.f;
  for (int e0 = grp;; e0 += kBatch * NG) {
#pragma unroll
    for (int v = 0; v < kBatch; ++v) {
      const int e = e0 + v * NG;
      if (e < p.width) o = fmaf(wts[e], pv[v], o);
    }
    if (e0 + kBatch * NG >= p.width) break;
#pragma unroll
    for (int v = 0; v < kBatch; ++v) {
      const int e = e0 + kBatch * NG + v * NG;
      pv[v] = e < p.width ? __ldcg(pb + e * pstride + 4 + col) : 0.f;
    }
  }
  red[grp * kDecCombCols + lane] = o;
  __syncthreads();
  if (tid < kDecCombCols) {
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < NG; ++r) acc += red[r * kDecCombCols + tid];
    const float inv = s_l > 0.f ? 1.f / s_l : 0.f;
    static_cast<T*>(p.out)[off] = from_f32<T>(sigmoidf_(gt) * acc * inv);
  }
}

// ------------------------------------------------------------------ kernel

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_step_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(16) unsigned char dec_smem[];
  float* sm = reinterpret_cast<float*>(dec_smem);
  const bool ranked = p.kk > 0 && p.kk < p.n_cand;
  const int BG = p.B * p.Hkv;
  const int n_score = ranked ? BG * p.n_chunks : 0;
  const int n_lin = p.n_linear * p.B * p.H;

  // P0, units in order (scores first, so that the selections start early):
  // scores + histograms (+ selection by the CTA that scores the last chunk
  // of each (b, g)), the sparse layer's cache append and queries, direct
  // index rows when nothing ranks, the linear layers.
  const int n_direct = ranked ? 0 : BG;
  dec_unit_loop(dec_work(p.ctl, 0), n_score + p.B + n_direct + n_lin, [&](int u) {
    if (u < n_score) dec_score_unit<T, D>(p, u, sm);
    else if (u < n_score + p.B) dec_sparse_prep_unit<T, D>(p, u - n_score);
    else if (u < n_score + p.B + n_direct) dec_direct_row(p, u - n_score - p.B);
    else dec_linear_unit<T, D>(p, u - n_score - p.B - n_direct, sm);
  });
  if (!dec_grid_sync(dec_bar_count(p.ctl, 0))) return;
  // P1: attention partials
  const int n_att = BG * p.width;
  if (p.Hq / p.Hkv <= 16)
    dec_unit_loop(dec_work(p.ctl, 1), n_att, [&](int u) { dec_attn_unit_mma<D>(p, u, dec_smem); });
  else
    dec_unit_loop(dec_work(p.ctl, 1), n_att, [&](int u) { dec_attn_unit<D>(p, u, dec_smem); });
  if (!dec_grid_sync(dec_bar_count(p.ctl, 1))) return;
  // P2: combine and gate
  for (int u = blockIdx.x; u < p.B * p.Hq * (D / kDecCombCols); u += gridDim.x) {
    dec_combine_unit<T, D>(p, u, sm);
    __syncthreads();
  }
}

// Dynamic shared memory of the step: the largest phase's need.
inline size_t decode_smem_bytes(int D, int G, int topk, long long kstride, int width) {
  const size_t score = (size_t)(kDecWarps + 1) * D * 4 + (size_t)kDecBins * 4;
  const size_t lin = (size_t)(3 * D + kDecThreads) * 4;
  const size_t attn = G <= 16
      ? (size_t)2 * 64 * D * 2 + (size_t)16 * (D + 8) * 2 + (size_t)16 * 64 * 4 +
            (size_t)16 * (64 + 8) * 2                                     // dec_attn_unit_mma
      : (size_t)2 * 64 * D * 2 + (size_t)G * D * 4 + (size_t)G * 64 * 4 +
            (size_t)2 * G * D * 4 + (size_t)G * 8;                        // dec_attn_unit
  const size_t resolve = (size_t)2 * topk * 4 + 16 +
                         (size_t)kDecBndMax * 8 + (size_t)kstride * 4;   // dec_select_bg
  const size_t comb = (size_t)2 * width * 4 + (size_t)kDecThreads * 4;
  return std::max(std::max(std::max(score, lin), std::max(attn, resolve)), comb);
}

}  // namespace sala
