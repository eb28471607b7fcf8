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
//
// Three launches per token: (1) linear-layer state updates and the sparse
// layer's normalisation / cache append in one grid; (2) block scores with a
// per-chunk top-k, merged exactly by the last CTA of each kv head; (3) one
// CTA per selected block computing partial softmax sums, combined and gated
// by the last CTA of each kv head.
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

struct DecodeSparseArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* wq;
  const float* wk;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  float* kbar;
  float* ksum;
  float* qhat;          // [B, Hq, D] normalised queries
  float* qgrp;          // [B, Hkv, D] group sums
  unsigned* counters;   // [B, Hkv, 2]: select / attention completion counts
};

// cos / sin of p * base^(-2i/D): the argument is formed and reduced modulo
// 2 pi in fp64 (|p| < 2^53), then evaluated in fp32 on [-pi, pi].
__device__ __forceinline__ void rope_cs(long long p, int i, int D, double log2_base, float& c,
                                        float& s) {
  const double a = (double)p * exp2(-2.0 * i / D * log2_base);
  const double two_pi = 6.283185307179586476925286766559;
  const double r = a - rint(a / two_pi) * two_pi;
  sincosf((float)r, &s, &c);
}

// Stage 1.  CTAs [0, n_lin): one per (linear layer, batch, head, 64-column
// slice) updating S <- lam S + k^T v and writing out = sigmoid(g) q^ S.
// CTAs [n_lin, n_lin + B): the sparse layer of batch b (normalise k and
// append it and v to the caches, update the running block sum / mean,
// normalise q, form the group sums, reset the completion counters).
constexpr int kDecodeMaxQHeads = 64;   // q heads of the sparse layer handled by stage 1

template <typename T, int D>
__global__ void __launch_bounds__(256)
decode_stage1_kernel(DecodeLinearArgs a, DecodeSparseArgs sp, int n_lin, int B, int H, int Hq,
                     int Hkv, long long cap, long long pos, int BLK, double log2_base, float eps_l,
                     float eps_s, float scale) {
  __shared__ float sh[D * 3 + 256];
  __shared__ float qsm[kDecodeMaxQHeads * D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if ((int)blockIdx.x < n_lin) {
    constexpr int NSL = D / 64;
    float* qh = sh;
    float* kh = sh + D;
    float* vv = sh + 2 * D;
    float* part = sh + 3 * D;          // [4][64]
    const int slice = blockIdx.x % NSL;
    const int h = (blockIdx.x / NSL) % H;
    const int b = (blockIdx.x / (NSL * H)) % B;
    const int layer = blockIdx.x / (NSL * H * B);
    const long long voff = ((long long)b * H + h) * D;
    if (warp < 2) {
      const T* src = static_cast<const T*>(warp == 0 ? a.q[layer] : a.k[layer]);
      const float* w = warp == 0 ? a.wq[layer] : a.wk[layer];
      float* dst = warp == 0 ? qh : kh;
      float ss = 0.f;
      for (int e = lane; e < D; e += 32) { const float x = to_f32(src[voff + e]); ss += x * x; }
      ss = warp_sum(ss);
      const float r = rsqrtf(ss / D + eps_l);
      for (int i = lane; i < D / 2; i += 32) {
        const float x1 = to_f32(src[voff + i]) * r * w[i];
        const float x2 = to_f32(src[voff + i + D / 2]) * r * w[i + D / 2];
        float c, s;
        rope_cs(pos, i, D, log2_base, c, s);
        dst[i] = x1 * c - x2 * s;
        dst[i + D / 2] = x2 * c + x1 * s;
      }
    } else if (warp == 2) {
      const T* v = static_cast<const T*>(a.v[layer]);
      for (int e = lane; e < D; e += 32) vv[e] = to_f32(v[voff + e]);
    }
    __syncthreads();
    const int col = slice * 64 + (tid & 63);
    const int rg = tid >> 6;
    const float lam = a.lambda[layer][h];
    float* S = a.state[layer] + ((long long)b * H + h) * D * D;
    const float vc = vv[col];
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
    for (int r = rg * (D / 4); r < (rg + 1) * (D / 4); r += 2) {
      const float s0 = lam * S[(long long)r * D + col] + kh[r] * vc;
      const float s1 = lam * S[(long long)(r + 1) * D + col] + kh[r + 1] * vc;
      S[(long long)r * D + col] = s0;
      S[(long long)(r + 1) * D + col] = s1;
      acc0 = fmaf(qh[r], s0, acc0);
      acc1 = fmaf(qh[r + 1], s1, acc1);
    }
    part[rg * 64 + (tid & 63)] = acc0 + acc1;
    __syncthreads();
    if (tid < 64) {
      const float o = scale * (part[tid] + part[64 + tid] + part[128 + tid] + part[192 + tid]);
      const T* g = static_cast<const T*>(a.gate[layer]);
      T* out = static_cast<T*>(a.out[layer]);
      out[voff + col] = from_f32<T>(sigmoidf_(to_f32(g[voff + col])) * o);
    }
    return;
  }
  // ---- sparse layer of batch b
  const int b = blockIdx.x - n_lin;
  const int G = Hq / Hkv;
  const bool closes = ((pos + 1) % BLK) == 0;
  float* qs = sh;                         // this CTA's q^ rows, reused per group
  const T* q = static_cast<const T*>(sp.q);
  const T* k = static_cast<const T*>(sp.k);
  const T* v = static_cast<const T*>(sp.v);
  if (tid < 2 * Hkv) sp.counters[(long long)b * Hkv * 2 + tid] = 0u;
  for (int r = warp; r < Hkv + Hq; r += 8) {
    const bool isk = r < Hkv;
    const int h = isk ? r : r - Hkv;
    const T* src = isk ? k + ((long long)b * Hkv + h) * D : q + ((long long)b * Hq + h) * D;
    const float* w = isk ? sp.wk : sp.wq;
    float x[D / 32];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) { x[e] = to_f32(src[lane + 32 * e]); ss += x[e] * x[e]; }
    ss = warp_sum(ss);
    const float rn = rsqrtf(ss / D + eps_s);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) x[e] = x[e] * rn * w[lane + 32 * e];
    if (isk) {
      const long long crow = (((long long)b * cap + pos) * Hkv + h) * D;
      float* ks = sp.ksum + ((long long)b * Hkv + h) * D;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) {
        const int d = lane + 32 * e;
        sp.k_cache[crow + d] = __float2bfloat16_rn(x[e]);
        sp.v_cache[crow + d] = __float2bfloat16_rn(to_f32(v[((long long)b * Hkv + h) * D + d]));
        const float s = ks[d] + x[e];
        if (closes) {
          sp.kbar[(((long long)b * (cap / BLK) + pos / BLK) * Hkv + h) * D + d] = s / (float)BLK;
          ks[d] = 0.f;
        } else {
          ks[d] = s;
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < D / 32; ++e) {
        sp.qhat[((long long)b * Hq + h) * D + lane + 32 * e] = x[e];
        qsm[h * D + lane + 32 * e] = x[e];
      }
    }
  }
  __syncthreads();
  // group sums (fixed order) from shared memory
  for (int e = tid; e < Hkv * D; e += 256) {
    const int g = e / D, d = e % D;
    float s = 0.f;
    for (int hh = 0; hh < G; ++hh) s += qsm[(g * G + hh) * D + d];
    sp.qgrp[((long long)b * Hkv + g) * D + d] = s;
  }
  (void)qs;
}

// Top-k of the scored candidates: rows of the candidate chunks and, in the
// last CTA of each (batch, kv head), the exact merge.  Chunk `ck` scores
// candidates [ck * chunk, ck * chunk + chunk) of [n_init, n_init + n_cand)
// and keeps its local top-k (ascending block order); the union of the local
// lists contains the global top-k, so the last CTA selects it exactly (same
// tie rule: equal scores go to the lower block).  Dynamic smem: chunk keys.
template <int D>
__global__ void __launch_bounds__(kSelectThreads)
decode_select_kernel(const float* __restrict__ qgrp, const float* __restrict__ kbar,
                     uint32_t* __restrict__ cand_key, int32_t* __restrict__ cand_idx,
                     int32_t* __restrict__ idx, unsigned* __restrict__ counters, int Hkv,
                     long long cap_blocks, int bcur, int topk, int n_init, int n_local, int width,
                     int chunk, int n_chunks) {
  extern __shared__ uint32_t keys[];        // max(chunk, n_chunks * k) keys + as many ints
  __shared__ float qv[D];
  __shared__ int hist[256];
  __shared__ int scan_scratch[kSelectThreads / 32 + 1];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  __shared__ int s_last;
  const int ck = blockIdx.x % n_chunks;
  const int g = (blockIdx.x / n_chunks) % Hkv;
  const int b = blockIdx.x / (n_chunks * Hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* row = idx + ((long long)b * Hkv + g) * width;
  const int n_cand = max(0, bcur - n_local + 1 - n_init);
  const int k = min(topk, n_cand);
  const int n_first = min(n_init, bcur + 1);
  const int local_lo = max(n_init, bcur - n_local + 1);
  const int n_loc = max(0, bcur - local_lo + 1);
  if (k == 0 || k == n_cand) {
    if (ck != 0) return;
    for (int e = tid; e < n_first; e += kSelectThreads) row[e] = e;
    for (int e = tid; e < k; e += kSelectThreads) row[n_first + e] = n_init + e;
    for (int e = tid; e < n_loc; e += kSelectThreads) row[n_first + k + e] = local_lo + e;
    for (int e = n_first + k + n_loc + tid; e < width; e += kSelectThreads) row[e] = -1;
    return;
  }
  // ---- score this chunk
  const int c0 = ck * chunk, nc = min(chunk, n_cand - c0);
  for (int e = tid; e < D; e += kSelectThreads) qv[e] = qgrp[((long long)b * Hkv + g) * D + e];
  __syncthreads();
  // one thread per candidate: its whole block-mean row is read with 16-byte
  // loads that are all independent, so many rows are in flight at once
  const float inv_sqrt_d = rsqrtf((float)D);
  for (int c = tid; c < nc; c += kSelectThreads) {
    const float4* kr = reinterpret_cast<const float4*>(
        kbar + (((long long)b * cap_blocks + n_init + c0 + c) * Hkv + g) * D);
    float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
    for (int e = 0; e < D / 4; ++e) {
      const float4 kv = kr[e];
      p0 = fmaf(qv[4 * e], kv.x, p0);
      p1 = fmaf(qv[4 * e + 1], kv.y, p1);
      p2 = fmaf(qv[4 * e + 2], kv.z, p2);
      p3 = fmaf(qv[4 * e + 3], kv.w, p3);
    }
    keys[c] = score_key(((p0 + p1) + (p2 + p3)) * inv_sqrt_d);
  }
  (void)lane;
  (void)warp;
  __syncthreads();
  // ---- local top-k: positions into the ints after the keys
  int32_t* pos_list = reinterpret_cast<int32_t*>(keys + chunk);
  const int kl = min(k, nc);
  if (kl == nc) {
    for (int e = tid; e < nc; e += kSelectThreads) pos_list[e] = e;
  } else {
    topk_emit_sorted(keys, nc, kl, pos_list, 0, hist, scan_scratch, &s_prefix, &s_need);
  }
  __syncthreads();
  const long long cbase = (((long long)b * Hkv + g) * n_chunks + ck) * topk;
  for (int e = tid; e < k; e += kSelectThreads) {
    if (e < kl) {
      cand_key[cbase + e] = keys[pos_list[e]];
      cand_idx[cbase + e] = n_init + c0 + pos_list[e];
    } else {
      cand_key[cbase + e] = 0u;       // below every real score key
      cand_idx[cbase + e] = -1;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0)
    s_last = atomicAdd(counters + ((long long)b * Hkv + g) * 2, 1u) == (unsigned)(n_chunks - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // ---- exact merge of the n_chunks local lists (chunk order = block order)
  const int total = n_chunks * k;
  uint32_t* mk = keys;
  int32_t* mi = reinterpret_cast<int32_t*>(keys + total);
  const long long gbase = ((long long)b * Hkv + g) * n_chunks * topk;
  for (int e = tid; e < total; e += kSelectThreads) {
    const int chk = e / k, r = e % k;
    mk[e] = cand_key[gbase + (long long)chk * topk + r];
    mi[e] = cand_idx[gbase + (long long)chk * topk + r];
  }
  __syncthreads();
  int32_t* chosen = mi + total;       // k positions
  topk_emit_sorted(mk, total, k, chosen, 0, hist, scan_scratch, &s_prefix, &s_need);
  __syncthreads();
  for (int e = tid; e < n_first; e += kSelectThreads) row[e] = e;
  for (int e = tid; e < k; e += kSelectThreads) row[n_first + e] = mi[chosen[e]];
  for (int e = tid; e < n_loc; e += kSelectThreads) row[n_first + k + e] = local_lo + e;
  for (int e = n_first + k + n_loc + tid; e < width; e += kSelectThreads) row[e] = -1;
}

// Partial attention of the group's G heads over one selected block, then the
// combine + gate in the last CTA of the (batch, kv head).  Keys / values are
// staged as bf16 in shared memory with 16-byte chunks XOR-swizzled by row.
// Partials: [B, Hkv, width, G, D + 4] = (m, l, -, -, o[D]) in base-2 logits.
template <typename T, int D>
__global__ void __launch_bounds__(256)
decode_attn_kernel(const float* __restrict__ qhat, const __nv_bfloat16* __restrict__ k_cache,
                   const __nv_bfloat16* __restrict__ v_cache, const int32_t* __restrict__ idx,
                   float* __restrict__ part, unsigned* __restrict__ counters,
                   const T* __restrict__ gate, T* __restrict__ out, int Hq, int Hkv,
                   long long cap, long long pos, int BLK, int width, float sl2) {
  constexpr int NC = D / 8;                 // 16-byte chunks per row
  constexpr int DP = D + 4;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint4* ks = reinterpret_cast<uint4*>(smem_raw);                 // [64][NC]
  uint4* vs = ks + 64 * NC;                                       // [64][NC]
  const int G = Hq / Hkv;
  float* qs = reinterpret_cast<float*>(vs + 64 * NC);             // [G][D]
  float* lg = qs + G * D;                                         // [G][64]
  float* ml = lg + G * 64;                                        // [G][2]
  __shared__ int s_last;
  const int slot = blockIdx.x % width;
  const int g = (blockIdx.x / width) % Hkv;
  const int b = blockIdx.x / (width * Hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = idx[((long long)b * Hkv + g) * width + slot];
  float* pbase = part + (((long long)b * Hkv + g) * width + slot) * G * DP;
  const bool valid = j >= 0 && (long long)j * BLK <= pos;
  if (j >= 0 && !valid) set_status(kStatusBounds);
  if (!valid) {
    // an empty slot: weight 0 in the combine, with finite (zero) partials
    for (int e = tid; e < G * DP; e += 256) pbase[e] = (e % DP) == 0 ? -INFINITY : 0.f;
  } else {
    const long long kend = ((long long)(j + 1) * BLK < pos + 1) ? (long long)(j + 1) * BLK : pos + 1;
    const int nk = (int)(kend - (long long)j * BLK);
    // all loads of this thread are issued before the first shared-memory store
    constexpr int PER = 64 * NC / 256;
    uint4 kr[PER], vr[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + 256 * u, s = e / NC, c = e % NC;
      kr[u] = vr[u] = make_uint4(0, 0, 0, 0);
      if (s < nk) {
        const long long off = (((long long)b * cap + (long long)j * BLK + s) * Hkv + g) * D + 8 * c;
        kr[u] = *reinterpret_cast<const uint4*>(k_cache + off);
        vr[u] = *reinterpret_cast<const uint4*>(v_cache + off);
      }
    }
    const float4* qsrc = reinterpret_cast<const float4*>(qhat + ((long long)b * Hq + g * G) * D);
    float4* qdst = reinterpret_cast<float4*>(qs);
    for (int e = tid; e < G * D / 4; e += 256) qdst[e] = qsrc[e];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + 256 * u, s = e / NC, c = e % NC;
      ks[s * NC + (c ^ (s & (NC - 1)))] = kr[u];
      vs[s * NC + (c ^ (s & (NC - 1)))] = vr[u];
    }
    __syncthreads();
    // logits: thread (key s, head hq + 4 m)
    {
      const int s = tid & 63;
      for (int h = tid >> 6; h < G; h += 4) {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        const float* qr = qs + h * D;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          float kf[8];
          load8(reinterpret_cast<const __nv_bfloat16*>(&ks[s * NC + (c ^ (s & (NC - 1)))]), kf);
          a0 = fmaf(kf[0], qr[8 * c + 0], a0); a1 = fmaf(kf[1], qr[8 * c + 1], a1);
          a2 = fmaf(kf[2], qr[8 * c + 2], a2); a3 = fmaf(kf[3], qr[8 * c + 3], a3);
          a0 = fmaf(kf[4], qr[8 * c + 4], a0); a1 = fmaf(kf[5], qr[8 * c + 5], a1);
          a2 = fmaf(kf[6], qr[8 * c + 6], a2); a3 = fmaf(kf[7], qr[8 * c + 7], a3);
        }
        lg[h * 64 + s] = s < nk ? ((a0 + a1) + (a2 + a3)) * sl2 : -INFINITY;
      }
    }
    __syncthreads();
    // softmax per head (one warp per head, two logits per lane)
    for (int h = warp; h < G; h += 8) {
      const float x0 = lg[h * 64 + lane], x1 = lg[h * 64 + lane + 32];
      const float m = warp_max(fmaxf(x0, x1));
      const float p0 = exp2f(x0 - m), p1 = exp2f(x1 - m);
      const float l = warp_sum(p0 + p1);
      lg[h * 64 + lane] = p0;
      lg[h * 64 + lane + 32] = p1;
      if (lane == 0) { ml[2 * h] = m; ml[2 * h + 1] = l; }
    }
    __syncthreads();
    // P V: thread (head, 8-column chunk)
    for (int e = tid; e < G * NC; e += 256) {
      const int h = e / NC, c = e % NC;
      float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < nk; ++s) {
        float vf[8];
        load8(reinterpret_cast<const __nv_bfloat16*>(&vs[s * NC + (c ^ (s & (NC - 1)))]), vf);
        const float p = lg[h * 64 + s];
#pragma unroll
        for (int u = 0; u < 8; ++u) o[u] = fmaf(p, vf[u], o[u]);
      }
      float* pr = pbase + h * DP;
      *reinterpret_cast<float4*>(pr + 4 + 8 * c) = make_float4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<float4*>(pr + 8 + 8 * c) = make_float4(o[4], o[5], o[6], o[7]);
      if (c == 0) { pr[0] = ml[2 * h]; pr[1] = ml[2 * h + 1]; }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0)
    s_last = atomicAdd(counters + ((long long)b * Hkv + g) * 2 + 1, 1u) == (unsigned)(width - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // ---- combine the width partials of each head and apply the gate: the
  // (m, l) pairs of every slot are staged in shared memory first, turned into
  // weights 2^(m - M), then each thread streams its 8 output columns
  const float* gb = part + ((long long)b * Hkv + g) * width * G * DP;
  float* wgt = reinterpret_cast<float*>(smem_raw);        // [width][G] weights
  float* lv = wgt + width * G;                            // [width][G] partial sums
  float* lsum = lv + width * G;                           // [G]
  for (int e = tid; e < width * G; e += 256) {
    const float* pr = gb + (long long)e * DP;             // slot e / G, head e % G
    wgt[e] = pr[0];
    lv[e] = pr[1];
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int sl = 0; sl < width; ++sl) M = fmaxf(M, wgt[sl * G + tid]);
    float L = 0.f;
    for (int sl = 0; sl < width; ++sl) {
      const float m = wgt[sl * G + tid];
      const float f = m == -INFINITY ? 0.f : exp2f(m - M);
      wgt[sl * G + tid] = f;
      L = fmaf(f, lv[sl * G + tid], L);
    }
    lsum[tid] = L;
  }
  __syncthreads();
  for (int e = tid; e < G * NC; e += 256) {
    const int h = e / NC, c = e % NC;
    const float L = lsum[h];
    float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // 8 slots per batch: their 16 loads are issued before any is used
    for (int s0 = 0; s0 < width; s0 += 8) {
      float4 a[8], bq[8];
      float f[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int sl = min(s0 + u, width - 1);
        const float* pr = gb + ((long long)sl * G + h) * DP;
        a[u] = *reinterpret_cast<const float4*>(pr + 4 + 8 * c);
        bq[u] = *reinterpret_cast<const float4*>(pr + 8 + 8 * c);
        f[u] = s0 + u < width ? wgt[sl * G + h] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        o[0] = fmaf(f[u], a[u].x, o[0]); o[1] = fmaf(f[u], a[u].y, o[1]);
        o[2] = fmaf(f[u], a[u].z, o[2]); o[3] = fmaf(f[u], a[u].w, o[3]);
        o[4] = fmaf(f[u], bq[u].x, o[4]); o[5] = fmaf(f[u], bq[u].y, o[5]);
        o[6] = fmaf(f[u], bq[u].z, o[6]); o[7] = fmaf(f[u], bq[u].w, o[7]);
      }
    }
    const long long off = ((long long)b * Hq + g * G + h) * D + 8 * c;
    float gv[8];
    load8(gate + off, gv);
    const float inv = 1.f / L;
#pragma unroll
    for (int u = 0; u < 8; ++u) gv[u] = sigmoidf_(gv[u]) * o[u] * inv;
    store8(out + off, gv);
  }
}

}  // namespace sala
