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
// Four launches per token: (1) linear-layer state updates and the sparse
// layer's normalisation / cache append in one grid; (2) block scores with a
// per-chunk top-k, merged exactly by the last CTA of each kv head; (3) one
// CTA per selected block computing partial softmax sums; (4) their combine
// and the gate, one CTA per q head.
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
  unsigned* counters;   // [B, Hkv, 2]: selection completion counts (second unused)
};


// cos / sin of p * base^(-2i/D): the argument is formed and reduced modulo
// 2 pi in fp64 (|p| < 2^53), then evaluated in fp32 on [-pi, pi].
__device__ __forceinline__ void rope_cs(long long p, double inv_freq, float& c, float& s) {
  const double a = (double)p * inv_freq;
  const double two_pi = 6.283185307179586476925286766559;
  const double r = a - rint(a / two_pi) * two_pi;
  sincosf((float)r, &s, &c);
}

// Stage 1.  CTAs [0, n_lin): one per (linear layer, batch, head, 64-column
// slice) updating S <- lam S + k^T v and writing out = sigmoid(g) q^ S.
// CTAs [n_lin, n_lin + B * n_sp): the sparse layer, one warp per row of the
// Hkv keys and Hq queries of batch b (normalise k and append it and v to the
// caches, update the running block sum / mean; normalise q); the first of
// them also resets the completion counters.
constexpr int kDecodeMaxQHeads = 64;   // largest sparse-layer q head count the decode step takes
constexpr int kDecodeRowsPerCta = 8;   // sparse-layer rows per stage-1 CTA

template <typename T, int D>
__global__ void __launch_bounds__(256)
decode_stage1_kernel(DecodeLinearArgs a, DecodeSparseArgs sp, int n_lin, int n_sp, int B, int H,
                     int Hq, int Hkv, long long cap, long long pos, int BLK, RopeFreq rf,
                     float eps_l, float eps_s, float scale) {
  __shared__ float sh[D * 3 + 256];
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
        rope_cs(pos, rf.inv[i], c, s);
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
    // all D/4 state loads of this thread are in flight before the first use
    constexpr int RPT = D / 4;
    float sv[RPT];
#pragma unroll
    for (int u = 0; u < RPT; ++u) sv[u] = S[(long long)(rg * RPT + u) * D + col];
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int u = 0; u < RPT; u += 2) {
      const int r = rg * RPT + u;
      const float s0 = lam * sv[u] + kh[r] * vc;
      const float s1 = lam * sv[u + 1] + kh[r + 1] * vc;
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
  // ---- sparse layer of batch b, rows [rc * 8, rc * 8 + 8) of its Hkv + Hq
  const int b = (blockIdx.x - n_lin) / n_sp;
  const int rc = (blockIdx.x - n_lin) % n_sp;
  const bool closes = ((pos + 1) % BLK) == 0;
  const T* q = static_cast<const T*>(sp.q);
  const T* k = static_cast<const T*>(sp.k);
  const T* v = static_cast<const T*>(sp.v);
  if (rc == 0 && tid < 2 * Hkv) sp.counters[(long long)b * Hkv * 2 + tid] = 0u;
  {
    const int r = rc * kDecodeRowsPerCta + warp;
    if (warp >= kDecodeRowsPerCta || r >= Hkv + Hq) return;
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
      for (int e = 0; e < D / 32; ++e) sp.qhat[((long long)b * Hq + h) * D + lane + 32 * e] = x[e];
    }
  }
}

// Top-k of the scored candidates: rows of the candidate chunks and, in the
// last CTA of each (batch, kv head), the exact merge.  Chunk `ck` scores
// candidates [ck * chunk, ck * chunk + chunk) of [n_init, n_init + n_cand)
// and keeps its local top-k (ascending block order); the union of the local
// lists contains the global top-k, so the last CTA selects it exactly (same
// tie rule: equal scores go to the lower block).  Dynamic smem: chunk keys.
template <int D>
__global__ void __launch_bounds__(kSelectThreads)
decode_select_kernel(const float* __restrict__ qhat, const float* __restrict__ kbar,
                     uint32_t* __restrict__ cand_key, int32_t* __restrict__ cand_idx,
                     int32_t* __restrict__ idx, unsigned* __restrict__ counters, int Hq, int Hkv,
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
  // group-summed query (fixed head order)
  const int G = Hq / Hkv;
  for (int e = tid; e < D; e += kSelectThreads) {
    float s = 0.f;
    for (int hh = 0; hh < G; ++hh) s += qhat[((long long)b * Hq + g * G + hh) * D + e];
    qv[e] = s;
  }
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

// Partial attention of the group's G heads over up to kDecodeBlocksPerCta
// selected blocks (online softmax across them).  Keys / values are staged as
// bf16 in shared memory with 16-byte chunks XOR-swizzled by row; the next
// block's loads are in flight while the current one is processed.  Partials:
// [B, Hkv, n_parts, G, D + 4] = (m, l, -, -, o[D]) in base-2 logits; they are
// combined by decode_combine_kernel.
constexpr int kDecodeBlocksPerCta = 1;

template <typename T, int D>
__global__ void __launch_bounds__(256)
decode_attn_kernel(const float* __restrict__ qhat, const __nv_bfloat16* __restrict__ k_cache,
                   const __nv_bfloat16* __restrict__ v_cache, const int32_t* __restrict__ idx,
                   float* __restrict__ part, int Hq, int Hkv, long long cap, long long pos,
                   int BLK, int width, int n_parts, float sl2) {
  constexpr int NC = D / 8;                 // 16-byte chunks per row
  constexpr int DP = D + 4;
  constexpr int PER = 64 * NC / 256;        // 16-byte K (and V) chunks per thread and block
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint4* ks = reinterpret_cast<uint4*>(smem_raw);                 // [64][NC]
  uint4* vs = ks + 64 * NC;                                       // [64][NC]
  const int G = Hq / Hkv;
  float* qs = reinterpret_cast<float*>(vs + 64 * NC);             // [G][D]
  float* lg = qs + G * D;                                         // [G][64]
  float* os = lg + G * 64;                                        // [G][D] running outputs
  float* ml = os + G * D;                                         // [G][2] running (m, l)
  float* fs = ml + 2 * G;                                         // [G] rescale factors
  const int pidx = blockIdx.x % n_parts;
  const int g = (blockIdx.x / n_parts) % Hkv;
  const int b = blockIdx.x / (n_parts * Hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* irow = idx + ((long long)b * Hkv + g) * width;
  float* pbase = part + (((long long)b * Hkv + g) * n_parts + pidx) * G * DP;
  const int slot0 = pidx * kDecodeBlocksPerCta;
  const int nslot = min(kDecodeBlocksPerCta, width - slot0);
  // blocks of this CTA that hold keys (entries of the list are ascending)
  auto block_of = [&](int u) -> int {
    const int j = irow[slot0 + u];
    if (j >= 0 && (long long)j * BLK > pos) {
      set_status(kStatusBounds);
      return -1;
    }
    return j;
  };
  auto load_block = [&](int j, uint4* kr, uint4* vr) {
    const long long kend = ((long long)(j + 1) * BLK < pos + 1) ? (long long)(j + 1) * BLK : pos + 1;
    const int nk = (int)(kend - (long long)j * BLK);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + 256 * u, sr = e / NC, c = e % NC;
      kr[u] = vr[u] = make_uint4(0, 0, 0, 0);
      if (sr < nk) {
        const long long off = (((long long)b * cap + (long long)j * BLK + sr) * Hkv + g) * D + 8 * c;
        kr[u] = *reinterpret_cast<const uint4*>(k_cache + off);
        vr[u] = *reinterpret_cast<const uint4*>(v_cache + off);
      }
    }
    return nk;
  };
  {
    const float4* qsrc = reinterpret_cast<const float4*>(qhat + ((long long)b * Hq + g * G) * D);
    float4* qdst = reinterpret_cast<float4*>(qs);
    for (int e = tid; e < G * D / 4; e += 256) qdst[e] = qsrc[e];
    for (int e = tid; e < G * D; e += 256) os[e] = 0.f;
    for (int e = tid; e < G; e += 256) { ml[2 * e] = -INFINITY; ml[2 * e + 1] = 0.f; }
  }
  uint4 kr[PER], vr[PER];
  int u = 0, j = -1, nk = 0;
  while (u < nslot && (j = block_of(u)) < 0) ++u;
  if (j >= 0) nk = load_block(j, kr, vr);
  while (j >= 0) {
    __syncthreads();                      // previous block's readers are done
#pragma unroll
    for (int w = 0; w < PER; ++w) {
      const int e = tid + 256 * w, sr = e / NC, c = e % NC;
      ks[sr * NC + (c ^ (sr & (NC - 1)))] = kr[w];
      vs[sr * NC + (c ^ (sr & (NC - 1)))] = vr[w];
    }
    const int cur_nk = nk;
    // next block's loads overlap this block's arithmetic
    int jn = -1;
    ++u;
    while (u < nslot && (jn = block_of(u)) < 0) ++u;
    if (u >= nslot) jn = -1;
    if (jn >= 0) nk = load_block(jn, kr, vr);
    __syncthreads();
    // logits: thread (key s, head hq + 4 m)
    {
      const int sr = tid & 63;
      for (int h = tid >> 6; h < G; h += 4) {
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
        lg[h * 64 + sr] = sr < cur_nk ? ((a0 + a1) + (a2 + a3)) * sl2 : -INFINITY;
      }
    }
    __syncthreads();
    // online softmax per head (one warp per head, two logits per lane)
    for (int h = warp; h < G; h += 8) {
      const float x0 = lg[h * 64 + lane], x1 = lg[h * 64 + lane + 32];
      const float mo = ml[2 * h];
      const float mn = fmaxf(mo, warp_max(fmaxf(x0, x1)));
      const float p0 = exp2f(x0 - mn), p1 = exp2f(x1 - mn);
      const float ls = warp_sum(p0 + p1);
      lg[h * 64 + lane] = p0;
      lg[h * 64 + lane + 32] = p1;
      if (lane == 0) {
        const float f = mo == -INFINITY ? 0.f : exp2f(mo - mn);
        fs[h] = f;
        ml[2 * h] = mn;
        ml[2 * h + 1] = ml[2 * h + 1] * f + ls;
      }
    }
    __syncthreads();
    // O = f O + P V: thread (head, 8-column chunk)
    for (int e = tid; e < G * NC; e += 256) {
      const int h = e / NC, c = e % NC;
      float o[8];
      const float f = fs[h];
#pragma unroll
      for (int w = 0; w < 8; ++w) o[w] = os[h * D + 8 * c + w] * f;
      for (int sr = 0; sr < cur_nk; ++sr) {
        float vf[8];
        load8(reinterpret_cast<const __nv_bfloat16*>(&vs[sr * NC + (c ^ (sr & (NC - 1)))]), vf);
        const float p = lg[h * 64 + sr];
#pragma unroll
        for (int w = 0; w < 8; ++w) o[w] = fmaf(p, vf[w], o[w]);
      }
#pragma unroll
      for (int w = 0; w < 8; ++w) os[h * D + 8 * c + w] = o[w];
    }
    j = jn;
  }
  __syncthreads();
  // partial of this CTA (m = -inf, zeros when it held no key)
  for (int e = tid; e < G * DP; e += 256) {
    const int h = e / DP, c = e % DP;
    pbase[e] = c == 0 ? ml[2 * h] : (c == 1 ? ml[2 * h + 1] : (c < 4 ? 0.f : os[h * D + c - 4]));
  }
}

// Combine of the n_parts partials of one q head and the output gate: one CTA
// per (batch, q head), one thread per output column.
template <typename T, int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const float* __restrict__ part, const T* __restrict__ gate,
                      T* __restrict__ out, int Hq, int Hkv, int n_parts) {
  constexpr int DP = D + 4;
  extern __shared__ float wl[];                          // [n_parts] weights, [n_parts] sums
  __shared__ float s_l;
  const int hq = blockIdx.x % Hq;
  const int b = blockIdx.x / Hq;
  const int G = Hq / Hkv, g = hq / G, h = hq % G;
  const int tid = threadIdx.x;
  const float* pb = part + (((long long)b * Hkv + g) * n_parts * G + h) * DP;
  const long long pstride = (long long)G * DP;
  for (int e = tid; e < n_parts; e += D) {
    wl[e] = pb[e * pstride];
    wl[n_parts + e] = pb[e * pstride + 1];
  }
  __syncthreads();
  if (tid < 32) {
    float M = -INFINITY;
    for (int e = tid; e < n_parts; e += 32) M = fmaxf(M, wl[e]);
    M = warp_max(M);
    float L = 0.f;
    for (int e = tid; e < n_parts; e += 32) {
      const float f = wl[e] == -INFINITY ? 0.f : exp2f(wl[e] - M);
      L = fmaf(f, wl[n_parts + e], L);
      wl[e] = f;
    }
    L = warp_sum(L);
    if (tid == 0) s_l = L;
  }
  __syncthreads();
  // 8 independent partial sums so that the loads of 8 partials overlap
  float o8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int e = 0;
  for (; e + 8 <= n_parts; e += 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) o8[u] = fmaf(wl[e + u], pb[(e + u) * pstride + 4 + tid], o8[u]);
  }
  for (; e < n_parts; ++e) o8[0] = fmaf(wl[e], pb[e * pstride + 4 + tid], o8[0]);
  const float o = ((o8[0] + o8[1]) + (o8[2] + o8[3])) + ((o8[4] + o8[5]) + (o8[6] + o8[7]));
  const long long off = ((long long)b * Hq + hq) * D + tid;
  out[off] = from_f32<T>(sigmoidf_(to_f32(gate[off])) * o / s_l);
}

}  // namespace sala
