// Sequence-parallel chunked linear attention on the 5th-generation tensor
// cores (bf16 activations, head_dim 128).
//
// Lightning attention (acgfav.com "SALA 混合架构": linear layers at O(N);
// MiniCPM-SALA paper section 2.1: constant-size state).  The kernels read the
// RAW q and k tiles and apply QK-RMSNorm and RoPE in shared memory (QK
// normalisation in every layer: MiniCPM-SALA paper, summary; RoPE kept in the
// linear layers: acgfav.com "SALA 混合架构"), so the normalised tensors never
// travel through HBM.  With q^, k^ normalised and rotated, the state after
// token t is
//   S_t = lam S_{t-1} + k^_t^T v_t,     o_t = scale * q^_t S_t,
// so the state entering any token range is a decayed sum over everything
// before it.  The sequence of every (batch, head) is cut into segments of
// whole 128-token tiles and computed in three launches:
//
//   1. segment sums   dS_s = sum_{j in s} lam^(end_s - 1 - j) k^_j^T v_j
//                     (one CTA per segment, K^T V on the tensor cores with
//                     the decay folded into the K rows in shared memory);
//   2. scan           S_start(0) = state_in (or 0),
//                     S_start(s+1) = lam^len_s S_start(s) + dS_s,
//                     state_out = S_start(n_seg)   (element-wise, fp32);
//   3. outputs        one CTA per segment, all 128 value columns, walking its
//                     tiles from S_start(s): per tile of L tokens
//                       P  = (Q^ K^T) . D,       D_ij = lam^(i-j), j <= i
//                       O  = Q' S_prev + P V,    Q'_i = lam^(i+1) q^_i
//                       S <- lam^L S_prev + K'^T V,   K'_j = lam^(L-1-j) k^_j
//                       out = sigmoid(G) . scale O
//                     (Q' and K' are the Q^ / K^ tiles rescaled in shared
//                     memory once Q^ K^T has read them, so both products
//                     accumulate into one TMEM accumulator.)
//
// Chunking (and segmenting) is exact, so the tile and segment sizes only
// change the rounding order.  Every mbarrier wait is bounded; a wait that
// runs out sets the device status word and the CTA winds down.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "prologue.cuh"
#include "tc_ptx.cuh"

namespace sala {

constexpr int kLsTile = 128;
constexpr int kLsTargetCtas = 1184;    // 8 waves of one CTA on each of 148 SMs

struct LinSegPlan {
  int n_tiles, seg_tiles, n_seg;
};
inline LinSegPlan lin_seg_plan(int batch, int heads, int N) {
  LinSegPlan p;
  p.n_tiles = (N + kLsTile - 1) / kLsTile;
  const int bh = batch * heads;
  int want = (kLsTargetCtas + bh - 1) / bh;
  want = want < 1 ? 1 : (want > p.n_tiles ? p.n_tiles : want);
  p.seg_tiles = (p.n_tiles + want - 1) / want;
  p.n_seg = (p.n_tiles + p.seg_tiles - 1) / p.seg_tiles;
  return p;
}

// Row r of a [128 x 128] bf16 tile stored as two 128-byte-swizzled column
// atoms of 64 (the TMA layout of a 64 x 128 box): multiply in place by f
// (packed bf16 multiplies; f itself is rounded to bf16).  The 16 chunks are
// loaded before any is written back so that their latencies overlap.
__device__ __forceinline__ void sw128_scale_row(uint8_t* tile, int r, float f) {
  const __nv_bfloat162 f2 = __float2bfloat162_rn(f);
  uint4 u[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    u[i] = *reinterpret_cast<const uint4*>(tile + (i >> 3) * 16384 + r * 128 + (((i & 7) ^ (r & 7)) << 4));
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u[i]);
#pragma unroll
    for (int e = 0; e < 4; ++e) h2[e] = __hmul2(h2[e], f2);
    *reinterpret_cast<uint4*>(tile + (i >> 3) * 16384 + r * 128 + (((i & 7) ^ (r & 7)) << 4)) = u[i];
  }
}

// RoPE frequencies base^(-2i/128), i < 64, rounded to fp32 (kernel parameter).
struct RopeF32 {
  float th[64];
};

// Frequencies theta_l and theta_{l+32} (fp64) of lane l of the calling warp,
// read once per kernel and kept in registers.
__device__ __forceinline__ double2 rope_lane_freqs(const RopeFreq& rf) {
  const int lane = threadIdx.x & 31;
  return make_double2(rf.inv[lane], rf.inv[lane + 32]);
}

// Base angles of a tile that starts at position p: lane l of the calling warp
// returns (p * theta_l, p * theta_{l+32}) reduced modulo 2 pi, formed in fp64
// (|p| < 2^53) and rounded to fp32.
__device__ __forceinline__ float2 rope_tile_base(long long p, double2 th) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
  const double a = (double)p * th.x, b = (double)p * th.y;
  return make_float2((float)fma(-rint(a * kInvTwoPi), kTwoPi, a),
                     (float)fma(-rint(b * kInvTwoPi), kTwoPi, b));
}

// Row r of the same layout holds one token's raw q (or k) vector of one head,
// at position (tile start + r): replace it in place by
//   f * RoPE(RMSNorm(x) * w, position)
// (RMSNorm over the 128 values, fp32, with the weights w [128] in shared
// memory; rotate-half RoPE, pairs (i, i + 64) = chunk c of atom 0 and chunk
// c of atom 1 at the same swizzled offset).  The angle of frequency i is
// base_i + r * theta_i, with base_i (the tile start's angle, reduced in fp64:
// rope_tile_base) taken from lane i % 32 of the warp's `base`; it lies in
// [-pi, pi + 127], where the special-function unit's sine and cosine are
// accurate to about 1e-6 without a further reduction.  All 32 lanes must
// call this.
__device__ __forceinline__ void sw128_norm_rope_row(uint8_t* tile, int r, const float* wsm,
                                                    float eps, float2 base, const RopeF32& rt,
                                                    float f) {
  uint8_t* row0 = tile + r * 128;
  uint8_t* row1 = tile + 16384 + r * 128;
  float ss = 0.f;
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    const int o = (ch ^ (r & 7)) << 4;
    float a[8], b[8];
    load8(reinterpret_cast<const __nv_bfloat16*>(row0 + o), a);
    load8(reinterpret_cast<const __nv_bfloat16*>(row1 + o), b);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(a[e], a[e], fmaf(b[e], b[e], ss));
  }
  const float sc = rsqrtf(ss * (1.0f / 128) + eps) * f;
  const float rr = (float)r;
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    const int o = (ch ^ (r & 7)) << 4;
    float a[8], b[8], wa[8], wb[8];
    load8(reinterpret_cast<const __nv_bfloat16*>(row0 + o), a);
    load8(reinterpret_cast<const __nv_bfloat16*>(row1 + o), b);
    load8(wsm + ch * 8, wa);
    load8(wsm + 64 + ch * 8, wb);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = ch * 8 + e;
      // (x1, x2) = the pair (i, i + 64) times its weights; (c, s) = sc (cos, sin)
      const float2 x = __fmul2_rn(make_float2(a[e], b[e]), make_float2(wa[e], wb[e]));
      const float b0 = __shfl_sync(0xffffffffu, i < 32 ? base.x : base.y, i & 31);
      float sn, cs;
      __sincosf(fmaf(rr, rt.th[i], b0), &sn, &cs);
      const float2 cr = __fmul2_rn(make_float2(cs, sn), make_float2(sc, sc));
      // (x1 c - x2 s, x2 c + x1 s)
      const float2 y = __ffma2_rn(make_float2(x.x, x.y), make_float2(cr.x, cr.x),
                                  __fmul2_rn(make_float2(x.y, x.x), make_float2(-cr.y, cr.y)));
      a[e] = y.x;
      b[e] = y.y;
    }
    store8(reinterpret_cast<__nv_bfloat16*>(row0 + o), a);
    store8(reinterpret_cast<__nv_bfloat16*>(row1 + o), b);
  }
}

// 32 fp32 values -> bf16 columns [32 j, 32 j + 32) of row r of the same layout.
__device__ __forceinline__ void sw128_store_row32(uint8_t* tile, int r, int j, const float* v) {
  uint8_t* atom = tile + (j >> 1) * 16384 + r * 128;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ch = (j & 1) * 4 + q;
    uint4 u;
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) h2[e] = __floats2bfloat162_rn(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1]);
    *reinterpret_cast<uint4*>(atom + ((ch ^ (r & 7)) << 4)) = u;
  }
}

// --------------------------------------------------------------------------
// 1. Segment sums
// --------------------------------------------------------------------------

constexpr int kLsSumThreads = 512;     // warps 0-3: TMA, MMA, TMEM; 4-15: one scaling WG per stage
constexpr int kLsSumStages = 3;

struct LsSumLayout {
  static constexpr int kStage = 65536;               // K^ tile, V tile (2 atoms x 16 KB each)
  static constexpr int kV = 32768;
  static constexpr int kPw = kLsSumStages * kStage;  // lam^m, m = 0..128
  static constexpr int kBar = kPw + 4 * 132;         // ld_full[S], ld_empty[S], k_ready[S], done
  static constexpr int kMisc = kBar + 8 * (3 * kLsSumStages + 1);
  // 16-byte aligned: read with 16-byte vector loads
  static constexpr int kW = (kMisc + 16 + 15) / 16 * 16;   // RMSNorm weights of k, 128 floats
  static constexpr int kBytes = kW + 512;
  static_assert(kW % 16 == 0 && kBar % 8 == 0, "shared-memory alignment");
};

__global__ void __launch_bounds__(kLsSumThreads, 1)
linear_segsum_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const float* __restrict__ lambda,
                     const float* __restrict__ wk, float eps, long long pos0,
                     const __grid_constant__ RopeFreq rf, const __grid_constant__ RopeF32 rt,
                     float* __restrict__ seg_state, int N, int H, int seg_tiles, int n_seg) {
  using L = LsSumLayout;
  constexpr int D = 128;
  extern __shared__ __align__(1024) uint8_t smem_ls[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_ls) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* ld_full = bars;
  uint64_t* ld_empty = bars + kLsSumStages;
  uint64_t* k_ready = bars + 2 * kLsSumStages;
  uint64_t* done = bars + 3 * kLsSumStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  float* pw = reinterpret_cast<float*>(smem + L::kPw);
  float* wsm = reinterpret_cast<float*>(smem + L::kW);

  const int s = blockIdx.x % n_seg;
  const int h = (blockIdx.x / n_seg) % H;
  const int b = blockIdx.x / (n_seg * H);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = s * seg_tiles;
  const int n_tiles_all = (N + kLsTile - 1) / kLsTile;
  const int nt = min(seg_tiles, n_tiles_all - t0);
  const int seg_end = min(N, (t0 + nt) * kLsTile);
  const float lam = lambda[h];

  if (threadIdx.x == 0) {
    for (int i = 0; i < kLsSumStages; ++i) {
      tc::mbar_init(ld_full + i, 1);
      tc::mbar_init(ld_empty + i, 1);
      tc::mbar_init(k_ready + i, 4);
    }
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  if (threadIdx.x <= kLsTile) pw[threadIdx.x] = (float)pow((double)lam, (double)threadIdx.x);
  if (threadIdx.x < D) wsm[threadIdx.x] = wk[threadIdx.x];
  if (warp == 2) {
    tc::tmem_alloc(tmem_slot, 128);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (tc::elect_one()) {
      tc::tma_prefetch(&kmap);
      tc::tma_prefetch(&vmap);
      for (int c = 0; c < nt; ++c) {
        const int st = c % kLsSumStages, use = c / kLsSumStages;
        if (use > 0 && !tc::mbar_wait(ld_empty + st, (use - 1) & 1)) break;
        uint8_t* stage = smem + st * L::kStage;
        tc::mbar_expect_tx(ld_full + st, L::kStage);
        const int row0 = b * N + (t0 + c) * kLsTile;
        for (int a = 0; a < 2; ++a) {
          tc::tma_load_2d(stage + a * 16384, &kmap, ld_full + st, h * D + 64 * a, row0);
          tc::tma_load_2d(stage + L::kV + a * 16384, &vmap, ld_full + st, h * D + 64 * a, row0);
        }
      }
    }
  } else if (warp == 1) {
    if (tc::elect_one()) {
      constexpr uint32_t id = tc::idesc_bf16_f32(128, 128, true, true);
      const uint32_t base = tc::smem_u32(smem);
      bool ok = true;
      for (int c = 0; ok && c < nt; ++c) {
        const int st = c % kLsSumStages;
        if (!(ok = tc::mbar_wait(k_ready + st, (c / kLsSumStages) & 1))) break;
        tc::tc_fence_after();
        const uint32_t k = base + st * L::kStage, v = k + L::kV;
        // dS += K'^T V   (A = K' read MN-major, B = V MN-major)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16_ss(tmem, tc::smem_desc_sw128(k + kk * 2048, 16384, 1024),
                          tc::smem_desc_sw128(v + kk * 2048, 16384, 1024), id, c > 0 || kk > 0);
        tc::mma_commit(ld_empty + st);
      }
      tc::mma_commit(done);
    }
  } else if (warp >= 4) {
    // scaling warpgroup a handles the tiles of stage a (c = a, a + 3, ...)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int a = (warp - 4) >> 2;
    const double2 th = rope_lane_freqs(rf);
    bool ok = true;
    for (int c = a; ok && c < nt; c += kLsSumStages) {
      const int st = a;
      const int tile_start = (t0 + c) * kLsTile;
      const int Lt = min(kLsTile, N - tile_start);
      // k^_j (normalised, rotated at its position) scaled by
      // lam^(seg_end - 1 - j) = lam^(seg_end - tile_end) lam^(L - 1 - r); the
      // tile factor is formed in fp64 by one lane while the loads land
      float ft = 0.f;
      if (lane == 0) ft = (float)pow((double)lam, (double)(seg_end - (tile_start + Lt)));
      ft = __shfl_sync(0xffffffffu, ft, 0);
      const float2 base = rope_tile_base(pos0 + tile_start, th);
      ok = __all_sync(0xffffffffu, tc::mbar_wait(ld_full + st, (c / kLsSumStages) & 1));
      if (!ok) break;
      const float f = r < Lt ? ft * pw[Lt - 1 - r] : 0.f;
      sw128_norm_rope_row(smem + st * L::kStage, r, wsm, eps, base, rt, f);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(k_ready + st);
    }
    // dS (row r = key dim, 128 value columns) -> seg_state, by warpgroup 0
    if (a == 0 && __all_sync(0xffffffffu, ok && tc::mbar_wait(done, 0))) {
      tc::tc_fence_after();
      float* dst = seg_state + ((((long long)b * H + h) * n_seg + s) * D + r) * D;
      const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float x[32];
        tc::tmem_ld32(lane_base + 32 * j, x);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + 32 * j + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 128);
  }
}

// --------------------------------------------------------------------------
// 2. Scan over segments (one thread per state element)
// --------------------------------------------------------------------------

constexpr int kLsScanThreads = 256;

__global__ void __launch_bounds__(kLsScanThreads)
linear_segscan_kernel(const float* __restrict__ lambda, const float* __restrict__ state_in,
                      float* __restrict__ state_out, float* __restrict__ seg_state, int N, int H,
                      int seg_tiles, int n_seg, long long n_elems) {
  constexpr int DD = 128 * 128;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_elems) return;
  const long long bh = i / DD;
  const int e = (int)(i % DD);
  const int h = (int)(bh % H);
  const double lam = lambda[h];
  const int seg_len = seg_tiles * kLsTile;
  const float lam_full = (float)pow(lam, (double)seg_len);
  const float lam_last = (float)pow(lam, (double)(N - (n_seg - 1) * seg_len));
  float S = state_in ? state_in[i] : 0.f;
  float* p = seg_state + bh * n_seg * DD + e;
  // segment sums are read 16 at a time so that the loads overlap
  for (int s0 = 0; s0 < n_seg; s0 += 16) {
    float ds[16];
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (s0 + u < n_seg) ds[u] = p[(long long)(s0 + u) * DD];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int s = s0 + u;
      if (s < n_seg) {
        p[(long long)s * DD] = S;                   // state entering segment s
        S = fmaf(s + 1 == n_seg ? lam_last : lam_full, S, ds[u]);
      }
    }
  }
  if (state_out) state_out[i] = S;
}

// --------------------------------------------------------------------------
// 3. Outputs
// --------------------------------------------------------------------------

constexpr int kLsOutThreads = 512;

struct LsOutLayout {
  static constexpr int kQ = 0, kK = 32768, kV = 65536;   // per stage, 2 atoms x 16 KB each
  static constexpr int kStage = 98304;
  static constexpr int kS = 2 * kStage;                  // S_prev bf16, 2 atoms x 16 KB
  static constexpr int kPw = kS + 32768;                 // lam^m, m = 0..128
  static constexpr int kBar = kPw + 4 * 132;
  // ld_full[2], ld_empty[2], qk_full, qk_empty, p_full, qk_scaled, s_scaled, s_full,
  // s_smem_full, s_smem_empty, o_full[2], o_empty[2], fin, qk_ready
  static constexpr int kNumBars = 4 + 8 + 4 + 1 + 1;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  // 16-byte aligned: read with 16-byte vector loads
  static constexpr int kW = (kMisc + 16 + 15) / 16 * 16;  // RMSNorm weights of q, k: 2 x 128 floats
  static constexpr int kBytes = kW + 1024;
  static_assert(kW % 16 == 0 && kBar % 8 == 0, "shared-memory alignment");
  // TMEM columns
  static constexpr int kColQK = 0;     // Q^ K^T; P (bf16 pairs) overwrites its first 64 columns
  static constexpr int kColO = 128;    // O of tile c in columns 128 + 128 (c & 1)
  static constexpr int kColS = 384;    // state (fp32), rows = key dim
};

// Warpgroup roles: warpgroup 0 holds the TMA producer (warp 0), the MMA
// issuer (warp 1, one elected thread) and the TMEM owner (warp 2) and gives
// registers away (56 per thread); warpgroups 1-3 take them (152 per thread):
// warpgroup 1 normalises and rotates the raw Q rows of each tile in place and
// rescales Q^ into Q', warpgroup 2 does the same for K; warpgroup 3 (one warp
// per TMEM lane quadrant) builds P, carries the state (fp32 in TMEM; a bf16
// copy in shared memory is the B operand of the next Q' S product) and runs
// the gated epilogue of tile c while tile c + 1 accumulates into the other O
// buffer.  The row transforms of tile c + 1 thus run while P, P V and the
// epilogue of tile c do.  56 x 128 + 152 x 384 = 65536 = 128 x 512, the
// registers the block is launched with (the host checks the 128).
constexpr int kLsOutRegsLaunch = 128;
constexpr int kLsOutRegsLow = 56;
constexpr int kLsOutRegsHigh = 152;
static_assert(kLsOutRegsLow * 128 + kLsOutRegsHigh * 384 <= kLsOutRegsLaunch * kLsOutThreads,
              "register split exceeds the launch allocation");
template <typename T>
__global__ void __launch_bounds__(kLsOutThreads, 1)
linear_segout_kernel(const __grid_constant__ CUtensorMap qmap,
                     const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap,
                     const __grid_constant__ CUtensorMap gmap, const T* __restrict__ gate,
                     const float* __restrict__ lambda, const float* __restrict__ wq,
                     const float* __restrict__ wk, float eps, long long pos0,
                     const __grid_constant__ RopeFreq rf, const __grid_constant__ RopeF32 rt,
                     const float* __restrict__ seg_state,
                     T* __restrict__ out, int N, int H, int seg_tiles, int n_seg, float scale) {
  using L = LsOutLayout;
  constexpr int D = 128;
  extern __shared__ __align__(1024) uint8_t smem_lo[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_lo) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* ld_full = bars;              // [2]
  uint64_t* ld_empty = bars + 2;         // [2]
  uint64_t* qk_full = bars + 4;
  uint64_t* qk_empty = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* qk_scaled = bars + 7;
  uint64_t* s_scaled = bars + 8;
  uint64_t* s_full = bars + 9;
  uint64_t* s_smem_full = bars + 10;
  uint64_t* s_smem_empty = bars + 11;
  uint64_t* o_full = bars + 12;          // [2]
  uint64_t* o_empty = bars + 14;         // [2]
  uint64_t* fin = bars + 16;
  uint64_t* qk_ready = bars + 17;        // raw Q and K of the tile normalised and rotated
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  float* pw = reinterpret_cast<float*>(smem + L::kPw);
  float* wsm = reinterpret_cast<float*>(smem + L::kW);   // [0, 128): wq, [128, 256): wk

  const int s = blockIdx.x % n_seg;
  const int h = (blockIdx.x / n_seg) % H;
  const int b = blockIdx.x / (n_seg * H);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = s * seg_tiles;
  const int nt = min(seg_tiles, (N + kLsTile - 1) / kLsTile - t0);
  const float lam = lambda[h];
  auto tile_len = [&](int c) { return min(kLsTile, N - (t0 + c) * kLsTile); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(ld_full + i, 1);
      tc::mbar_init(ld_empty + i, 1);
    }
    tc::mbar_init(qk_full, 1);
    tc::mbar_init(qk_empty, 1);
    tc::mbar_init(p_full, 4);
    tc::mbar_init(qk_scaled, 8);
    tc::mbar_init(s_scaled, 4);
    tc::mbar_init(s_full, 1);
    tc::mbar_init(s_smem_full, 4);
    tc::mbar_init(s_smem_empty, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(o_full + i, 1);
      tc::mbar_init(o_empty + i, 4);
    }
    tc::mbar_init(fin, 1);
    tc::mbar_init(qk_ready, 8);
    tc::fence_barrier_init();
  }
  if (threadIdx.x <= kLsTile) pw[threadIdx.x] = (float)pow((double)lam, (double)threadIdx.x);
  if (threadIdx.x < 2 * D) wsm[threadIdx.x] = threadIdx.x < D ? wq[threadIdx.x] : wk[threadIdx.x - D];
  if (warp == 2) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // each role starts with its register reallocation, so that the compiler
  // allocates every role's code within its own budget
  if (warp < 4) {
    tc::setmaxnreg_dec<kLsOutRegsLow>();
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (tc::elect_one()) {
        tc::tma_prefetch(&qmap);
        tc::tma_prefetch(&kmap);
        tc::tma_prefetch(&vmap);
        for (int c = 0; c < nt; ++c) {
          const int st = c & 1, use = c >> 1;
          if (use > 0 && !tc::mbar_wait(ld_empty + st, (use - 1) & 1)) break;
          uint8_t* stage = smem + st * L::kStage;
          tc::mbar_expect_tx(ld_full + st, L::kStage);
          const int row0 = b * N + (t0 + c) * kLsTile;
          for (int a = 0; a < 2; ++a) {
            tc::tma_load_2d(stage + L::kQ + a * 16384, &qmap, ld_full + st, h * D + 64 * a, row0);
            tc::tma_load_2d(stage + L::kK + a * 16384, &kmap, ld_full + st, h * D + 64 * a, row0);
            tc::tma_load_2d(stage + L::kV + a * 16384, &vmap, ld_full + st, h * D + 64 * a, row0);
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (tc::elect_one()) {
        constexpr uint32_t id_kk = tc::idesc_bf16_f32(128, 128, false, false);   // A, B K-major
        constexpr uint32_t id_kn = tc::idesc_bf16_f32(128, 128, false, true);    // B MN-major
        constexpr uint32_t id_nn = tc::idesc_bf16_f32(128, 128, true, true);     // A, B MN-major
        const uint32_t base = tc::smem_u32(smem);
        const uint32_t sb = base + L::kS;
        bool ok = true;
        for (int c = 0; ok && c < nt; ++c) {
          const int st = c & 1;
          const uint32_t q = base + st * L::kStage + L::kQ, k = base + st * L::kStage + L::kK,
                         v = base + st * L::kStage + L::kV;
          // QK = Q^ K^T (raw tiles normalised and rotated in place first)
          if (!(ok = tc::mbar_wait(ld_full + st, (c >> 1) & 1))) break;
          if (!(ok = tc::mbar_wait(qk_ready, c & 1))) break;
          if (c > 0 && !(ok = tc::mbar_wait(qk_empty, (c - 1) & 1))) break;
          tc::tc_fence_after();
  #pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_bf16_ss(tmem + L::kColQK, tc::smem_desc_sw128(q + off, 16, 1024),
                            tc::smem_desc_sw128(k + off, 16, 1024), id_kk, kk > 0);
          }
          tc::mma_commit(qk_full);
          // O = Q' S_prev  (Q' rescaled in place; B = S bf16, MN-major)
          const uint32_t o = tmem + L::kColO + 128 * (c & 1);
          if (!(ok = tc::mbar_wait(qk_scaled, c & 1))) break;
          if (!(ok = tc::mbar_wait(s_smem_full, c & 1))) break;
          if (c >= 2 && !(ok = tc::mbar_wait(o_empty + (c & 1), ((c >> 1) - 1) & 1))) break;
          tc::tc_fence_after();
  #pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_bf16_ss(o, tc::smem_desc_sw128(q + off, 16, 1024),
                            tc::smem_desc_sw128(sb + kk * 2048, 16384, 1024), id_kn, kk > 0);
          }
          tc::mma_commit(s_smem_empty);
          // S = lam^L S_prev + K'^T V  (S already scaled in TMEM; A = K' MN-major)
          if (!(ok = tc::mbar_wait(s_scaled, c & 1))) break;
          tc::tc_fence_after();
  #pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16_ss(tmem + L::kColS, tc::smem_desc_sw128(k + kk * 2048, 16384, 1024),
                            tc::smem_desc_sw128(v + kk * 2048, 16384, 1024), id_nn, true);
          tc::mma_commit(s_full);
          // O += P V  (P from TMEM)
          if (!(ok = tc::mbar_wait(p_full, c & 1))) break;
          tc::tc_fence_after();
  #pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16_ts(o, tmem + L::kColQK + kk * 8,
                            tc::smem_desc_sw128(v + kk * 2048, 16384, 1024), id_kn, true);
          tc::mma_commit(qk_empty);
          tc::mma_commit(o_full + (c & 1));
          tc::mma_commit(ld_empty + st);
        }
        tc::mma_commit(fin);
        tc::mbar_wait(fin, 0);
      }
    }

  } else if (warp < 12) {
    // -------------------------------------------- Q (warps 4-7) / K (warps 8-11)
    // Normalise and rotate the raw rows of each tile in place, then rescale
    // them into Q' / K' once Q^ K^T has read the tile.  Nothing else: the
    // transform of tile c + 1 runs while warps 12-15 build P of tile c.
    tc::setmaxnreg_inc<kLsOutRegsHigh>();
    const bool is_k = warp >= 8;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int part = is_k ? L::kK : L::kQ;
    const float* w = wsm + (is_k ? D : 0);
    const double2 th = rope_lane_freqs(rf);
    for (int c = 0; c < nt; ++c) {
      const int Lt = tile_len(c);
      // raw row -> q^ / k^ (RMSNorm, RoPE at its position), in place
      const float2 base = rope_tile_base(pos0 + (long long)(t0 + c) * kLsTile, th);
      if (!__all_sync(0xffffffffu, tc::mbar_wait(ld_full + (c & 1), (c >> 1) & 1))) break;
      sw128_norm_rope_row(smem + (c & 1) * L::kStage + part, r, w, eps, base, rt, 1.f);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(qk_ready);
      if (!__all_sync(0xffffffffu, tc::mbar_wait(qk_full, c & 1))) break;
      // Q'_r = lam^(r+1) q^_r;  K'_r = lam^(L-1-r) k^_r (0 past the end)
      const float f = is_k ? (r < Lt ? pw[Lt - 1 - r] : 0.f) : pw[r + 1];
      sw128_scale_row(smem + (c & 1) * L::kStage + part, r, f);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(qk_scaled);
    }
  } else {
    // ------------------------------------- P, state and gated epilogue (warps 12-15)
    tc::setmaxnreg_inc<kLsOutRegsHigh>();
    const int quad = warp & 3;
    const int r = quad * 32 + lane;     // token row of P and O; key-dim row of S
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    // S_start: bf16 copy for the first Q^ S product, lam^L0 S_start into TMEM
    {
      const float* src = seg_state + ((((long long)b * H + h) * n_seg + s) * D + r) * D;
      const float f0 = pw[tile_len(0)];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float x[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 t = *reinterpret_cast<const float4*>(src + 32 * j + e);
          x[e] = t.x; x[e + 1] = t.y; x[e + 2] = t.z; x[e + 3] = t.w;
        }
        sw128_store_row32(smem + L::kS, r, j, x);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] *= f0;
        tc::tmem_st32(lane_base + L::kColS + 32 * j, x);
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(s_smem_full);
        tc::mbar_arrive(s_scaled);
      }
    }
    constexpr int kGW = 16 * (int)sizeof(T) / 16;     // 16-byte words per 16 gate values
    const float2 hs2 = make_float2(0.5f * scale, 0.5f * scale);
    // The gate tile of tile c + 1 is pulled into L2 by a bulk tensor prefetch
    // while tile c is written out; each thread then loads its whole gate row
    // before waiting for the accumulator.
    auto prefetch_gate = [&](int c) {
      if (warp == 12 && lane == 0 && c < nt) {
        const int row = b * N + (t0 + c) * kLsTile;
        tc::tma_prefetch_l2_2d(&gmap, h * D, row);
        tc::tma_prefetch_l2_2d(&gmap, h * D + 64, row);
      }
    };
    if (warp == 12 && lane == 0) tc::tma_prefetch(&gmap);
    prefetch_gate(0);
    for (int c = 0; c < nt; ++c) {
      // ---- P_rj = QK_rj lam^(r-j) for j <= r (rows past the end are never stored)
      // Row quadrant q has 32-column chunks 0..q on or below the diagonal; chunk
      // u of P (bf16 pairs) lands on columns [16 u, 16 u + 16) of the same rows,
      // which were read with chunk u / 2 <= u, so each chunk is written back as
      // soon as it is built.
      if (!__all_sync(0xffffffffu, tc::mbar_wait(qk_full, c & 1))) break;
      tc::tc_fence_after();
#pragma unroll
      for (int q0 = 0; q0 < 4; ++q0) {
        uint32_t pk[16];
        if (q0 <= quad) {
          float xv[32];
          tc::tmem_ld32(lane_base + L::kColQK + 32 * q0, xv);
          tc::tmem_wait_ld();
          if (q0 == quad) {
#pragma unroll
            for (int e = 0; e < 32; ++e) xv[e] = e <= lane ? xv[e] * pw[lane - e] : 0.f;
          } else {
            // element e decays by lam^(r - 32 q0 - e): pairs (e, e + 1) from the top
            const int a = r - 32 * q0;
            float2 dcy = make_float2(pw[a - 30], pw[a - 31]);
            const float2 l2 = make_float2(pw[2], pw[2]);
#pragma unroll
            for (int e = 30; e >= 0; e -= 2) {
              const float2 y = __fmul2_rn(make_float2(xv[e], xv[e + 1]), dcy);
              xv[e] = y.x;
              xv[e + 1] = y.y;
              dcy = __fmul2_rn(dcy, l2);
            }
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(xv[2 * e], xv[2 * e + 1]);
            pk[e] = *reinterpret_cast<uint32_t*>(&h2);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;      // above the diagonal
        }
        tc::tmem_st16_u(lane_base + L::kColQK + 16 * q0, pk);
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full);
      // ---- S_c: bf16 copy for the next Q^ S product, lam^L(c+1) S_c back into TMEM
      if (c + 1 < nt) {
        bool ok = __all_sync(0xffffffffu, tc::mbar_wait(s_full, c & 1));
        if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait(s_smem_empty, c & 1));
        if (!ok) break;
        tc::tc_fence_after();
        const float f = pw[tile_len(c + 1)];
        const float2 f2 = make_float2(f, f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float x[32];
          tc::tmem_ld32(lane_base + L::kColS + 32 * j, x);
          tc::tmem_wait_ld();
          sw128_store_row32(smem + L::kS, r, j, x);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 y = __fmul2_rn(make_float2(x[e], x[e + 1]), f2);
            x[e] = y.x;
            x[e + 1] = y.y;
          }
          tc::tmem_st32(lane_base + L::kColS + 32 * j, x);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(s_smem_full);
          tc::mbar_arrive(s_scaled);
        }
      }
      // ---- gated epilogue of tile c
      prefetch_gate(c + 1);
      const bool valid = r < tile_len(c);
      const long long row_off = (((long long)b * N + (long long)(t0 + c) * kLsTile + r) * H + h) * D;
      const uint4* gsrc = reinterpret_cast<const uint4*>(gate + row_off);
      T* dst = out + row_off;
      const uint32_t o = lane_base + L::kColO + 128 * (c & 1);
      uint4 graw[8][kGW];
      if (valid) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
          for (int e = 0; e < kGW; ++e) graw[j][e] = gsrc[j * kGW + e];
      }
      if (!__all_sync(0xffffffffu, tc::mbar_wait(o_full + (c & 1), (c >> 1) & 1))) break;
      tc::tc_fence_after();
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float ov[16];
        tc::tmem_ld16(o + 16 * j, ov);
        tc::tmem_wait_ld();
        if (j == 7) {
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(o_empty + (c & 1));
        }
        if (valid) {
          if constexpr (std::is_same<T, __nv_bfloat16>::value) {
            // out = (s/2 + s/2 tanh(g/2)) o = s sigmoid(g) o, in f32x2 pairs
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&graw[j][e]);
              uint4 res;
              __nv_bfloat162* r2 = reinterpret_cast<__nv_bfloat162*>(&res);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 hg = __fmul2_rn(__bfloat1622float2(g2[u]), make_float2(0.5f, 0.5f));
                float tx, ty;
                asm("tanh.approx.f32 %0, %1;" : "=f"(tx) : "f"(hg.x));
                asm("tanh.approx.f32 %0, %1;" : "=f"(ty) : "f"(hg.y));
                const float2 sg = __ffma2_rn(make_float2(tx, ty), hs2, hs2);
                const float2 ou = __fmul2_rn(sg, make_float2(ov[8 * e + 2 * u], ov[8 * e + 2 * u + 1]));
                r2[u] = __floats2bfloat162_rn(ou.x, ou.y);
              }
              *reinterpret_cast<uint4*>(dst + 16 * j + 8 * e) = res;
            }
          } else {
            const T* g = reinterpret_cast<const T*>(graw[j]);
#pragma unroll
            for (int e = 0; e < 16; e += 8) {
              float gv[8], o8[8];
              load8(g + e, gv);
#pragma unroll
              for (int u = 0; u < 8; ++u) o8[u] = sigmoid_tanh(gv[u]) * (scale * ov[e + u]);
              store8(dst + 16 * j + e, o8);
            }
          }
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace sala
