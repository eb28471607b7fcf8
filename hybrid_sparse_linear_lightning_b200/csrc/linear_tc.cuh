// Chunked linear attention on the 5th-generation tensor cores.
//
// Lightning attention (acgfav.com "SALA 混合架构": linear layers at O(N);
// MiniCPM-SALA paper section 2.1: constant-size state) computed over tiles of
// T = 128 tokens (two chunks of 64 at once: chunking is exact, so the tile
// size only changes the rounding order).  For tile c with L valid tokens,
// q^, k^ already normalised and rotated:
//   P       = (Q^ K^T) . D,            D_ij = lam^(i-j) for j <= i < L, else 0
//   O_intra = P V
//   O_inter = Q^ S_prev,               used as lam^(i+1) O_inter
//   dS      = K^T V',                  V'_j = lam^(L-1-j) v_j (0 for j >= L)
//   S       = lam^L S_prev + dS        (fp32, in registers)
//   out     = sigmoid(G) . scale (O_intra + lam^(i+1) O_inter)
//
// One CTA owns (batch, head, 32 value columns): 4 CTAs per head at d = 128,
// reading the same Q^/K^ tiles (shared through L2).  The d x 32 fp32 state
// slice lives in the registers of one warpgroup (one key-dim row per
// thread); a bf16 copy is written to shared memory as the B operand of the
// next tile's Q^ S product.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer (one
// elected thread), warp 2 TMEM owner, warps 4-7 build V' and P, warps 8-11
// update the state and run the gated epilogue.  Waits are bounded.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sala {

constexpr int kLinTcThreads = 384;
constexpr int kLinTile = 128;
constexpr int kLinCols = 32;
constexpr int kLinStages = 2;

struct LinTcLayout {
  // per stage: Q^ tile (2 atoms x 16 KB), K^ tile (same), V slice (128 rows x 64 B)
  static constexpr int kQ = 0;
  static constexpr int kK = 32768;
  static constexpr int kV = 65536;
  static constexpr int kStage = 65536 + 8192;
  static constexpr int kP = kLinStages * kStage;         // P: 2 atoms x [128 x 128 B]
  static constexpr int kVp = kP + 32768;                 // V': 128 rows x 64 B
  static constexpr int kS = kVp + 8192;                  // S bf16: 2 buffers x 128 rows x 64 B
  static constexpr int kPw = kS + 2 * 8192;              // lam^m, m = 0..128
  static constexpr int kBar = kPw + 4 * 132;
  // ld_full[2], ld_empty[2], qk_full, qk_empty, vp_full, vp_empty, p_full, p_empty,
  // ds_full, ds_empty, s_full[2], s_empty[2], o_full, o_empty, fin
  static constexpr int kNumBars = 2 * kLinStages + 10 + 4 + 1;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kTmemCols = 256;
  static constexpr int kColQK = 0, kColDS = 128, kColOi = 160, kColOe = 192;
};

// bf16 row of 32 values at row r of a 64-byte-swizzled tile
__device__ __forceinline__ void sw64_store_row(uint8_t* tile, int r, const float* v) {
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint4 u;
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) h2[e] = __floats2bfloat162_rn(v[ch * 8 + 2 * e], v[ch * 8 + 2 * e + 1]);
    *reinterpret_cast<uint4*>(tile + r * 64 + ((ch ^ ((r >> 1) & 3)) << 4)) = u;
  }
}
__device__ __forceinline__ void sw64_load_row(const uint8_t* tile, int r, float* v) {
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    const uint4 u = *reinterpret_cast<const uint4*>(tile + r * 64 + ((ch ^ ((r >> 1) & 3)) << 4));
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      v[ch * 8 + 2 * e] = f.x;
      v[ch * 8 + 2 * e + 1] = f.y;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kLinTcThreads, 1)
linear_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const T* __restrict__ gate,
                      const float* __restrict__ lambda, const float* __restrict__ state_in,
                      float* __restrict__ state_out, T* __restrict__ out, int N, int H,
                      float scale) {
  using L = LinTcLayout;
  constexpr int D = 128;
  constexpr int NS = D / kLinCols;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* ld_full = bars;
  uint64_t* ld_empty = bars + kLinStages;
  uint64_t* qk_full = bars + 2 * kLinStages;
  uint64_t* qk_empty = qk_full + 1;
  uint64_t* vp_full = qk_full + 2;
  uint64_t* vp_empty = qk_full + 3;
  uint64_t* p_full = qk_full + 4;
  uint64_t* p_empty = qk_full + 5;
  uint64_t* ds_full = qk_full + 6;
  uint64_t* ds_empty = qk_full + 7;
  uint64_t* o_full = qk_full + 8;
  uint64_t* o_empty = qk_full + 9;
  uint64_t* s_full = qk_full + 10;    // [2]
  uint64_t* s_empty = qk_full + 12;   // [2]
  uint64_t* fin = qk_full + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  float* pw = reinterpret_cast<float*>(smem + L::kPw);

  const int slice = blockIdx.x % NS;
  const int h = (blockIdx.x / NS) % H;
  const int b = blockIdx.x / (NS * H);
  const int col0 = slice * kLinCols;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + kLinTile - 1) / kLinTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLinStages; ++s) {
      tc::mbar_init(ld_full + s, 1);
      tc::mbar_init(ld_empty + s, 1);
    }
    tc::mbar_init(qk_full, 1);
    tc::mbar_init(qk_empty, 4);
    tc::mbar_init(vp_full, 4);
    tc::mbar_init(vp_empty, 1);
    tc::mbar_init(p_full, 4);
    tc::mbar_init(p_empty, 1);
    tc::mbar_init(ds_full, 1);
    tc::mbar_init(ds_empty, 4);
    tc::mbar_init(o_full, 1);
    tc::mbar_init(o_empty, 4);
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(s_full + x, 4);
      tc::mbar_init(s_empty + x, 1);
    }
    tc::mbar_init(fin, 1);
    tc::fence_barrier_init();
  }
  if (threadIdx.x <= kLinTile) pw[threadIdx.x] = (float)pow((double)lambda[h], (double)threadIdx.x);
  if (warp == 2) {
    tc::tmem_alloc(tmem_slot, L::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      tc::tma_prefetch(&qmap);
      tc::tma_prefetch(&kmap);
      tc::tma_prefetch(&vmap);
      for (int c = 0; c < n_tiles; ++c) {
        const int st = c % kLinStages, use = c / kLinStages;
        if (use > 0 && !tc::mbar_wait(ld_empty + st, (use - 1) & 1)) break;
        uint8_t* stage = smem + st * L::kStage;
        tc::mbar_expect_tx(ld_full + st, L::kStage);
        const int row0 = b * N + c * kLinTile;
        for (int a = 0; a < 2; ++a) {
          tc::tma_load_2d(stage + L::kQ + a * 16384, &qmap, ld_full + st, h * D + 64 * a, row0);
          tc::tma_load_2d(stage + L::kK + a * 16384, &kmap, ld_full + st, h * D + 64 * a, row0);
        }
        tc::tma_load_2d(stage + L::kV, &vmap, ld_full + st, h * D + col0, row0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      constexpr uint32_t id_qk = tc::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_ds = tc::idesc_bf16_f32(128, kLinCols, true, true);
      constexpr uint32_t id_o = tc::idesc_bf16_f32(128, kLinCols, false, true);
      const uint32_t base = tc::smem_u32(smem);
      bool ok = true;
      for (int c = 0; ok && c < n_tiles; ++c) {
        const int st = c % kLinStages;
        const uint32_t q = base + st * L::kStage + L::kQ, k = base + st * L::kStage + L::kK,
                       v = base + st * L::kStage + L::kV;
        if (!(ok = tc::mbar_wait(ld_full + st, (c / kLinStages) & 1))) break;
        if (c > 0 && !(ok = tc::mbar_wait(qk_empty, (c - 1) & 1))) break;
        tc::tc_fence_after();
        // QK = Q^ K^T  (A, B K-major)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + L::kColQK, tc::smem_desc_sw128(q + off, 16, 1024),
                          tc::smem_desc_sw128(k + off, 16, 1024), id_qk, kk > 0);
        }
        tc::mma_commit(qk_full);
        // dS = K^T V'  (A = K^ read MN-major, B = V' MN-major)
        if (!(ok = tc::mbar_wait(vp_full, c & 1))) break;
        if (c > 0 && !(ok = tc::mbar_wait(ds_empty, (c - 1) & 1))) break;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16_ss(tmem + L::kColDS, tc::smem_desc_sw128(k + kk * 2048, 16384, 1024),
                          tc::smem_desc_sw64(base + L::kVp + kk * 1024, 8192, 512), id_ds, kk > 0);
        tc::mma_commit(ds_full);
        tc::mma_commit(vp_empty);
        // O_inter = Q^ S_prev  (B = S bf16 MN-major)
        if (!(ok = tc::mbar_wait(s_full + (c & 1), (c >> 1) & 1))) break;
        if (c > 0 && !(ok = tc::mbar_wait(o_empty, (c - 1) & 1))) break;
        tc::tc_fence_after();
        const uint32_t sb = base + L::kS + (c & 1) * 8192;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + L::kColOe, tc::smem_desc_sw128(q + off, 16, 1024),
                          tc::smem_desc_sw64(sb + kk * 1024, 8192, 512), id_o, kk > 0);
        }
        tc::mma_commit(s_empty + (c & 1));
        // O_intra = P V
        if (!(ok = tc::mbar_wait(p_full, c & 1))) break;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + L::kColOi, tc::smem_desc_sw128(base + L::kP + off, 16, 1024),
                          tc::smem_desc_sw64(v + kk * 1024, 8192, 512), id_o, kk > 0);
        }
        tc::mma_commit(p_empty);
        tc::mma_commit(o_full);
        tc::mma_commit(ld_empty + st);
      }
      tc::mma_commit(fin);
      tc::mbar_wait(fin, 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ V' and P
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t qk_addr = tmem + ((uint32_t)(quad * 32) << 16) + L::kColQK;
    uint8_t* sP = smem + L::kP;
    uint8_t* sVp = smem + L::kVp;
    bool ok = true;
    for (int c = 0; ok && c < n_tiles; ++c) {
      const int st = c % kLinStages;
      const int Lv = min(kLinTile, N - c * kLinTile);
      // V'_r = lam^(L-1-r) v_r
      ok = __all_sync(0xffffffffu, tc::mbar_wait(ld_full + st, (c / kLinStages) & 1));
      if (ok && c > 0) ok = __all_sync(0xffffffffu, tc::mbar_wait(vp_empty, (c - 1) & 1));
      if (!ok) break;
      {
        float vv[32];
        sw64_load_row(smem + st * L::kStage + L::kV, r, vv);
        const float f = r < Lv ? pw[Lv - 1 - r] : 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) vv[e] *= f;
        sw64_store_row(sVp, r, vv);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(vp_full);
      }
      // P_rj = QK_rj lam^(r-j) for j <= r < L
      ok = __all_sync(0xffffffffu, tc::mbar_wait(qk_full, c & 1));
      if (ok && c > 0) ok = __all_sync(0xffffffffu, tc::mbar_wait(p_empty, (c - 1) & 1));
      if (!ok) break;
      tc::tc_fence_after();
#pragma unroll 1
      for (int q0 = 0; q0 < 4; ++q0) {
        float x[32];
        if (q0 <= quad) {              // warp-uniform: columns beyond the warp's rows are 0
          tc::tmem_ld32(qk_addr + 32 * q0, x);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = 32 * q0 + e;
            x[e] = (j <= r && r < Lv) ? x[e] * pw[r - j] : 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = 0.f;
        }
        // columns 32*q0 .. +31 -> atom q0/2, chunks (q0%2)*4 .. +3
        uint8_t* row = sP + (q0 >> 1) * 16384 + r * 128;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 u;
          __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            h2[e] = __floats2bfloat162_rn(x[ch * 8 + 2 * e], x[ch * 8 + 2 * e + 1]);
          const int chunk = (q0 & 1) * 4 + ch;
          *reinterpret_cast<uint4*>(row + ((chunk ^ (r & 7)) << 4)) = u;
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(qk_empty);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ state + epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;     // key-dim row of S; token row of O
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const long long sbase = (((long long)b * H + h) * D + r) * D + col0;
    float S[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) S[e] = state_in ? state_in[sbase + e] : 0.f;
    sw64_store_row(smem + L::kS, r, S);               // S_{-1} -> buffer 0
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(s_full);
    bool ok = true;
    for (int c = 0; ok && c < n_tiles; ++c) {
      const int Lv = min(kLinTile, N - c * kLinTile);
      // S_c = lam^L S_{c-1} + dS
      ok = __all_sync(0xffffffffu, tc::mbar_wait(ds_full, c & 1));
      if (!ok) break;
      tc::tc_fence_after();
      float ds[32];
      tc::tmem_ld32(lane_base + L::kColDS, ds);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(ds_empty);
      const float lamL = pw[Lv];
#pragma unroll
      for (int e = 0; e < 32; ++e) S[e] = fmaf(lamL, S[e], ds[e]);
      const int buf = (c + 1) & 1;
      if (c >= 1) ok = __all_sync(0xffffffffu, tc::mbar_wait(s_empty + buf, ((((c + 1) >> 1) - 1) & 1)));
      if (!ok) break;
      sw64_store_row(smem + L::kS + buf * 8192, r, S);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_full + buf);
      // epilogue of tile c: row r = token
      const long long off = (((long long)b * N + (long long)c * kLinTile + r) * H + h) * D + col0;
      float gv[32];
      if (r < Lv) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) load8(gate + off + e, gv + e);
      }
      ok = __all_sync(0xffffffffu, tc::mbar_wait(o_full, c & 1));
      if (!ok) break;
      tc::tc_fence_after();
      float oi[32], oe[32];
      tc::tmem_ld32(lane_base + L::kColOi, oi);
      tc::tmem_ld32(lane_base + L::kColOe, oe);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(o_empty);
      if (r < Lv) {
        const float fi = pw[r + 1];
#pragma unroll
        for (int e = 0; e < 32; ++e) gv[e] = sigmoidf_(gv[e]) * scale * fmaf(fi, oe[e], oi[e]);
#pragma unroll
        for (int e = 0; e < 32; e += 8) store8(out + off + e, gv + e);
      }
    }
    if (ok && state_out) {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(state_out + sbase + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace sala
