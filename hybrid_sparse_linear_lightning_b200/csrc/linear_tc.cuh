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
// Warp roles (512 threads): warp 0 TMA producer, warp 1 MMA issuer (one
// elected thread), warps 2-7 build P (balanced 32-column chunks; warp 2 also
// owns TMEM) and write it to TMEM as the A operand of P V, warps 8-11 update
// the state and build V' for the next tile (the short chain that feeds the
// next dS and Q S products), warps 12-15 run the gated epilogue.  The QK, dS
// and O accumulators are double-buffered in TMEM so the tensor work of tile
// c+1 overlaps the element-wise work of tile c.  Waits are bounded.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sala {

constexpr int kLinTcThreads = 512;
constexpr int kLinTile = 128;
constexpr int kLinCols = 32;
constexpr int kLinStages = 2;

struct LinTcLayout {
  // per stage: Q^ tile and K^ tile (2 atoms x 16 KB each); V slices in their own ring
  static constexpr int kQ = 0;
  static constexpr int kK = 32768;
  static constexpr int kStage = 65536;
  static constexpr int kV = kLinStages * kStage;         // [2] x V slice, 128 rows x 64 B (SW64)
  static constexpr int kVp = kV + 2 * 8192;              // V': 128 rows x 64 B
  static constexpr int kS = kVp + 8192;                  // S bf16: 2 buffers x 128 rows x 64 B
  static constexpr int kPw = kS + 2 * 8192;              // lam^m, m = 0..128
  static constexpr int kBar = kPw + 4 * 132;
  // ld_full[S], ld_empty[S], v_full[2], v_empty[2], qk_full[2], qk_empty[2], ds_full[2],
  // ds_empty[2], o_full[2], o_empty[2], s_full[2], s_empty[2], vp_full, vp_empty, p_full,
  // p_empty, fin
  static constexpr int kNumBars = 2 * kLinStages + 4 + 12 + 5;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kTmemCols = 512;
  // TMEM columns of buffer x in {0, 1}
  static constexpr int col_qk(int x) { return 128 * x; }
  static constexpr int col_ds(int x) { return 256 + 32 * x; }
  static constexpr int col_oi(int x) { return 320 + 32 * x; }
  static constexpr int col_oe(int x) { return 384 + 32 * x; }
  static constexpr int kColP = 448;     // P (bf16 pairs): 128 keys in 64 columns, A of P V
};

// Warps that build the P chunks of each tile: warp w (TMEM lane quadrant
// w & 3) handles 32-column chunks [kPChunkLo[w], kPChunkHi[w]) of its rows.
// Row quadrant q has chunks 0..q below or on the diagonal (chunk q).
__device__ __forceinline__ void p_chunks(int warp, int& lo, int& hi) {
  switch (warp) {
    case 2: lo = 0; hi = 1; break;    // quadrant 2: chunk 0
    case 3: lo = 0; hi = 2; break;    // quadrant 3: chunks 0, 1
    case 4: lo = 0; hi = 1; break;    // quadrant 0: chunk 0 (diagonal)
    case 5: lo = 0; hi = 2; break;    // quadrant 1: chunks 0, 1 (1 diagonal)
    case 6: lo = 1; hi = 3; break;    // quadrant 2: chunks 1, 2 (2 diagonal)
    case 7: lo = 2; hi = 4; break;    // quadrant 3: chunks 2, 3 (3 diagonal)
    default: lo = hi = 0;
  }
}
constexpr int kPWarps = 6;

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
  extern __shared__ __align__(1024) uint8_t smem_tc[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_tc) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* ld_full = bars;
  uint64_t* ld_empty = bars + kLinStages;
  uint64_t* v_full = bars + 2 * kLinStages;    // [2]
  uint64_t* v_empty = v_full + 2;              // [2]
  uint64_t* qk_full = v_full + 4;              // [2]
  uint64_t* qk_empty = qk_full + 2;            // [2]
  uint64_t* ds_full = qk_full + 4;             // [2]
  uint64_t* ds_empty = qk_full + 6;            // [2]
  uint64_t* o_full = qk_full + 8;              // [2]
  uint64_t* o_empty = qk_full + 10;            // [2]
  uint64_t* s_full = qk_full + 12;             // [2]
  uint64_t* s_empty = qk_full + 14;            // [2]
  uint64_t* vp_full = qk_full + 16;
  uint64_t* vp_empty = qk_full + 17;
  uint64_t* p_full = qk_full + 18;
  uint64_t* p_empty = qk_full + 19;
  uint64_t* fin = qk_full + 20;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  float* pw = reinterpret_cast<float*>(smem + L::kPw);

  const int slice = blockIdx.x % NS;
  const int h = (blockIdx.x / NS) % H;
  const int b = blockIdx.x / (NS * H);
  const int col0 = slice * kLinCols;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + kLinTile - 1) / kLinTile;
  const float lam = lambda[h];

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLinStages; ++s) {
      tc::mbar_init(ld_full + s, 1);
      tc::mbar_init(ld_empty + s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(v_full + x, 1);
      tc::mbar_init(v_empty + x, 1);
      tc::mbar_init(qk_full + x, 1);
      tc::mbar_init(qk_empty + x, kPWarps);
      tc::mbar_init(ds_full + x, 1);
      tc::mbar_init(ds_empty + x, 4);
      tc::mbar_init(o_full + x, 1);
      tc::mbar_init(o_empty + x, 4);
      tc::mbar_init(s_full + x, 4);
      tc::mbar_init(s_empty + x, 1);
    }
    tc::mbar_init(vp_full, 4);
    tc::mbar_init(vp_empty, 1);
    tc::mbar_init(p_full, kPWarps);
    tc::mbar_init(p_empty, 1);
    tc::mbar_init(fin, 1);
    tc::fence_barrier_init();
  }
  if (threadIdx.x <= kLinTile) pw[threadIdx.x] = (float)pow((double)lam, (double)threadIdx.x);
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
        const int vs = c & 1;
        if (c >= 2 && !tc::mbar_wait(v_empty + vs, ((c >> 1) - 1) & 1)) break;
        tc::mbar_expect_tx(v_full + vs, 8192);
        tc::tma_load_2d(smem + L::kV + vs * 8192, &vmap, v_full + vs, h * D + col0, row0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      constexpr uint32_t id_qk = tc::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_ds = tc::idesc_bf16_f32(128, kLinCols, true, true);
      constexpr uint32_t id_o = tc::idesc_bf16_f32(128, kLinCols, false, true);
      const uint32_t base = tc::smem_u32(smem);
      auto stage_addr = [&](int c) { return base + (c % kLinStages) * L::kStage; };
      // QK(c) = Q^ K^T into buffer c & 1 (A, B K-major)
      auto issue_qk = [&](int c) -> bool {
        const int st = c % kLinStages, x = c & 1;
        if (!tc::mbar_wait(ld_full + st, (c / kLinStages) & 1)) return false;
        if (c >= 2 && !tc::mbar_wait(qk_empty + x, ((c >> 1) - 1) & 1)) return false;
        tc::tc_fence_after();
        const uint32_t q = stage_addr(c) + L::kQ, k = stage_addr(c) + L::kK;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + L::col_qk(x), tc::smem_desc_sw128(q + off, 16, 1024),
                          tc::smem_desc_sw128(k + off, 16, 1024), id_qk, kk > 0);
        }
        tc::mma_commit(qk_full + x);
        return true;
      };
      // Order per tile: dS(c), O_inter(c), QK(c+1), PV(c): the QK of the next
      // tile runs while P(c) is being built.
      bool ok = n_tiles > 0 && issue_qk(0);
      for (int c = 0; ok && c < n_tiles; ++c) {
        const int st = c % kLinStages, x = c & 1;
        const uint32_t prev = ((c >> 1) - 1) & 1;     // parity of this buffer's previous use
        const uint32_t q = stage_addr(c) + L::kQ, k = stage_addr(c) + L::kK,
                       v = base + L::kV + x * 8192;
        // dS = K^T V'  (A = K^ read MN-major, B = V' MN-major)
        if (!(ok = tc::mbar_wait(vp_full, c & 1))) break;
        if (c >= 2 && !(ok = tc::mbar_wait(ds_empty + x, prev))) break;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16_ss(tmem + L::col_ds(x), tc::smem_desc_sw128(k + kk * 2048, 16384, 1024),
                          tc::smem_desc_sw64(base + L::kVp + kk * 1024, 8192, 512), id_ds, kk > 0);
        tc::mma_commit(ds_full + x);
        tc::mma_commit(vp_empty);
        // O_inter = Q^ S_prev  (B = S bf16 MN-major); S_{c-1} sits in buffer c & 1
        if (!(ok = tc::mbar_wait(s_full + x, (c >> 1) & 1))) break;
        if (c >= 2 && !(ok = tc::mbar_wait(o_empty + x, prev))) break;
        tc::tc_fence_after();
        const uint32_t sb = base + L::kS + x * 8192;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + L::col_oe(x), tc::smem_desc_sw128(q + off, 16, 1024),
                          tc::smem_desc_sw64(sb + kk * 1024, 8192, 512), id_o, kk > 0);
        }
        tc::mma_commit(s_empty + x);
        tc::mma_commit(ld_empty + st);        // Q^ / K^ of tile c are no longer read
        if (c + 1 < n_tiles && !(ok = issue_qk(c + 1))) break;
        // O_intra = P V  (P from TMEM)
        if (!(ok = tc::mbar_wait(p_full, c & 1))) break;
        if (!(ok = tc::mbar_wait(v_full + x, (c >> 1) & 1))) break;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16_ts(tmem + L::col_oi(x), tmem + L::kColP + kk * 8,
                          tc::smem_desc_sw64(v + kk * 1024, 8192, 512), id_o, kk > 0);
        tc::mma_commit(p_empty);
        tc::mma_commit(o_full + x);
        tc::mma_commit(v_empty + x);
      }
      tc::mma_commit(fin);
      tc::mbar_wait(fin, 0);
    }
  }

  if (warp >= 2 && warp < 8) {
    // ------------------------------------------------------------ P (warps 2-7)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    int clo, chi;
    p_chunks(warp, clo, chi);
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    bool ok = true;
    for (int c = 0; ok && c < n_tiles; ++c) {
      const int x = c & 1;
      // P_rj = QK_rj lam^(r-j) for j <= r (rows past the end are never stored)
      ok = __all_sync(0xffffffffu, tc::mbar_wait(qk_full + x, (c >> 1) & 1));
      if (ok && c > 0) ok = __all_sync(0xffffffffu, tc::mbar_wait(p_empty, (c - 1) & 1));
      if (!ok) break;
      tc::tc_fence_after();
      // both chunk loads are in flight before the single wait
      float xv[2][32];
      tc::tmem_ld32(lane_base + L::col_qk(x) + 32 * clo, xv[0]);
      if (chi - clo > 1) tc::tmem_ld32(lane_base + L::col_qk(x) + 32 * (clo + 1), xv[1]);
      tc::tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int q0 = clo + u;
        if (q0 >= chi) break;
        if (q0 == quad) {
          // diagonal chunk: column e of the chunk is visible iff e <= lane
#pragma unroll
          for (int e = 0; e < 32; ++e) xv[u][e] = e <= lane ? xv[u][e] * pw[lane - e] : 0.f;
        } else {
          // below the diagonal: decay lam^(r - 32 q0 - e), applied from e = 31 down
          float dcy = pw[r - 32 * q0 - 31];
#pragma unroll
          for (int e = 31; e >= 0; --e) {
            xv[u][e] *= dcy;
            dcy *= lam;
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(xv[u][2 * e], xv[u][2 * e + 1]);
          pk[e] = *reinterpret_cast<uint32_t*>(&h2);
        }
        tc::tmem_st16_u(lane_base + L::kColP + 16 * q0, pk);
      }
      if (c == 0 && warp >= 4) {          // chunks above the diagonal stay zero
        uint32_t z[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = 0u;
        for (int q0 = quad + 1; q0 < 4; ++q0) tc::tmem_st16_u(lane_base + L::kColP + 16 * q0, z);
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(qk_empty + x);
        tc::mbar_arrive(p_full);
      }
    }
  } else if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------ state and V'
    const int quad = warp & 3;
    const int r = quad * 32 + lane;     // key-dim row of S; token row of V'
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const long long sbase = (((long long)b * H + h) * D + r) * D + col0;
    float S[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) S[e] = state_in ? state_in[sbase + e] : 0.f;
    sw64_store_row(smem + L::kS, r, S);               // S_{-1} -> buffer 0
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(s_full);
    // V'_r = lam^(L-1-r) v_r of tile c (0 past the end of the sequence)
    auto make_vp = [&](int c) -> bool {
      const int Lv = min(kLinTile, N - c * kLinTile);
      bool okv = __all_sync(0xffffffffu, tc::mbar_wait(v_full + (c & 1), (c >> 1) & 1));
      if (okv && c > 0) okv = __all_sync(0xffffffffu, tc::mbar_wait(vp_empty, (c - 1) & 1));
      if (!okv) return false;
      float vv[32];
      sw64_load_row(smem + L::kV + (c & 1) * 8192, r, vv);
      const float f = r < Lv ? pw[Lv - 1 - r] : 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) vv[e] *= f;
      sw64_store_row(smem + L::kVp, r, vv);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(vp_full);
      return true;
    };
    bool ok = n_tiles > 0 && make_vp(0);
    for (int c = 0; ok && c < n_tiles; ++c) {
      const int Lv = min(kLinTile, N - c * kLinTile), x = c & 1;
      // S_c = lam^L S_{c-1} + dS
      ok = __all_sync(0xffffffffu, tc::mbar_wait(ds_full + x, (c >> 1) & 1));
      if (!ok) break;
      tc::tc_fence_after();
      float ds[32];
      tc::tmem_ld32(lane_base + L::col_ds(x), ds);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(ds_empty + x);
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
      if (c + 1 < n_tiles && !(ok = make_vp(c + 1))) break;
    }
    if (ok && state_out) {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(state_out + sbase + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ gated epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;     // token row of O
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    // gate rows are fetched one tile ahead as raw 16-byte words (converted at
    // use, so the load latency overlaps the previous tile)
    constexpr int kGW = 32 * (int)sizeof(T) / 16;
    uint4 graw[kGW];
    auto fetch_gate = [&](int c) {
      const long long off = (((long long)b * N + (long long)c * kLinTile + r) * H + h) * D + col0;
      if (c < n_tiles && c * kLinTile + r < N) {
        const uint4* src = reinterpret_cast<const uint4*>(gate + off);
#pragma unroll
        for (int e = 0; e < kGW; ++e) graw[e] = src[e];
      }
    };
    fetch_gate(0);
    const float fs = scale;
    for (int c = 0; c < n_tiles; ++c) {
      const int Lv = min(kLinTile, N - c * kLinTile), x = c & 1;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(o_full + x, (c >> 1) & 1))) break;
      tc::tc_fence_after();
      const long long off = (((long long)b * N + (long long)c * kLinTile + r) * H + h) * D + col0;
      const float fi = pw[r + 1] * fs;
      float gv[32];
#pragma unroll
      for (int e = 0; e < 32; e += 8)
        load8(reinterpret_cast<const T*>(graw) + e, gv + e);
      float oi[32], oe[32];
      tc::tmem_ld32(lane_base + L::col_oi(x), oi);
      tc::tmem_ld32(lane_base + L::col_oe(x), oe);
      tc::tmem_wait_ld();
      if (r < Lv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) oi[e] = sigmoidf_(gv[e]) * fmaf(fi, oe[e], fs * oi[e]);
#pragma unroll
        for (int e = 0; e < 32; e += 8) store8(out + off + e, oi + e);
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(o_empty + x);
      fetch_gate(c + 1);
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
