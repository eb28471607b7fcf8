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
// elected thread), warps 4-7 build V' and the diagonal 32-column chunks of
// P, warps 2-3 (also the TMEM owner) and warps 6-7 the off-diagonal chunks,
// warps 8-11 update the state and run the gated epilogue.  The QK, dS and O
// accumulators are double-buffered in TMEM so the tensor work of tile c+1
// overlaps the element-wise work of tile c.  Waits are bounded.
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
  // ld_full[S], ld_empty[S], qk_full[2], qk_empty[2], ds_full[2], ds_empty[2],
  // o_full[2], o_empty[2], s_full[2], s_empty[2], vp_full, vp_empty, p_full, p_empty, fin
  static constexpr int kNumBars = 2 * kLinStages + 12 + 5;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kTmemCols = 512;
  // TMEM columns of buffer x in {0, 1}
  static constexpr int col_qk(int x) { return 128 * x; }
  static constexpr int col_ds(int x) { return 256 + 32 * x; }
  static constexpr int col_oi(int x) { return 320 + 32 * x; }
  static constexpr int col_oe(int x) { return 384 + 32 * x; }
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
  uint64_t* qk_full = bars + 2 * kLinStages;   // [2]
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
                       v = stage_addr(c) + L::kV;
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
        if (c + 1 < n_tiles && !(ok = issue_qk(c + 1))) break;
        // O_intra = P V
        if (!(ok = tc::mbar_wait(p_full, c & 1))) break;
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + L::col_oi(x), tc::smem_desc_sw128(base + L::kP + off, 16, 1024),
                          tc::smem_desc_sw64(v + kk * 1024, 8192, 512), id_o, kk > 0);
        }
        tc::mma_commit(p_empty);
        tc::mma_commit(o_full + x);
        tc::mma_commit(ld_empty + st);
      }
      tc::mma_commit(fin);
      tc::mbar_wait(fin, 0);
    }
  }

  if ((warp >= 2 && warp < 8) && warp != 1) {
    // ------------------------------------------------------------ V' (warps 4-7) and P
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    int clo, chi;
    p_chunks(warp, clo, chi);
    uint8_t* sP = smem + L::kP;
    uint8_t* sVp = smem + L::kVp;
    bool ok = true;
    for (int c = 0; ok && c < n_tiles; ++c) {
      const int st = c % kLinStages, x = c & 1;
      if (warp >= 4) {
        // V'_r = lam^(L-1-r) v_r (0 past the end of the sequence)
        const int Lv = min(kLinTile, N - c * kLinTile);
        ok = __all_sync(0xffffffffu, tc::mbar_wait(ld_full + st, (c / kLinStages) & 1));
        if (ok && c > 0) ok = __all_sync(0xffffffffu, tc::mbar_wait(vp_empty, (c - 1) & 1));
        if (!ok) break;
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
      // P_rj = QK_rj lam^(r-j) for j <= r (rows past the end are never stored)
      ok = __all_sync(0xffffffffu, tc::mbar_wait(qk_full + x, (c >> 1) & 1));
      if (ok && c > 0) ok = __all_sync(0xffffffffu, tc::mbar_wait(p_empty, (c - 1) & 1));
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t qk_addr = tmem + ((uint32_t)(quad * 32) << 16) + L::col_qk(x);
      for (int q0 = clo; q0 < chi; ++q0) {
        float xv[32];
        tc::tmem_ld32(qk_addr + 32 * q0, xv);
        tc::tmem_wait_ld();
        if (q0 == quad) {
          // diagonal chunk: column e of the chunk is visible iff e <= lane
#pragma unroll
          for (int e = 0; e < 32; ++e) xv[e] = e <= lane ? xv[e] * pw[lane - e] : 0.f;
        } else {
          // below the diagonal: decay lam^(r - 32 q0 - e), applied from e = 31 down
          float dcy = pw[r - 32 * q0 - 31];
#pragma unroll
          for (int e = 31; e >= 0; --e) {
            xv[e] *= dcy;
            dcy *= lam;
          }
        }
        uint8_t* row = sP + (q0 >> 1) * 16384 + r * 128;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 u;
          __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            h2[e] = __floats2bfloat162_rn(xv[ch * 8 + 2 * e], xv[ch * 8 + 2 * e + 1]);
          const int chunk = (q0 & 1) * 4 + ch;
          *reinterpret_cast<uint4*>(row + ((chunk ^ (r & 7)) << 4)) = u;
        }
      }
      // chunks above the diagonal are zero: written once per buffer by the
      // diagonal owner (warps 4-7) on the first tile, never touched again
      if (c == 0 && warp >= 4) {
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int q0 = quad + 1; q0 < 4; ++q0) {
          uint8_t* row = sP + (q0 >> 1) * 16384 + r * 128;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int chunk = (q0 & 1) * 4 + ch;
            *reinterpret_cast<uint4*>(row + ((chunk ^ (r & 7)) << 4)) = z;
          }
        }
      }
      tc::tc_fence_before();
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(qk_empty + x);
        tc::mbar_arrive(p_full);
      }
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
    // gate rows are fetched one tile ahead into registers
    float gv[32];
    auto fetch_gate = [&](int c) {
      const long long off = (((long long)b * N + (long long)c * kLinTile + r) * H + h) * D + col0;
      if (c < n_tiles && c * kLinTile + r < N) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) load8(gate + off + e, gv + e);
      }
    };
    fetch_gate(0);
    bool ok = true;
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
      // epilogue of tile c: row r = token
      ok = __all_sync(0xffffffffu, tc::mbar_wait(o_full + x, (c >> 1) & 1));
      if (!ok) break;
      tc::tc_fence_after();
      float oi[32], oe[32];
      tc::tmem_ld32(lane_base + L::col_oi(x), oi);
      tc::tmem_ld32(lane_base + L::col_oe(x), oe);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(o_empty + x);
      if (r < Lv) {
        const long long off = (((long long)b * N + (long long)c * kLinTile + r) * H + h) * D + col0;
        const float fi = pw[r + 1] * scale;
        float res[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) res[e] = sigmoidf_(gv[e]) * fmaf(fi, oe[e], scale * oi[e]);
#pragma unroll
        for (int e = 0; e < 32; e += 8) store8(out + off + e, res + e);
      }
      fetch_gate(c + 1);
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
