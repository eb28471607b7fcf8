// Gathered block-sparse attention on the 5th-generation tensor cores.
//
// InfLLM-V2-style sparse layer (acgfav.com "SALA 混合架构": each query
// attends to a small set of selected key blocks), NoPE, output gate after the
// block (MiniCPM-SALA paper, summary).  For query block i of kv head g, the
// 64 tokens of every q head of the group share one list of selected key
// blocks, so a CTA takes FOUR q heads of the group (two 128-row tiles: 2 heads
// x 64 tokens each) and streams each selected K/V block through shared memory
// once for all 256 query rows (GQA sharing: one K/V fetch per CTA).
//
// Per selected block j (64 keys):  S_t = Q_t K_j^T  (tcgen05, M=128 N=64,
// fp32 in TMEM, two buffers per tile);  softmax warps read S_t one row per
// thread, apply the causal mask on the diagonal block, exponentiate against a
// running max and write P_t (bf16 pairs) over the S_t buffer they read;
// O_t += P_t V_j  (tcgen05 with A read from TMEM, M=128 N=d, fp32 in TMEM).
// S_t of block j+1 is issued before P_t V_j, into the other buffer, so the
// softmax of block j+1 starts as soon as P_t of block j is written.  Exact softmax: the running max is raised (and O, l rescaled) only
// when a row's max grows by more than 2^8, so values stay bounded; the final
// division by l makes the result independent of that choice up to rounding.
// Epilogue: out = sigmoid(gate) * O / l.
//
// Warp roles (384 threads): warp 0 issues TMA loads, warp 1 issues MMAs (one
// elected thread), warp 2 owns the TMEM allocation, warps 4-7 / 8-11 are the
// softmax + epilogue warpgroups of tile 0 / tile 1.  Every mbarrier wait is
// bounded; a wait that runs out sets the device status word and the CTA
// winds down without touching further data.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sala {

constexpr int kSpTcThreads = 384;
constexpr int kSpTcStages = 4;
constexpr int kSpTcHeadsPerCta = 4;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr int kSpPolyPairsPer8 = 2;         // exponential pairs evaluated on the FMA pipe

template <int D>
struct SpTcLayout {
  static constexpr int kAtoms = D / 64;                 // 128-byte column atoms of a row
  static constexpr int kQTile = 128 * D * 2;            // one 128-row Q tile
  static constexpr int kKV = 64 * D * 2;                // one 64-row K or V block
  static constexpr int kQ = 0;
  static constexpr int kKVBase = kQ + 2 * kQTile;
  static constexpr int kBar = kKVBase + kSpTcStages * 2 * kKV;
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[tile][buf], p_full[tile][buf],
  // o_done[tile][block parity], fin
  static constexpr int kNumBars = 1 + 2 * kSpTcStages + 4 + 4 + 4 + 1;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kSel = kMisc + 16;               // int sel[width]
  static constexpr int kBytes(int width) { return kSel + 4 * width; }
  static constexpr int kTmemCols = 512;
  // TMEM columns: S of tile t, buffer x at 64 (2 t + x) (64 fp32; P of the
  // same block overwrites its first 32 columns as bf16 pairs), O_0, O_1 (D each)
  static constexpr int col_s(int t, int x) { return 64 * (2 * t + x); }
  static constexpr int kColO0 = 256, kColO1 = 256 + D;
};

template <typename T, int D>
__global__ void __launch_bounds__(kSpTcThreads, 1)
sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap,
                      const int32_t* __restrict__ idx, const T* __restrict__ gate,
                      T* __restrict__ out, int N, int Hq, int Hkv, int width, float sl2) {
  using L = SpTcLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_tc[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_tc) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kSpTcStages;
  uint64_t* s_full = kv_empty + kSpTcStages;   // [tile * 2 + buffer]
  // P of block j of tile t is published on p_full[2 t + (j & 1)]. The softmax
  // of a tile can finish blocks j and j+1 while the MMA issuer still waits for
  // the other tile's block j (S of block j+1 is issued before that wait), but
  // not block j+2 (its S is issued after it): with one barrier per buffer
  // parity each barrier is at most one phase ahead of its waiter, where a
  // single barrier per tile could be two phases ahead and its parity wait
  // would never return
  uint64_t* p_full = s_full + 4;
  // P V of block j of tile t completes o_done[2 t + (j & 1)]: every wait on it
  // (for block j-1, by the softmax before a rescale and before the epilogue)
  // comes after P V of block j-3 has completed, so a parity wait is never
  // more than one phase behind
  uint64_t* o_done = p_full + 4;
  uint64_t* fin = o_done + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  int* n_sel_slot = reinterpret_cast<int*>(smem + L::kMisc + 4);
  int* sel = reinterpret_cast<int*>(smem + L::kSel);

  const int G = Hq / Hkv;
  const int nq = G / kSpTcHeadsPerCta;
  const int nb = N / 64;
  const int hq = blockIdx.x % nq;
  const int i = (blockIdx.x / nq) % nb;
  const int g = (blockIdx.x / (nq * nb)) % Hkv;
  const int b = blockIdx.x / (nq * nb * Hkv);
  const int hbase = g * G + hq * kSpTcHeadsPerCta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- setup: barriers, the Q tiles (loaded at once: they do not depend on
  // the block list), TMEM, the block list
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sKV = smem + L::kKVBase;
  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    for (int s = 0; s < kSpTcStages; ++s) {
      tc::mbar_init(kv_full + s, 1);
      tc::mbar_init(kv_empty + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      tc::mbar_init(s_full + 2 * t, 1);
      tc::mbar_init(s_full + 2 * t + 1, 1);
      tc::mbar_init(p_full + 2 * t, 4);
      tc::mbar_init(p_full + 2 * t + 1, 4);
      tc::mbar_init(o_done + 2 * t, 1);
      tc::mbar_init(o_done + 2 * t + 1, 1);
    }
    tc::mbar_init(fin, 1);
    tc::fence_barrier_init();
    tc::tma_prefetch(&qmap);
    tc::tma_prefetch(&kmap);
    tc::tma_prefetch(&vmap);
    tc::mbar_expect_tx(q_full, 2 * L::kQTile);
    const int row0 = b * N + i * 64;
    for (int t = 0; t < 2; ++t)
      for (int hl = 0; hl < 2; ++hl)
        for (int a = 0; a < L::kAtoms; ++a)
          tc::tma_load_2d(sQ + t * L::kQTile + a * (128 * 128) + hl * (64 * 128), &qmap, q_full,
                          (hbase + 2 * t + hl) * D + 64 * a, row0);
  }
  if (warp == 0) {
    // valid prefix of the ascending index row (entries in [0, i]), read by
    // the whole warp 32 entries at a time: it ends at the first -1 or at the
    // first entry out of range or out of order (which also sets the bounds bit)
    const int32_t* row = idx + (((long long)b * Hkv + g) * nb + i) * width;
    int n = 0, prev = -1;
    for (int e0 = 0; e0 < width; e0 += 32) {
      const int e = e0 + lane;
      const int j = e < width ? __ldg(row + e) : -1;
      int jp = __shfl_up_sync(0xffffffffu, j, 1);
      if (lane == 0) jp = prev;
      const bool good = j >= 0 && j <= i && j > jp;
      const unsigned gm = __ballot_sync(0xffffffffu, good);
      const int run = gm == 0xffffffffu ? 32 : __ffs(~gm) - 1;   // leading good lanes
      if (lane < run) sel[n + lane] = j;
      const int jstop = __shfl_sync(0xffffffffu, j, run & 31);
      if (run < 32 && jstop >= 0 && lane == 0) set_status(kStatusBounds);
      n += run;
      prev = __shfl_sync(0xffffffffu, j, (run + 31) & 31);
      if (run < 32) break;
    }
    // a valid row lists at least the query's own block; an empty row gets a
    // zero output and the bounds bit
    if (lane == 0) {
      if (n == 0) set_status(kStatusBounds);
      *n_sel_slot = n;
    }
  }
  if (warp == 2) {
    tc::tmem_alloc(tmem_slot, L::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_sel = *n_sel_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (tc::elect_one() && n_sel == 0) {
      // nothing reads the Q tiles: let their load land before the CTA ends
      tc::mbar_wait(q_full, 0);
    }
    if (tc::elect_one() && n_sel > 0) {
      for (int j = 0; j < n_sel; ++j) {
        const int st = j % kSpTcStages, use = j / kSpTcStages;
        if (use > 0 && !tc::mbar_wait(kv_empty + st, (use - 1) & 1)) break;
        tc::mbar_expect_tx(kv_full + st, 2 * L::kKV);
        uint8_t* k_dst = sKV + st * 2 * L::kKV;
        uint8_t* v_dst = k_dst + L::kKV;
        const int krow = b * N + sel[j] * 64;
        for (int a = 0; a < L::kAtoms; ++a) {
          tc::tma_load_2d(k_dst + a * (64 * 128), &kmap, kv_full + st, g * D + 64 * a, krow);
          tc::tma_load_2d(v_dst + a * (64 * 128), &vmap, kv_full + st, g * D + 64 * a, krow);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one() && n_sel > 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = tc::smem_u32(sQ), kv_addr = tc::smem_u32(sKV);
      auto issue_s = [&](int t, int j) {
        const uint32_t k_addr = kv_addr + (j % kSpTcStages) * 2 * L::kKV;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;   // 16 elements = 32 B inside the atom
          const uint64_t ad = tc::smem_desc_sw128(q_addr + t * L::kQTile + (kk >> 2) * (128 * 128) + off, 16, 1024);
          const uint64_t bd = tc::smem_desc_sw128(k_addr + (kk >> 2) * (64 * 128) + off, 16, 1024);
          tc::mma_bf16_ss(tmem + L::col_s(t, j & 1), ad, bd, idesc_s, kk > 0);
        }
        tc::mma_commit(s_full + 2 * t + (j & 1));
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t v_addr = kv_addr + (j % kSpTcStages) * 2 * L::kKV + L::kKV;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = tc::smem_desc_sw128(v_addr + kk * 2048, 64 * 128, 1024);
          tc::mma_bf16_ts(tmem + (t ? L::kColO1 : L::kColO0), tmem + L::col_s(t, j & 1) + kk * 8,
                          bd, idesc_o, (j > 0 || kk > 0));
        }
        tc::mma_commit(o_done + 2 * t + (j & 1));
      };
      // Issue order: S_0(0) S_1(0) | S_0(j+1) S_1(j+1) PV_0(j) PV_1(j) | ...  S of
      // the next block goes into the other buffer of its tile, so it is
      // ready when the softmax of block j finishes.
      bool ok = tc::mbar_wait(q_full, 0) && tc::mbar_wait(kv_full, 0);
      if (ok) {
        tc::tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
      }
      for (int j = 0; ok && j < n_sel; ++j) {
        if (j + 1 < n_sel) {
          if (!(ok = tc::mbar_wait(kv_full + (j + 1) % kSpTcStages, ((j + 1) / kSpTcStages) & 1))) break;
          // buffer (j+1) & 1 last held P of block j-1, read by P V of block
          // j-1; that MMA was issued before this one by this thread, and
          // tcgen05.mma operations from one thread execute in issue order, so
          // S of block j+1 needs no wait for it
          tc::tc_fence_after();
          for (int t = 0; t < 2; ++t) issue_s(t, j + 1);
        }
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = tc::mbar_wait(p_full + 2 * t + (j & 1), (j >> 1) & 1))) break;
          tc::tc_fence_after();
          issue_pv(t, j);
        }
        if (ok) tc::mma_commit(kv_empty + (j % kSpTcStages));
      }
      // drain: every MMA issued above has completed once `fin` fires
      tc::mma_commit(fin);
      tc::mbar_wait(fin, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;            // tile
    const int quad = warp & 3;                // TMEM lane quadrant
    const int r = quad * 32 + lane;           // row in the tile
    const int tok = r & 63;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t o_addr = lane_base + (t ? L::kColO1 : L::kColO0);
    const float2 sl2v = make_float2(sl2, sl2);
    float m = -INFINITY, l = 0.f;
    bool ok = n_sel > 0;
    for (int j = 0; ok && j < n_sel; ++j) {
      ok = __all_sync(0xffffffffu, tc::mbar_wait(s_full + 2 * t + (j & 1), (j >> 1) & 1));
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t s_addr = lane_base + L::col_s(t, j & 1);   // P of block j goes here too
      float x[64];
      tc::tmem_ld32(s_addr, x);
      tc::tmem_ld32(s_addr + 32, x + 32);
      tc::tmem_wait_ld();
      // causal mask on the diagonal block only (warp-uniform branch)
      if (sel[j] == i) {
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = c > tok ? -INFINITY : x[c];
      }
      // row max as a tree over 8 independent partial maxima, scaled once (sl2 > 0)
      float mp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mp[k] = x[k];
#pragma unroll
      for (int c = 8; c < 64; ++c) mp[c & 7] = fmaxf(mp[c & 7], x[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7]))) * sl2;
      if (j == 0) m = mx;
      if (j > 0) {
        // O is rescaled (after P V of block j-1 has landed) only when a row's
        // max grew by more than the threshold
        if (__any_sync(0xffffffffu, mx > m + kRescaleThreshold)) {
          ok = __all_sync(0xffffffffu,
                          tc::mbar_wait(o_done + 2 * t + ((j - 1) & 1), ((j - 1) >> 1) & 1));
          if (!ok) break;
          const float mnew = fmaxf(m, mx);
          const float f = exp2f(m - mnew);
          m = mnew;
          l *= f;
          tc::tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tc::tmem_ld32(o_addr + c0, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= f;
            tc::tmem_st32(o_addr + c0, o);
          }
          tc::tmem_wait_st();
        }
      }
      // P = 2^(x sl2 - m) packed as bf16 pairs into TMEM; row sum over 4 pair-accumulators
      const float2 negm = make_float2(-m, -m);
      float2 acc4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 tt = __ffma2_rn(make_float2(x[2 * e], x[2 * e + 1]), sl2v, negm);
        // kSpPolyPairsPer8 of every 8 pairs on the FMA pipe, the rest on the
        // special-function unit
        const float2 pv = (e & 7) < kSpPolyPairsPer8
                              ? tc::exp2_fma2(tt)
                              : make_float2(tc::ex2_approx(tt.x), tc::ex2_approx(tt.y));
        acc4[e & 3] = __fadd2_rn(acc4[e & 3], pv);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(pv.x, pv.y);
        pk[e] = *reinterpret_cast<uint32_t*>(&h2);
      }
      tc::tmem_st32_u(s_addr, pk);
      const float2 s01 = __fadd2_rn(__fadd2_rn(acc4[0], acc4[1]), __fadd2_rn(acc4[2], acc4[3]));
      l += s01.x + s01.y;
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full + 2 * t + (j & 1));
    }
    // epilogue: out = sigmoid(gate) * O / l
    if (ok)
      ok = __all_sync(0xffffffffu,
                      tc::mbar_wait(o_done + 2 * t + ((n_sel - 1) & 1), ((n_sel - 1) >> 1) & 1));
    if (n_sel == 0) {
      const int head = hbase + 2 * t + (r >> 6);
      const long long off = (((long long)b * N + (long long)i * 64 + tok) * Hq + head) * D;
      float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int c = 0; c < D; c += 8) store8(out + off + c, z);
    } else if (ok) {
      tc::tc_fence_after();
      const int head = hbase + 2 * t + (r >> 6);
      const long long off = (((long long)b * N + (long long)i * 64 + tok) * Hq + head) * D;
      const float inv_l = 1.f / l;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        tc::tmem_ld32(o_addr + c0, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          float gv[8];
          load8(gate + off + c0 + c, gv);
#pragma unroll
          for (int e = 0; e < 8; ++e) gv[e] = sigmoidf_(gv[e]) * o[c + e] * inv_l;
          store8(out + off + c0 + c, gv);
        }
      }
    }
  }

  // ---- teardown
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace sala
