// libsala C-ABI host layer: argument validation, workspace layout, launches.
//
// Every entry point validates its arguments before launching anything and
// returns SALA_ERR_INVALID_ARG / SALA_ERR_UNSUPPORTED / SALA_ERR_WORKSPACE
// synchronously; launches go to the caller's stream.  The library allocates
// no memory: scratch lives in the caller's workspace.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <type_traits>
#include <math.h>
#include <string.h>

#include "../../include/sala.h"
#include "block.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "linear_simt.cuh"
#include "linear_seg_tc.cuh"
#include "prologue.cuh"
#include "select.cuh"
#include "select_token.cuh"
#include "sparse_simt.cuh"
#include "sparse_tc.cuh"

#include <cublasLt.h>
#include <cudaTypedefs.h>

using namespace sala;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

inline bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }
inline bool aligned16_or_null(const void* p) { return !p || ((uintptr_t)p & 15u) == 0; }

std::atomic<uint64_t> g_launches{0};

// Called once after every kernel launch: counts it and maps the launch error.
inline sala_status launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? SALA_OK : SALA_ERR_CUDA;
}

template <typename K>
inline cudaError_t allow_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

sala_status check_linear(const sala_linear_desc* d) {
  if (!d) return SALA_ERR_INVALID_ARG;
  if (d->batch < 1 || d->seqlen < 1 || d->heads < 1 || d->chunk < 1) return SALA_ERR_INVALID_ARG;
  if (d->dtype != SALA_F32 && d->dtype != SALA_BF16) return SALA_ERR_INVALID_ARG;
  if (!(d->rms_eps >= 0.f) || !(d->rope_base > 0.f) || !isfinite(d->scale) || d->pos0 < 0)
    return SALA_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return SALA_ERR_UNSUPPORTED;
  if (d->seqlen % d->chunk != 0 || d->seqlen % kSimtChunk != 0) return SALA_ERR_UNSUPPORTED;
  return SALA_OK;
}

sala_status check_sparse(const sala_sparse_desc* d) {
  if (!d) return SALA_ERR_INVALID_ARG;
  if (d->batch < 1 || d->seqlen < 1 || d->q_heads < 1 || d->kv_heads < 1) return SALA_ERR_INVALID_ARG;
  if (d->q_heads % d->kv_heads != 0) return SALA_ERR_INVALID_ARG;
  if (d->topk < 0 || d->n_init < 0 || d->n_local < 1 || d->block < 1) return SALA_ERR_INVALID_ARG;
  if (d->dtype != SALA_F32 && d->dtype != SALA_BF16) return SALA_ERR_INVALID_ARG;
  if (!(d->rms_eps >= 0.f) || !isfinite(d->scale)) return SALA_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return SALA_ERR_UNSUPPORTED;
  if (d->block != 64 || d->seqlen % d->block != 0) return SALA_ERR_UNSUPPORTED;
  if (d->topk + d->n_init + d->n_local > 1024) return SALA_ERR_UNSUPPORTED;
  if (d->seqlen / d->block > 49152) return SALA_ERR_UNSUPPORTED;   // select smem: 4 B per block
  if (d->selection != SALA_SELECT_BLOCK_MEAN && d->selection != SALA_SELECT_TOKEN_SOFTMAX)
    return SALA_ERR_INVALID_ARG;
  if (d->selection == SALA_SELECT_TOKEN_SOFTMAX &&
      (d->seqlen / d->block > kTsMaxCand || d->q_heads / d->kv_heads > 64))
    return SALA_ERR_UNSUPPORTED;
  return SALA_OK;
}

inline float sparse_scale(const sala_sparse_desc* d) {
  return d->scale > 0.f ? d->scale : 1.0f / sqrtf((float)d->head_dim);
}

// Failure-detection self-test: one thread waits, with the library's bounded
// wait, on an mbarrier that no thread arrives at.  The wait runs out, sets
// the timeout bit of the status word and the kernel returns.
__global__ void selftest_unarrived_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)tc::mbar_wait(&bar, 0);
}

// base^(-2i/D) for i < D/2 in fp64
RopeFreq rope_freq(int D, float base) {
  RopeFreq rf;
  memset(&rf, 0, sizeof(rf));
  const double log2_base = log2((double)base);
  for (int i = 0; i < D / 2; ++i) rf.inv[i] = exp2(-2.0 * i / D * log2_base);
  return rf;
}

struct LinearWs {
  size_t qn, kn, seg, total;
};
inline bool linear_on_tc(const sala_linear_desc* d) {
  return d->dtype == SALA_BF16 && d->head_dim == 128;
}
// Workspace: the tensor-core path (bf16, head_dim 128) normalises and rotates
// Q and K inside its kernels and only needs the per-segment states; the
// CUDA-core path keeps normalised bf16 copies of Q and K.
LinearWs linear_ws(const sala_linear_desc* d) {
  const size_t n = (size_t)d->batch * d->seqlen * d->heads * d->head_dim;
  LinearWs w;
  if (linear_on_tc(d)) {
    const LinSegPlan p = lin_seg_plan(d->batch, d->heads, d->seqlen);
    w.qn = w.kn = w.seg = 0;
    w.total = align_up((size_t)d->batch * d->heads * p.n_seg * 128 * 128 * 4);
    return w;
  }
  w.qn = 0;
  w.kn = align_up(n * 2);
  w.seg = w.kn + align_up(n * 2);
  w.total = w.seg;
  return w;
}

sala_status run_linear_seg(const sala_linear_desc* d, const void* q, const void* k,
                           const void* v, const void* gate, const float* lambda,
                           const float* wq, const float* wk, const float* state_in,
                           float* state_out, void* out, float* seg_state, cudaStream_t st);

template <typename T, int D>
sala_status run_linear(const sala_linear_desc* d, const void* q, const void* k, const void* v,
                       const void* gate, const float* lambda, const float* wq, const float* wk,
                       const float* state_in, float* state_out, void* out, char* ws,
                       cudaStream_t st) {
  const LinearWs w = linear_ws(d);
  // bf16 activations with head_dim 128 run on the tensor cores (norm and RoPE
  // fused into the kernels); fp32 activations and head_dim 64 on CUDA cores
  // after a separate norm / RoPE prologue.
  if (std::is_same<T, __nv_bfloat16>::value && D == 128)
    return run_linear_seg(d, q, k, v, gate, lambda, wq, wk, state_in, state_out, out,
                          reinterpret_cast<float*>(ws + w.seg), st);
  auto* qn = reinterpret_cast<__nv_bfloat16*>(ws + w.qn);
  auto* kn = reinterpret_cast<__nv_bfloat16*>(ws + w.kn);
  const long long tokens = (long long)d->batch * d->seqlen;
  const int pro_blocks = (int)((tokens + kRopeTokens - 1) / kRopeTokens);
  linear_prologue_kernel<T, D><<<pro_blocks, kPrologueThreads, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), wq, wk, qn, kn, tokens, d->seqlen,
      d->heads, d->pos0, rope_freq(D, d->rope_base), d->rms_eps);
  if (launch_status() != SALA_OK) return SALA_ERR_CUDA;
  const size_t smem = sizeof(SimtSmem<D>);
  if (allow_smem(linear_chunk_simt_kernel<T, D>, smem) != cudaSuccess) return SALA_ERR_CUDA;
  const int grid = d->batch * d->heads * (D / kSimtCols);
  linear_chunk_simt_kernel<T, D><<<grid, kSimtThreads, smem, st>>>(
      qn, kn, static_cast<const T*>(v), static_cast<const T*>(gate), lambda, state_in, state_out,
      static_cast<T*>(out), d->seqlen, d->heads, d->scale);
  return launch_status();
}

// Normalisation and block means of the sparse layer: q_norm, k_norm, kbar,
// and qsum [B, nb, Hkv, D] = sum over the group's q heads of the block-mean
// normalised queries.
template <typename T, int D>
sala_status run_select_begin(const sala_sparse_desc* d, const void* q, const void* k,
                             const float* wq, const float* wk, void* q_norm, void* k_norm,
                             float* kbar, float* qsum, cudaStream_t st) {
  const int nb = d->seqlen / d->block;
  sparse_prologue_kernel<T, D><<<d->batch * nb * d->kv_heads, kPrologueThreads, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), wq, wk,
      static_cast<__nv_bfloat16*>(q_norm), static_cast<__nv_bfloat16*>(k_norm), qsum, kbar,
      d->seqlen, d->q_heads, d->kv_heads, d->block, d->rms_eps);
  return launch_status();
}

// SMs of the current device (cached per device).
int device_sms() {
  static int sms[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  return sms[dev];
}

// Block-mean ranking of every query block from qsum and kbar.
template <int D>
sala_status run_select_finish(const sala_sparse_desc* d, const float* qsum, const float* kbar,
                              int32_t* idx, cudaStream_t st) {
  const int nb = d->seqlen / d->block;
  const int width = d->topk + d->n_init + d->n_local;
  const int per = select_buffer_per(d->topk);
  const int tq = select_rows_per_cta((long long)d->batch * d->kv_heads * nb, per, std::max(device_sms(), 1));
  const size_t smem = (size_t)tq * per * kSelectThreads * 8;
  const int n_tiles = (nb + tq - 1) / tq;
  const int grid = d->batch * d->kv_heads * n_tiles;
  auto launch = [&](auto kern) {
    if (allow_smem(kern, smem) != cudaSuccess) return SALA_ERR_CUDA;
    kern<<<grid, kSelectThreads, smem, st>>>(qsum, kbar, idx, nb, d->kv_heads, d->topk, d->n_init,
                                             d->n_local, width, tq);
    return launch_status();
  };
  if (per == 2) return launch(select_topk_kernel<D, 2>);
  if (per == 4) return launch(select_topk_kernel<D, 4>);
  return launch(select_topk_kernel<D, 8>);
}

template <typename T, int D>
sala_status run_select(const sala_sparse_desc* d, const void* q, const void* k, const float* wq,
                       const float* wk, void* q_norm, void* k_norm, float* kbar, int32_t* idx,
                       char* ws, cudaStream_t st) {
  const int nb = d->seqlen / d->block;
  float* qsum = reinterpret_cast<float*>(ws);
  if (run_select_begin<T, D>(d, q, k, wq, wk, q_norm, k_norm, kbar, qsum, st) != SALA_OK)
    return SALA_ERR_CUDA;
  const int width = d->topk + d->n_init + d->n_local;
  if (d->selection == SALA_SELECT_TOKEN_SOFTMAX) {
    const size_t ts_smem = TsLayout<D>::bytes(nb);
    if (allow_smem(select_token_softmax_kernel<T, D>, ts_smem) != cudaSuccess) return SALA_ERR_CUDA;
    select_token_softmax_kernel<T, D><<<d->batch * d->kv_heads * nb, kTsThreads, ts_smem, st>>>(
        static_cast<const T*>(q), wq, kbar, idx, nb, d->q_heads, d->kv_heads, d->topk, d->n_init,
        d->n_local, width, d->rms_eps);
    return launch_status();
  }
  return run_select_finish<D>(d, qsum, kbar, idx, st);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D bf16 view [rows, cols] (cols contiguous) loaded in boxes of
// box_cols x box_rows.  With 128-byte swizzle and 64-column boxes one box
// fills box_rows x 128 B of a K-major or MN-major MMA operand; with 64-byte
// swizzle and 32-column boxes, box_rows x 64 B.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                    uint32_t box_cols = 64, uint32_t box_rows = 64,
                    CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

sala_status run_linear_seg(const sala_linear_desc* d, const void* q, const void* k,
                           const void* v, const void* gate, const float* lambda,
                           const float* wq, const float* wk, const float* state_in,
                           float* state_out, void* out, float* seg_state, cudaStream_t st) {
  constexpr int D = 128;
  const LinSegPlan p = lin_seg_plan(d->batch, d->heads, d->seqlen);
  const uint64_t rows = (uint64_t)d->batch * d->seqlen, cols = (uint64_t)d->heads * D;
  const RopeFreq rf = rope_freq(D, d->rope_base);
  RopeF32 rt;
  for (int i = 0; i < 64; ++i) rt.th[i] = (float)rf.inv[i];
  CUtensorMap qm, km, vm, gm;
  if (!make_tmap_bf16(&qm, q, cols, rows, 64, kLsTile) ||
      !make_tmap_bf16(&km, k, cols, rows, 64, kLsTile) ||
      !make_tmap_bf16(&vm, v, cols, rows, 64, kLsTile) ||
      !make_tmap_bf16(&gm, gate, cols, rows, 64, kLsTile))
    return SALA_ERR_CUDA;
  const int grid = d->batch * d->heads * p.n_seg;
  // 1. segment sums
  const size_t smem_a = LsSumLayout::kBytes + 1024;
  if (allow_smem(linear_segsum_kernel, smem_a) != cudaSuccess) return SALA_ERR_CUDA;
  linear_segsum_kernel<<<grid, kLsSumThreads, smem_a, st>>>(
      km, vm, lambda, wk, d->rms_eps, d->pos0, rf, rt, seg_state, d->seqlen, d->heads, p.seg_tiles,
      p.n_seg);
  if (launch_status() != SALA_OK) return SALA_ERR_CUDA;
  // 2. scan over segments
  const long long n_el = (long long)d->batch * d->heads * D * D;
  linear_segscan_kernel<<<(unsigned)((n_el + kLsScanThreads - 1) / kLsScanThreads), kLsScanThreads,
                          0, st>>>(lambda, state_in, state_out, seg_state, d->seqlen, d->heads,
                                   p.seg_tiles, p.n_seg, n_el);
  if (launch_status() != SALA_OK) return SALA_ERR_CUDA;
  // 3. outputs
  const size_t smem_b = LsOutLayout::kBytes + 1024;
  auto kern = linear_segout_kernel<__nv_bfloat16>;
  if (allow_smem(kern, smem_b) != cudaSuccess) return SALA_ERR_CUDA;
  // The in-kernel register split assumes this launch allocation exactly.
  // The build refuses to produce a library where it differs; this cached
  // check only keeps a library built some other way from launching a split
  // larger than its allocation (which would never finish).
  static std::atomic<int> regs_ok{0};   // 0 unknown, 1 matches, 2 differs
  if (regs_ok.load(std::memory_order_relaxed) == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return SALA_ERR_CUDA;
    regs_ok.store(fa.numRegs == kLsOutRegsLaunch ? 1 : 2, std::memory_order_relaxed);
  }
  if (regs_ok.load(std::memory_order_relaxed) != 1) return SALA_ERR_UNSUPPORTED;
  kern<<<grid, kLsOutThreads, smem_b, st>>>(qm, km, vm, gm, static_cast<const __nv_bfloat16*>(gate),
                                            lambda, wq, wk, d->rms_eps, d->pos0, rf, rt, seg_state,
                                            static_cast<__nv_bfloat16*>(out), d->seqlen, d->heads,
                                            p.seg_tiles, p.n_seg, d->scale);
  return launch_status();
}

template <int D>
sala_status run_sparse_prefill_tc(const sala_sparse_desc* d, const void* qn, const void* kn,
                                  const void* v, const void* gate, const int32_t* idx, void* out,
                                  cudaStream_t st) {
  const int nb = d->seqlen / d->block;
  const uint64_t rows = (uint64_t)d->batch * d->seqlen;
  CUtensorMap qm, km, vm;
  if (!make_tmap_bf16(&qm, qn, (uint64_t)d->q_heads * D, rows) ||
      !make_tmap_bf16(&km, kn, (uint64_t)d->kv_heads * D, rows) ||
      !make_tmap_bf16(&vm, v, (uint64_t)d->kv_heads * D, rows))
    return SALA_ERR_CUDA;
  const int width = d->topk + d->n_init + d->n_local;
  const size_t smem = SpTcLayout<D>::kBytes(width) + 1024;
  auto kern = sparse_attn_tc_kernel<__nv_bfloat16, D>;
  if (allow_smem(kern, smem) != cudaSuccess) return SALA_ERR_CUDA;
  const int G = d->q_heads / d->kv_heads;
  const long long grid = (long long)d->batch * d->kv_heads * nb * (G / kSpTcHeadsPerCta);
  const float sl2 = sparse_scale(d) * 1.4426950408889634f;
  kern<<<(unsigned)grid, kSpTcThreads, smem, st>>>(
      qm, km, vm, idx, static_cast<const __nv_bfloat16*>(gate), static_cast<__nv_bfloat16*>(out),
      d->seqlen, d->q_heads, d->kv_heads, width, sl2);
  return launch_status();
}

template <typename T, int D>
sala_status run_sparse_prefill(const sala_sparse_desc* d, const void* qn, const void* kn,
                               const void* v, const void* gate, const int32_t* idx, void* out,
                               cudaStream_t st) {
  // bf16 activations with a GQA group of a multiple of 4 q heads run on the
  // tensor cores; other shapes (fp32 activations, small groups) on CUDA cores.
  if (std::is_same<T, __nv_bfloat16>::value && (d->q_heads / d->kv_heads) % kSpTcHeadsPerCta == 0)
    return run_sparse_prefill_tc<D>(d, qn, kn, v, gate, idx, out, st);
  const int nb = d->seqlen / d->block;
  const size_t smem = sizeof(SpSimtSmem<D>);
  if (allow_smem(sparse_attn_simt_kernel<T, D>, smem) != cudaSuccess) return SALA_ERR_CUDA;
  sparse_attn_simt_kernel<T, D><<<d->batch * nb * d->kv_heads, kSpSimtThreads, smem, st>>>(
      static_cast<const __nv_bfloat16*>(qn), static_cast<const __nv_bfloat16*>(kn),
      static_cast<const T*>(v), static_cast<const T*>(gate), idx, static_cast<T*>(out),
      d->seqlen, d->q_heads, d->kv_heads, d->topk + d->n_init + d->n_local, sparse_scale(d));
  return launch_status();
}

struct DecodeWs {
  size_t ctl, hist, keys, idx, qhat, part, total, zero_bytes;
};
DecodeWs decode_ws(const sala_decode_desc* d) {
  const sala_sparse_desc& s = d->sp;
  const size_t B = s.batch, Hq = s.q_heads, Hkv = s.kv_heads, D = s.head_dim;
  const size_t BG = B * Hkv, G = Hq / Hkv;
  const size_t width = s.topk + s.n_init + s.n_local;
  const size_t capb = (size_t)(d->cache_capacity / s.block);
  DecodeWs w;
  w.ctl = 0;
  w.hist = w.ctl + align_up(dec_ctl_words((int)BG) * 4);
  w.keys = w.hist + align_up(BG * kDecBins * 4);
  w.zero_bytes = w.keys;                         // control words and histograms
  w.idx = w.keys + align_up(BG * dec_key_stride((long long)capb) * 4);
  w.qhat = w.idx + align_up(BG * width * 4);
  w.part = w.qhat + align_up(B * Hq * D * 4);
  w.total = w.part + align_up(BG * width * G * (D + 4) * 4);
  return w;
}

sala_status check_decode(const sala_decode_desc* d) {
  if (!d) return SALA_ERR_INVALID_ARG;
  if (d->n_linear < 1 || d->n_linear > SALA_MAX_LAYERS - 1) return SALA_ERR_INVALID_ARG;
  sala_linear_desc l = d->lin;
  l.seqlen = l.chunk = 64;
  l.pos0 = 0;
  sala_status s = check_linear(&l);
  if (s != SALA_OK) return s;
  sala_sparse_desc sp = d->sp;
  sp.seqlen = sp.block;
  s = check_sparse(&sp);
  if (s != SALA_OK) return s;
  if (d->lin.batch != d->sp.batch || d->lin.dtype != d->sp.dtype) return SALA_ERR_INVALID_ARG;
  if (d->cache_capacity < d->sp.block || d->cache_capacity % d->sp.block != 0) return SALA_ERR_INVALID_ARG;
  if (d->cache_capacity / d->sp.block > 49152) return SALA_ERR_UNSUPPORTED;
  if (d->sp.q_heads > kDecodeMaxQHeads) return SALA_ERR_UNSUPPORTED;
  if (d->sp.selection != SALA_SELECT_BLOCK_MEAN) return SALA_ERR_UNSUPPORTED;
  return SALA_OK;
}

template <typename T, int D>
sala_status run_decode(const sala_decode_desc* d, const sala_decode_io* io, void* k_cache,
                       void* v_cache, float* kbar, float* ksum, int64_t cur_len, char* ws,
                       cudaStream_t st) {
  const sala_linear_desc& L = d->lin;
  const sala_sparse_desc& S = d->sp;
  const DecodeWs w = decode_ws(d);
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  for (int l = 0; l < d->n_linear; ++l) {
    p.lq[l] = io->q[l]; p.lk[l] = io->k[l]; p.lv[l] = io->v[l]; p.lgate[l] = io->gate[l];
    p.lwq[l] = io->wq[l]; p.lwk[l] = io->wk[l]; p.llam[l] = io->lambda[l];
    p.lstate[l] = io->lin_state[l]; p.lout[l] = io->out[l];
  }
  p.n_linear = d->n_linear;
  p.B = L.batch;
  p.H = L.heads;
  p.eps_l = L.rms_eps;
  p.scale_l = L.scale;
  const int sl = d->n_linear;
  p.q = io->q[sl]; p.k = io->k[sl]; p.v = io->v[sl]; p.gate = io->gate[sl]; p.out = io->out[sl];
  p.wq = io->wq[sl]; p.wk = io->wk[sl];
  p.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  p.kbar = kbar;
  p.ksum = ksum;
  p.Hq = S.q_heads; p.Hkv = S.kv_heads; p.BLK = S.block; p.topk = S.topk; p.n_init = S.n_init;
  p.n_local = S.n_local; p.width = S.topk + S.n_init + S.n_local;
  p.cap = d->cache_capacity;
  p.capb = d->cache_capacity / S.block;
  p.kstride = dec_key_stride(p.capb);
  p.pos = cur_len;
  p.eps_s = S.rms_eps;
  p.sl2 = sparse_scale(&S) * 1.4426950408889634f;
  p.bcur = (int)(cur_len / S.block);
  p.n_cand = std::max(0, p.bcur - S.n_local + 1 - S.n_init);
  p.kk = std::min(S.topk, p.n_cand);
  p.n_chunks = std::max(1, (p.n_cand + kDecChunk - 1) / kDecChunk);
  p.ctl = reinterpret_cast<unsigned*>(ws + w.ctl);
  p.hist = reinterpret_cast<unsigned*>(ws + w.hist);
  p.keys = reinterpret_cast<uint32_t*>(ws + w.keys);
  p.idx = reinterpret_cast<int*>(ws + w.idx);
  p.qhat = reinterpret_cast<float*>(ws + w.qhat);
  p.part = reinterpret_cast<float*>(ws + w.part);
  p.rf = rope_freq(D, L.rope_base);
  // barrier counters, per-(batch, kv head) counts and histograms start at zero
  if (cudaMemsetAsync(ws, 0, w.zero_bytes, st) != cudaSuccess) return SALA_ERR_CUDA;
  const int G = S.q_heads / S.kv_heads;
  const size_t smem = decode_smem_bytes(D, G, S.topk, p.kstride, p.width);
  auto kern = decode_step_kernel<T, D>;
  if (allow_smem(kern, smem) != cudaSuccess) return SALA_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecThreads, smem) !=
          cudaSuccess || per_sm < 1)
    return SALA_ERR_CUDA;
  const int grid = device_sms() * std::min(per_sm, 1);
  if (grid < 1) return SALA_ERR_CUDA;
  void* args[] = {&p};
  const cudaError_t e = cudaLaunchCooperativeKernel((const void*)kern, grid, kDecThreads, args,
                                                    smem, st);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return e == cudaSuccess ? SALA_OK : SALA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Allocation-free selection (sala_sparse_select_noalloc).
//
// Some callers cannot call cudaMalloc at all: code running inside an
// allocator-free runtime or a memory pool that forbids extra device
// allocations, or a host that must not allocate while a stream is being
// captured.  For them the selection's scratch (the group-summed query block
// means, B * (N/block) * Hkv * head_dim fp32 values) lives in this
// file-scope device array instead of a caller workspace.  It is loaded with
// the library and stays resident on every GPU that loads it until the
// process exits.
constexpr size_t kNoAllocScratchBytes = SALA_NOALLOC_SCRATCH_BYTES;   // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  Host code only
// sees a host-side stand-in under that name, so the address is looked up
// once per device (with that device current) and cached.
sala_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SALA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SALA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SALA_OK;
}

// ---------------------------------------------------------------------------
// Decoder block around the attention: GEMMs in cuBLASLt.

// One cuBLASLt handle per device, created on first use with that device
// current (host-side object; it allocates no device memory).
cublasLtHandle_t lt_handle() {
  static std::mutex mu;
  static cublasLtHandle_t handles[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!handles[dev] && cublasLtCreate(&handles[dev]) != CUBLAS_STATUS_SUCCESS) handles[dev] = nullptr;
  return handles[dev];
}

constexpr size_t kLtWorkspace = (size_t)32 << 20;

// D[m, o] = alpha * sum_k X[m, k] W[o, k] + beta * C[m, o]   (X, W bf16 row
// major; C, D of type `cd`, row major; fp32 accumulation).  In cuBLASLt's
// column-major terms: D^T [out, rows] = op_T(W^T [in, out]) * X^T [in, rows].
sala_status lt_gemm(cudaStream_t st, const void* W, const void* X, const void* C, void* D,
                    long long rows, int in, int out, cudaDataType_t cd, float beta, void* lt_ws) {
  cublasLtHandle_t h = lt_handle();
  if (!h) return SALA_ERR_CUDA;
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  sala_status res = SALA_ERR_CUDA;
  const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
  const float alpha = 1.0f;
  size_t ws_bytes = kLtWorkspace;
  cublasLtMatmulHeuristicResult_t heur;
  int found = 0;
  if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) goto done;
  if (cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta)) ||
      cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb)))
    goto done;
  if (cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, in, out, in) ||
      cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, in, rows, in) ||
      cublasLtMatrixLayoutCreate(&lc, cd, out, rows, out))
    goto done;
  if (cublasLtMatmulPreferenceCreate(&pref) ||
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES,
                                           &ws_bytes, sizeof(ws_bytes)))
    goto done;
  if (cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &heur, &found) ||
      found < 1)
    goto done;
  if (cublasLtMatmul(h, op, &alpha, W, la, X, lb, &beta, C ? C : D, lc, D, lc, &heur.algo, lt_ws,
                     kLtWorkspace, st) == CUBLAS_STATUS_SUCCESS)
    res = SALA_OK;
done:
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return res;
}

struct BlockWs {
  size_t xn, q, k, v, g, a, u, s, lt, att, total;
  int hq, hk, d;
  long long rows;
};

sala_status check_block(const sala_block_desc* b, const sala_linear_desc* lin,
                        const sala_sparse_desc* sp, BlockWs* w) {
  if (!b || (!lin) == (!sp)) return SALA_ERR_INVALID_ARG;
  if (b->hidden < 8 || b->hidden % 8 || b->ffn < 8 || b->ffn % 8 || !(b->rms_eps >= 0.f))
    return SALA_ERR_INVALID_ARG;
  sala_status s = lin ? check_linear(lin) : check_sparse(sp);
  if (s != SALA_OK) return s;
  if ((lin ? lin->dtype : sp->dtype) != SALA_BF16) return SALA_ERR_UNSUPPORTED;
  w->d = lin ? lin->head_dim : sp->head_dim;
  w->hq = lin ? lin->heads : sp->q_heads;
  w->hk = lin ? lin->heads : sp->kv_heads;
  if (w->hq * w->d != b->hidden) return SALA_ERR_INVALID_ARG;
  w->rows = (long long)(lin ? lin->batch : sp->batch) * (lin ? lin->seqlen : sp->seqlen);
  const size_t R = (size_t)w->rows;
  w->xn = 0;
  w->q = w->xn + align_up(R * b->hidden * 2);
  w->k = w->q + align_up(R * w->hq * w->d * 2);
  w->v = w->k + align_up(R * w->hk * w->d * 2);
  w->g = w->v + align_up(R * w->hk * w->d * 2);
  w->a = w->g + align_up(R * w->hq * w->d * 2);
  w->u = w->a + align_up(R * w->hq * w->d * 2);
  w->s = w->u + align_up(R * 2 * (size_t)b->ffn * 2);
  w->lt = w->s + align_up(R * (size_t)b->ffn * 2);
  w->att = w->lt + align_up(kLtWorkspace);
  if (lin) {
    w->total = w->att + align_up(linear_ws(lin).total);
  } else {
    const size_t nb = (size_t)sp->batch * (sp->seqlen / sp->block);
    const size_t sel = align_up(nb * sp->kv_heads * sp->head_dim * 4);          // qsum
    const size_t qn = align_up(R * sp->q_heads * sp->head_dim * 2);
    const size_t kn = align_up(R * sp->kv_heads * sp->head_dim * 2);
    const size_t kb = align_up(nb * sp->kv_heads * sp->head_dim * 4);
    const size_t ix = align_up(nb * sp->kv_heads * (sp->topk + sp->n_init + sp->n_local) * 4);
    w->total = w->att + sel + qn + kn + kb + ix;
  }
  return SALA_OK;
}

template <int D>
sala_status run_block(const sala_block_desc* b, const sala_linear_desc* lin,
                      const sala_sparse_desc* sp, const sala_block_weights* wt,
                      const float* lambda, const float* x, float* y, float* state_out, char* ws,
                      const BlockWs& w, cudaStream_t st) {
  using bf = __nv_bfloat16;
  const long long R = w.rows;
  const int H = b->hidden;
  bf* xn = reinterpret_cast<bf*>(ws + w.xn);
  void* q = ws + w.q;
  void* k = ws + w.k;
  void* v = ws + w.v;
  void* g = ws + w.g;
  void* a = ws + w.a;
  void* lt = ws + w.lt;
  // attention sub-block
  block_rmsnorm_kernel<<<(unsigned)R, kBlkNormThreads, 0, st>>>(x, wt->norm_attn, xn, H, b->rms_eps);
  if (launch_status() != SALA_OK) return SALA_ERR_CUDA;
  if (lt_gemm(st, wt->wq, xn, nullptr, q, R, H, w.hq * D, CUDA_R_16BF, 0.f, lt) ||
      lt_gemm(st, wt->wk, xn, nullptr, k, R, H, w.hk * D, CUDA_R_16BF, 0.f, lt) ||
      lt_gemm(st, wt->wv, xn, nullptr, v, R, H, w.hk * D, CUDA_R_16BF, 0.f, lt) ||
      lt_gemm(st, wt->wg, xn, nullptr, g, R, H, w.hq * D, CUDA_R_16BF, 0.f, lt))
    return SALA_ERR_CUDA;
  sala_status s;
  char* att = ws + w.att;
  if (lin) {
    s = run_linear<bf, D>(lin, q, k, v, g, lambda, wt->qk_norm_q, wt->qk_norm_k, nullptr,
                          state_out, a, att, st);
  } else {
    const size_t nb = (size_t)sp->batch * (sp->seqlen / sp->block);
    char* qsum = att;
    char* qn = qsum + align_up(nb * sp->kv_heads * D * 4);
    char* kn = qn + align_up((size_t)R * sp->q_heads * D * 2);
    char* kb = kn + align_up((size_t)R * sp->kv_heads * D * 2);
    char* ix = kb + align_up(nb * sp->kv_heads * D * 4);
    s = run_select<bf, D>(sp, q, k, wt->qk_norm_q, wt->qk_norm_k, qn, kn,
                          reinterpret_cast<float*>(kb), reinterpret_cast<int32_t*>(ix), qsum, st);
    if (s == SALA_OK)
      s = run_sparse_prefill<bf, D>(sp, qn, kn, v, g, reinterpret_cast<int32_t*>(ix), a, st);
  }
  if (s != SALA_OK) return s;
  // h = x + a Wo^T (fp32 residual stream, in y)
  if (lt_gemm(st, wt->wo, a, x, y, R, w.hq * D, H, CUDA_R_32F, 1.f, lt)) return SALA_ERR_CUDA;
  // feed-forward sub-block
  block_rmsnorm_kernel<<<(unsigned)R, kBlkNormThreads, 0, st>>>(y, wt->norm_ffn, xn, H, b->rms_eps);
  if (launch_status() != SALA_OK) return SALA_ERR_CUDA;
  void* u = ws + w.u;
  bf* sg = reinterpret_cast<bf*>(ws + w.s);
  if (lt_gemm(st, wt->w13, xn, nullptr, u, R, H, 2 * b->ffn, CUDA_R_16BF, 0.f, lt))
    return SALA_ERR_CUDA;
  const long long n8 = R * (b->ffn / 8);
  block_swiglu_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(static_cast<const bf*>(u), sg, R,
                                                                     b->ffn);
  if (launch_status() != SALA_OK) return SALA_ERR_CUDA;
  if (lt_gemm(st, wt->w2, sg, y, y, R, b->ffn, H, CUDA_R_32F, 1.f, lt)) return SALA_ERR_CUDA;
  return SALA_OK;
}

}  // namespace

extern "C" {

int sala_sparse_index_width(const sala_sparse_desc* d) {
  return d ? d->topk + d->n_init + d->n_local : -1;
}

size_t sala_linear_workspace_size(const sala_linear_desc* d) {
  if (check_linear(d) != SALA_OK) return 0;
  return linear_ws(d).total;
}

sala_status sala_linear_prefill(const sala_linear_desc* d, const void* q, const void* k,
                                const void* v, const void* gate, const float* lambda,
                                const float* wq, const float* wk, const float* state_in,
                                float* state_out, void* out, void* workspace, size_t ws_bytes,
                                void* stream) {
  sala_status s = check_linear(d);
  if (s != SALA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(out) ||
      !aligned16(lambda) || !aligned16(wq) || !aligned16(wk) || !aligned16_or_null(state_in) ||
      !aligned16_or_null(state_out))
    return SALA_ERR_INVALID_ARG;
  if (ws_bytes < linear_ws(d).total || !aligned16(workspace)) return SALA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (d->dtype == SALA_BF16) {
    if (d->head_dim == 128)
      return run_linear<__nv_bfloat16, 128>(d, q, k, v, gate, lambda, wq, wk, state_in, state_out, out, ws, st);
    return run_linear<__nv_bfloat16, 64>(d, q, k, v, gate, lambda, wq, wk, state_in, state_out, out, ws, st);
  }
  if (d->head_dim == 128)
    return run_linear<float, 128>(d, q, k, v, gate, lambda, wq, wk, state_in, state_out, out, ws, st);
  return run_linear<float, 64>(d, q, k, v, gate, lambda, wq, wk, state_in, state_out, out, ws, st);
}

size_t sala_sparse_workspace_size(const sala_sparse_desc* d) {
  if (check_sparse(d) != SALA_OK) return 0;
  return align_up((size_t)d->batch * (d->seqlen / d->block) * d->kv_heads * d->head_dim * 4);
}

sala_status sala_sparse_select(const sala_sparse_desc* d, const void* q, const void* k,
                               const float* wq, const float* wk, void* q_norm, void* k_norm,
                               float* kbar, int32_t* idx, void* workspace, size_t ws_bytes,
                               void* stream) {
  sala_status s = check_sparse(d);
  if (s != SALA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(wq) || !aligned16(wk) || !aligned16(q_norm) ||
      !aligned16(k_norm) || !aligned16(kbar) || !aligned16(idx))
    return SALA_ERR_INVALID_ARG;
  if (ws_bytes < sala_sparse_workspace_size(d) || !aligned16(workspace)) return SALA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (d->dtype == SALA_BF16) {
    if (d->head_dim == 128)
      return run_select<__nv_bfloat16, 128>(d, q, k, wq, wk, q_norm, k_norm, kbar, idx, ws, st);
    return run_select<__nv_bfloat16, 64>(d, q, k, wq, wk, q_norm, k_norm, kbar, idx, ws, st);
  }
  if (d->head_dim == 128)
    return run_select<float, 128>(d, q, k, wq, wk, q_norm, k_norm, kbar, idx, ws, st);
  return run_select<float, 64>(d, q, k, wq, wk, q_norm, k_norm, kbar, idx, ws, st);
}

sala_status sala_sparse_select_begin(const sala_sparse_desc* d, const void* q, const void* k,
                                     const float* wq, const float* wk, void* q_norm,
                                     void* k_norm, float* kbar, float* qsum, void* stream) {
  sala_status s = check_sparse(d);
  if (s != SALA_OK) return s;
  if (d->selection != SALA_SELECT_BLOCK_MEAN) return SALA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(wq) || !aligned16(wk) || !aligned16(q_norm) ||
      !aligned16(k_norm) || !aligned16(kbar) || !aligned16(qsum))
    return SALA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->dtype == SALA_BF16) {
    if (d->head_dim == 128)
      return run_select_begin<__nv_bfloat16, 128>(d, q, k, wq, wk, q_norm, k_norm, kbar, qsum, st);
    return run_select_begin<__nv_bfloat16, 64>(d, q, k, wq, wk, q_norm, k_norm, kbar, qsum, st);
  }
  if (d->head_dim == 128)
    return run_select_begin<float, 128>(d, q, k, wq, wk, q_norm, k_norm, kbar, qsum, st);
  return run_select_begin<float, 64>(d, q, k, wq, wk, q_norm, k_norm, kbar, qsum, st);
}

sala_status sala_sparse_select_finish(const sala_sparse_desc* d, const float* qsum,
                                      const float* kbar, int32_t* idx, void* stream) {
  sala_status s = check_sparse(d);
  if (s != SALA_OK) return s;
  if (d->selection != SALA_SELECT_BLOCK_MEAN) return SALA_ERR_UNSUPPORTED;
  if (!aligned16(qsum) || !aligned16(kbar) || !aligned16(idx)) return SALA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->head_dim == 128) return run_select_finish<128>(d, qsum, kbar, idx, st);
  return run_select_finish<64>(d, qsum, kbar, idx, st);
}

sala_status sala_sparse_prefill(const sala_sparse_desc* d, const void* q_norm,
                                const void* k_norm, const void* v, const void* gate,
                                const int32_t* idx, void* out, void* workspace, size_t ws_bytes,
                                void* stream) {
  (void)workspace;
  (void)ws_bytes;
  sala_status s = check_sparse(d);
  if (s != SALA_OK) return s;
  if (!aligned16(q_norm) || !aligned16(k_norm) || !aligned16(v) || !aligned16(gate) ||
      !aligned16(idx) || !aligned16(out))
    return SALA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->dtype == SALA_BF16) {
    if (d->head_dim == 128)
      return run_sparse_prefill<__nv_bfloat16, 128>(d, q_norm, k_norm, v, gate, idx, out, st);
    return run_sparse_prefill<__nv_bfloat16, 64>(d, q_norm, k_norm, v, gate, idx, out, st);
  }
  if (d->head_dim == 128)
    return run_sparse_prefill<float, 128>(d, q_norm, k_norm, v, gate, idx, out, st);
  return run_sparse_prefill<float, 64>(d, q_norm, k_norm, v, gate, idx, out, st);
}

sala_status sala_sparse_select_noalloc(const sala_sparse_desc* d, const void* q, const void* k,
                                       const float* wq, const float* wk, void* q_norm,
                                       void* k_norm, float* kbar, int32_t* idx, void* stream) {
  sala_status s = check_sparse(d);
  if (s != SALA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(wq) || !aligned16(wk) || !aligned16(q_norm) ||
      !aligned16(k_norm) || !aligned16(kbar) || !aligned16(idx))
    return SALA_ERR_INVALID_ARG;
  // The scratch is written in full by the normalisation kernel before the
  // scoring kernel reads it, so nothing in it has to start at zero.
  if (sala_sparse_workspace_size(d) > kNoAllocScratchBytes) return SALA_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != SALA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(scratch);
  if (d->dtype == SALA_BF16) {
    if (d->head_dim == 128)
      return run_select<__nv_bfloat16, 128>(d, q, k, wq, wk, q_norm, k_norm, kbar, idx, ws, st);
    return run_select<__nv_bfloat16, 64>(d, q, k, wq, wk, q_norm, k_norm, kbar, idx, ws, st);
  }
  if (d->head_dim == 128)
    return run_select<float, 128>(d, q, k, wq, wk, q_norm, k_norm, kbar, idx, ws, st);
  return run_select<float, 64>(d, q, k, wq, wk, q_norm, k_norm, kbar, idx, ws, st);
}

size_t sala_decode_workspace_size(const sala_decode_desc* d) {
  if (check_decode(d) != SALA_OK) return 0;
  return decode_ws(d).total;
}

sala_status sala_decode_step(const sala_decode_desc* d, const sala_decode_io* io, void* k_cache,
                             void* v_cache, float* kbar, float* ksum, int64_t cur_len,
                             void* workspace, size_t ws_bytes, void* stream) {
  sala_status s = check_decode(d);
  if (s != SALA_OK) return s;
  if (!io || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(kbar) || !aligned16(ksum))
    return SALA_ERR_INVALID_ARG;
  if (cur_len < 0 || cur_len >= d->cache_capacity) return SALA_ERR_INVALID_ARG;
  for (int l = 0; l <= d->n_linear; ++l) {
    if (!aligned16(io->q[l]) || !aligned16(io->k[l]) || !aligned16(io->v[l]) ||
        !aligned16(io->gate[l]) || !aligned16(io->out[l]) || !aligned16(io->wq[l]) ||
        !aligned16(io->wk[l]))
      return SALA_ERR_INVALID_ARG;
    if (l < d->n_linear && (!aligned16(io->lambda[l]) || !aligned16(io->lin_state[l])))
      return SALA_ERR_INVALID_ARG;
  }
  if (ws_bytes < decode_ws(d).total || !aligned16(workspace)) return SALA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const int dl = d->lin.head_dim, ds = d->sp.head_dim;
  if (dl != ds) return SALA_ERR_UNSUPPORTED;
  if (d->lin.dtype == SALA_BF16) {
    if (dl == 128) return run_decode<__nv_bfloat16, 128>(d, io, k_cache, v_cache, kbar, ksum, cur_len, ws, st);
    return run_decode<__nv_bfloat16, 64>(d, io, k_cache, v_cache, kbar, ksum, cur_len, ws, st);
  }
  if (dl == 128) return run_decode<float, 128>(d, io, k_cache, v_cache, kbar, ksum, cur_len, ws, st);
  return run_decode<float, 64>(d, io, k_cache, v_cache, kbar, ksum, cur_len, ws, st);
}

size_t sala_block_workspace_size(const sala_block_desc* b, const sala_linear_desc* lin,
                                 const sala_sparse_desc* sp) {
  BlockWs w;
  if (check_block(b, lin, sp, &w) != SALA_OK) return 0;
  return w.total;
}

sala_status sala_block_prefill(const sala_block_desc* b, const sala_linear_desc* lin,
                               const sala_sparse_desc* sp, const sala_block_weights* wt,
                               const float* lambda, const float* x, float* y, float* state_out,
                               void* workspace, size_t ws_bytes, void* stream) {
  BlockWs w;
  sala_status s = check_block(b, lin, sp, &w);
  if (s != SALA_OK) return s;
  if (!wt || !aligned16(x) || !aligned16(y) || x == y || !aligned16(wt->norm_attn) ||
      !aligned16(wt->wq) || !aligned16(wt->wk) || !aligned16(wt->wv) || !aligned16(wt->wg) ||
      !aligned16(wt->qk_norm_q) || !aligned16(wt->qk_norm_k) || !aligned16(wt->wo) ||
      !aligned16(wt->norm_ffn) || !aligned16(wt->w13) || !aligned16(wt->w2) ||
      (lin && !aligned16(lambda)) || !aligned16_or_null(state_out))
    return SALA_ERR_INVALID_ARG;
  if (ws_bytes < w.total || !aligned16(workspace)) return SALA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (w.d == 128) return run_block<128>(b, lin, sp, wt, lambda, x, y, state_out, ws, w, st);
  return run_block<64>(b, lin, sp, wt, lambda, x, y, state_out, ws, w, st);
}

const char* sala_status_string(sala_status s) {
  switch (s) {
    case SALA_OK: return "ok";
    case SALA_ERR_INVALID_ARG: return "invalid argument";
    case SALA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case SALA_ERR_CUDA: return "CUDA error";
    case SALA_ERR_TIMEOUT: return "device wait timed out";
    case SALA_ERR_WORKSPACE: return "workspace too small";
    case SALA_ERR_DEVICE_FAULT: return "device bounds check failed";
  }
  return "unknown status";
}

sala_status sala_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SALA_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return SALA_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return SALA_ERR_CUDA;
  if (v & kStatusTimeout) return SALA_ERR_TIMEOUT;
  if (v & kStatusBounds) return SALA_ERR_DEVICE_FAULT;
  return SALA_OK;
}

sala_status sala_selftest_bounded_wait(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  selftest_unarrived_wait_kernel<<<1, 32, 0, st>>>();
  if (launch_status() != SALA_OK) return SALA_ERR_CUDA;
  return sala_get_device_status(stream);
}

int sala_version(void) { return 100; }

uint64_t sala_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
