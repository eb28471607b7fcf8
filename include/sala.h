/*
 * libsala: SALA hybrid attention (Lightning-style linear layers + InfLLM-V2-style
 * block-sparse layer) prefill and decode forward on NVIDIA B200 (sm_100a).
 *
 * Method sources (the pages name the mechanisms but print no formula):
 *   - MiniCPM-SALA paper (arXiv 2602.11761), summary, abstract and section 2.1
 *     "Model architecture": 1:3 sparse:linear layer mix, QK normalisation in
 *     every layer, RoPE only in the linear layers, an output gate after each
 *     attention block; linear layers keep a constant-size state.
 *   - acgfav.com press article, section "SALA 混合架构": Lightning Attention
 *     (O(N)) in linear layers; InfLLM-V2 block selection ("each query attends
 *     to a small set of key blocks") in sparse layers; HyPE: RoPE in linear
 *     layers, NoPE in sparse layers so the KV cache holds no position.
 *   - intelliparadigm.com blog section 2.2 and yunpan.plus post section 二.2:
 *     the same HyPE split.
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller owns every buffer.  The library allocates no
 *     device or host memory; scratch space is passed in as `workspace`, sized
 *     by the matching *_workspace_size() call.
 *   - Pointers: all tensor pointers are DEVICE pointers, 16-byte aligned,
 *     contiguous.  Activations use the layout [batch, seqlen, heads, head_dim]
 *     with head_dim innermost (the layout of a projection output).
 *   - dtype: SALA_BF16 (bf16 in, bf16 out) or SALA_F32 (fp32 in, fp32 out; the
 *     kernels round operands to bf16 and accumulate in fp32).
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on it.
 *   - Errors: argument errors are returned synchronously and nothing is
 *     launched (SALA_ERR_INVALID_ARG, SALA_ERR_UNSUPPORTED, SALA_ERR_WORKSPACE).
 *     A failed launch returns SALA_ERR_CUDA.  Faults detected on the device
 *     (a bounded wait that ran out, an index out of range) set a per-device
 *     status word that sala_get_device_status() returns and clears.
 *   - Supported shapes: head_dim in {64, 128}; seqlen a multiple of the linear
 *     chunk and of the sparse block (64); q_heads a multiple of kv_heads.
 */
#ifndef SALA_H_
#define SALA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SALA_OK = 0,
  SALA_ERR_INVALID_ARG = 1,   /* NULL or misaligned pointer, bad size or count */
  SALA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim 96)   */
  SALA_ERR_CUDA = 3,          /* a CUDA launch or runtime call failed           */
  SALA_ERR_TIMEOUT = 4,       /* a bounded device-side wait ran out             */
  SALA_ERR_WORKSPACE = 5,     /* workspace smaller than *_workspace_size()      */
  SALA_ERR_DEVICE_FAULT = 6   /* a device-side bounds check fired              */
} sala_status;

typedef enum { SALA_F32 = 0, SALA_BF16 = 1 } sala_dtype;

/* Linear (Lightning-style) layer.  Per head h with decay lambda[h]:
 *   q^ = RoPE(RMSNorm(q) * wq, pos0 + t), k^ = RoPE(RMSNorm(k) * wk, pos0 + t)
 *   S_t = lambda S_{t-1} + k^_t^T v_t,   o_t = scale * q^_t S_t,
 *   out = sigmoid(gate) * o
 * computed chunk-wise (intra-chunk (Q K^T . D) V plus the carried d x d
 * state).  RMSNorm: x / sqrt(mean(x^2) + rms_eps).  RoPE: rotate-half,
 * theta_i = rope_base^(-2i/d).  `chunk` is the chunk length of the method;
 * chunking is exact, so the result does not depend on it beyond rounding. */
typedef struct {
  int batch, seqlen, heads, head_dim, chunk;
  sala_dtype dtype;
  int64_t pos0;      /* position of token 0 (0 for a fresh prefill)      */
  float rope_base;   /* 10000                                              */
  float rms_eps;     /* 1e-6                                               */
  float scale;       /* 1.0                                                */
} sala_linear_desc;

/* How the sparse layer ranks its candidate blocks.
 *   SALA_SELECT_BLOCK_MEAN: score_j = <sum_{h in group} qbar_b^h, kbar_j> / sqrt(d)
 *     with qbar / kbar the block means of the normalised queries / keys.
 *   SALA_SELECT_TOKEN_SOFTMAX: every query token t of block b and head h of
 *     the group scores z = <q^_t^h, kbar_j> / sqrt(d); a softmax over the
 *     candidate blocks makes it a distribution; importance_j = the summed
 *     probability of all (t, h) (a reading of InfLLM-V2's block selection:
 *     MiniCPM-SALA paper, summary and section 2.1).  Prefill selection only;
 *     at most 8192 blocks (524288 tokens). */
typedef enum { SALA_SELECT_BLOCK_MEAN = 0, SALA_SELECT_TOKEN_SOFTMAX = 1 } sala_selection;

/* Sparse (InfLLM-V2-style) layer.  NoPE: RMSNorm only.  Blocks of `block`
 * tokens; query block b attends to the initial blocks [0, n_init), the local
 * blocks [b-n_local+1, b] and the top-`topk` candidate blocks in
 * [n_init, b-n_local], ranked by `selection` (ties to the lower index).
 * Attention is exact softmax with logits * scale over the selected blocks'
 * keys at positions <= the query's.  scale <= 0 selects 1/sqrt(head_dim). */
typedef struct {
  int batch, seqlen, q_heads, kv_heads, head_dim, block, topk, n_init, n_local;
  sala_dtype dtype;
  float rms_eps;
  float scale;
  sala_selection selection;   /* SALA_SELECT_BLOCK_MEAN (0) unless stated */
} sala_sparse_desc;

/* Width of one index row: topk + n_init + n_local. */
int sala_sparse_index_width(const sala_sparse_desc* d);

/* ------------------------------------------------------------------ prefill */

size_t sala_linear_workspace_size(const sala_linear_desc* d);

/* One Lightning-style linear layer over N tokens (acgfav.com article, section
 * "SALA 混合架构": linear layers at O(N); MiniCPM-SALA paper, section 2.1:
 * constant-size state; QK normalisation and RoPE in these layers: paper
 * summary and the HyPE sections of the articles).
 * q, k, v, gate, out: [B, N, H, d] of d->dtype.  lambda: [H] fp32.
 * wq, wk: [d] fp32 RMSNorm weights.  state_in: [B, H, d, d] fp32 (row = key
 * dim, column = value dim) or NULL for zeros.  state_out: same layout, or
 * NULL; it may alias state_in.  workspace: >= sala_linear_workspace_size(d)
 * bytes (may be NULL when that is 0). */
sala_status sala_linear_prefill(const sala_linear_desc* d, const void* q, const void* k,
                                const void* v, const void* gate, const float* lambda,
                                const float* wq, const float* wk, const float* state_in,
                                float* state_out, void* out, void* workspace,
                                size_t ws_bytes, void* stream);

size_t sala_sparse_workspace_size(const sala_sparse_desc* d);

/* Selection stage of the sparse layer (acgfav.com article, section
 * "SALA 混合架构": a fine-grained block selection lets each query attend to a
 * small set of key blocks; NoPE in the sparse layers under HyPE).
 * In:  q [B, N, Hq, d], k [B, N, Hkv, d] (d->dtype); wq, wk [d] fp32.
 * Out: q_norm [B, N, Hq, d] bf16 and k_norm [B, N, Hkv, d] bf16 (RMSNorm,
 *      no RoPE); kbar [B, N/block, Hkv, d] fp32 block means of the
 *      normalised keys (taken before rounding to bf16); idx
 *      [B, Hkv, N/block, width] int32, each row ascending, padded with -1. */
sala_status sala_sparse_select(const sala_sparse_desc* d, const void* q, const void* k,
                               const float* wq, const float* wk, void* q_norm, void* k_norm,
                               float* kbar, int32_t* idx, void* workspace, size_t ws_bytes,
                               void* stream);

/* Split form of sala_sparse_select, for a kv group whose q heads are spread
 * over several callers (head-sharded prefill on several GPUs).
 * sala_sparse_select_begin normalises and writes q_norm, k_norm and kbar as
 * sala_sparse_select does, plus qsum [B, N/block, Hkv, d] fp32: for each kv
 * head, the sum over THIS call's q heads of the block-mean normalised
 * queries.  The callers that share a kv group add their qsum (an
 * all-reduce), and each calls sala_sparse_select_finish with the total; it
 * ranks every query block by <qsum_b, kbar_j> / sqrt(d) and writes idx
 * exactly as sala_sparse_select does (SALA_SELECT_BLOCK_MEAN only; other
 * rules return SALA_ERR_UNSUPPORTED).  No workspace: qsum is the caller's.
 * Called back to back with one caller, the pair equals sala_sparse_select. */
sala_status sala_sparse_select_begin(const sala_sparse_desc* d, const void* q, const void* k,
                                     const float* wq, const float* wk, void* q_norm,
                                     void* k_norm, float* kbar, float* qsum, void* stream);
sala_status sala_sparse_select_finish(const sala_sparse_desc* d, const float* qsum,
                                      const float* kbar, int32_t* idx, void* stream);

/* Allocation-free variant of sala_sparse_select (no counterpart on the
 * pages: it exists for callers, not for the method).  Same arguments and
 * results, minus the workspace: its scratch is a fixed array of
 * SALA_NOALLOC_SCRATCH_BYTES (4 MiB) compiled into the library, which every
 * GPU that loads the library keeps until the process exits.  It serves
 * callers that cannot allocate device memory, e.g. code inside an
 * allocator-free runtime or a memory pool that forbids new allocations.
 *   - Limit: sala_sparse_workspace_size(d) must not exceed the array size
 *     (batch * seqlen/block * kv_heads * head_dim * 4 bytes; 262144 tokens
 *     at batch 1, 2 kv heads, head_dim 128); larger shapes return
 *     SALA_ERR_WORKSPACE and launch nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it; make
 *     that first call before any stream capture on the device.  The cached
 *     address belongs to the device's context as it was then: after
 *     cudaDeviceReset (or anything else that destroys and recreates that
 *     context) the cache is stale, so do not call this entry point again in
 *     a process that reset the device.
 *   - The library calls no cudaMalloc / cudaFree here.
 *   - All calls on one device share the array, so calls that may overlap on
 *     the GPU (different streams without ordering) race and must not be
 *     issued; calls ordered on one stream are safe.  The array keeps the
 *     last call's contents; each call overwrites what it reads. */
#define SALA_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
sala_status sala_sparse_select_noalloc(const sala_sparse_desc* d, const void* q, const void* k,
                                       const float* wq, const float* wk, void* q_norm,
                                       void* k_norm, float* kbar, int32_t* idx, void* stream);

/* Gathered block-sparse attention with the sigmoid gate (acgfav.com
 * article, section "SALA 混合架构": exact attention of each query over its
 * selected key blocks; MiniCPM-SALA paper, summary: an output gate after each
 * attention block).
 * In:  q_norm [B, N, Hq, d] bf16, k_norm [B, N, Hkv, d] bf16 (as written by
 *      sala_sparse_select), v [B, N, Hkv, d] and gate [B, N, Hq, d] of
 *      d->dtype, idx as written by sala_sparse_select (entries >= 0 must be
 *      ascending block numbers <= the row's own block; a row must list at
 *      least one block: an empty row gets a zero output and sets the bounds
 *      bit of the status word).
 * Out: out [B, N, Hq, d] of d->dtype.
 * workspace / ws_bytes: reserved (ignored; may be NULL / 0).  The call needs
 * no scratch today; the arguments keep the signature of the other prefill
 * calls so that a future split of long index lists can use them. */
sala_status sala_sparse_prefill(const sala_sparse_desc* d, const void* q_norm,
                                const void* k_norm, const void* v, const void* gate,
                                const int32_t* idx, void* out, void* workspace,
                                size_t ws_bytes, void* stream);

/* -------------------------------------------------------------- full block */

/* One SALA decoder block around one attention layer, over N tokens (no
 * counterpart in the pages' numbers: it turns the attention-only throughput
 * into a per-block figure of the kind of the pages' time to first token).
 * The pages fix the structure in words (MiniCPM-SALA paper, section 2.1:
 * every attention block is followed by an FFN block; summary: an output gate
 * after each attention block); the rest is the plainest reading for the
 * model family, with synthetic weights:
 *   xn = RMSNorm(x) * norm_attn                     (fp32 math, bf16 out)
 *   q, k, v, gate = xn Wq^T, xn Wk^T, xn Wv^T, xn Wg^T   (bf16, fp32 accum.)
 *   a  = the linear (sala_linear_prefill) or sparse (sala_sparse_select +
 *        sala_sparse_prefill) attention of q, k, v, gate
 *   h  = x + a Wo^T                                  (fp32 residual stream)
 *   hn = RMSNorm(h) * norm_ffn
 *   y  = h + (silu(hn W1^T) * (hn W3^T)) W2^T
 * The GEMMs run in cuBLASLt; norms, SwiGLU and the attention in this
 * library's kernels. */
typedef struct {
  int hidden;        /* residual width = q_heads * head_dim of the attention  */
  int ffn;           /* FFN inner width (a multiple of 8)                     */
  float rms_eps;     /* of the two pre-norms                                  */
} sala_block_desc;

/* bf16 weights use the [out, in] row-major layout of a torch Linear. */
typedef struct {
  const float* norm_attn;   /* [hidden] fp32                                  */
  const void* wq;           /* [Hq*d, hidden] bf16                            */
  const void* wk;           /* [Hk*d, hidden] bf16 (Hk = heads for a linear   */
  const void* wv;           /*   layer, kv_heads for the sparse one)          */
  const void* wg;           /* [Hq*d, hidden] bf16                            */
  const float* qk_norm_q;   /* [d] fp32 QK-RMSNorm weights of the attention   */
  const float* qk_norm_k;   /* [d] fp32                                       */
  const void* wo;           /* [hidden, Hq*d] bf16                            */
  const float* norm_ffn;    /* [hidden] fp32                                  */
  const void* w13;          /* [2*ffn, hidden] bf16: W1 rows, then W3 rows     */
  const void* w2;           /* [hidden, ffn] bf16                             */
} sala_block_weights;

/* Exactly one of lin / sp is non-NULL and names the attention; its dtype
 * must be SALA_BF16 and its seqlen / batch give the tokens. */
size_t sala_block_workspace_size(const sala_block_desc* b, const sala_linear_desc* lin,
                                 const sala_sparse_desc* sp);

/* x, y: [B, N, hidden] fp32 (y must not alias x).  lambda: [H] fp32 for a
 * linear layer (NULL for sparse).  state_out: optional [B, H, d, d] final
 * linear state.  workspace: >= sala_block_workspace_size bytes. */
sala_status sala_block_prefill(const sala_block_desc* b, const sala_linear_desc* lin,
                               const sala_sparse_desc* sp, const sala_block_weights* w,
                               const float* lambda, const float* x, float* y, float* state_out,
                               void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------- decode */

#define SALA_MAX_LAYERS 8

/* One decode token through a layer group of n_linear linear layers followed
 * by one sparse layer (MiniCPM-SALA paper, section 2.1: the linear layers
 * carry a constant-size state; acgfav.com article, section "SALA 混合架构":
 * the sparse layer's KV cache holds no position, so it is appended and
 * scored as is).  lin.seqlen, lin.pos0 and sp.seqlen are ignored: the new
 * token sits at position cur_len. */
typedef struct {
  sala_linear_desc lin;
  sala_sparse_desc sp;
  int n_linear;             /* 1 .. SALA_MAX_LAYERS-1                          */
  int64_t cache_capacity;   /* token rows of k_cache / v_cache per sequence    */
} sala_decode_desc;

/* Per-layer pointers; layers 0..n_linear-1 are linear, layer n_linear is the
 * sparse one.  q, k, v, gate, out: one token, [B, heads, d] of the dtype.
 * lin_state[l]: [B, H, d, d] fp32, read and updated in place.  lambda[l]:
 * [H] fp32.  wq[l], wk[l]: [d] fp32. */
typedef struct {
  const void* q[SALA_MAX_LAYERS];
  const void* k[SALA_MAX_LAYERS];
  const void* v[SALA_MAX_LAYERS];
  const void* gate[SALA_MAX_LAYERS];
  const float* wq[SALA_MAX_LAYERS];
  const float* wk[SALA_MAX_LAYERS];
  const float* lambda[SALA_MAX_LAYERS];
  float* lin_state[SALA_MAX_LAYERS];
  void* out[SALA_MAX_LAYERS];
} sala_decode_io;

size_t sala_decode_workspace_size(const sala_decode_desc* d);

/* The step runs as ONE cooperative kernel launch (its CTAs synchronise
 * through bounded grid barriers), preceded by a memset of the first bytes
 * of the workspace; it can be captured in a CUDA graph.
 * k_cache, v_cache: [B, cache_capacity, Hkv, d] bf16; rows [0, cur_len) hold
 * the normalised keys / raw values of the earlier tokens (the k_norm and v of
 * a prefill).  kbar: [B, cache_capacity/block, Hkv, d] fp32 block means of the
 * complete blocks (kbar of a prefill).  ksum: [B, Hkv, d] fp32 running sum of
 * the normalised keys of the incomplete last block (zeros when cur_len is a
 * multiple of the block).  The call appends row cur_len to the caches, adds
 * to ksum and, when the block completes, writes its kbar row and zeroes
 * ksum.  Requires cur_len < cache_capacity. */
sala_status sala_decode_step(const sala_decode_desc* d, const sala_decode_io* io,
                             void* k_cache, void* v_cache, float* kbar, float* ksum,
                             int64_t cur_len, void* workspace, size_t ws_bytes, void* stream);

/* -------------------------------------------------------------------- misc */

const char* sala_status_string(sala_status s);

/* Synchronises `stream`, then returns and clears the current device's status
 * word: SALA_OK, SALA_ERR_TIMEOUT or SALA_ERR_DEVICE_FAULT. */
sala_status sala_get_device_status(void* stream);

/* Failure-detection self-test (no counterpart on the pages; test support).
 * Launches one single-CTA kernel on `stream` that waits on an mbarrier no
 * thread ever arrives at.  The wait is bounded like every wait in the
 * library (about 2^31 SM cycles, roughly a second); when it runs out the
 * kernel sets the timeout bit of the status word and returns, leaving the
 * context usable.  Returns what sala_get_device_status() then reports
 * (SALA_ERR_TIMEOUT when the bound works) and clears the word, or
 * SALA_ERR_CUDA if the launch fails. */
sala_status sala_selftest_bounded_wait(void* stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int sala_version(void);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all entry points), for launch accounting by callers. */
uint64_t sala_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SALA_H_ */
