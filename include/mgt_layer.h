/*
 * mgt_layer.h -- C ABI of a B200-native (sm_100a) Megatron-style tensor-parallel GPT layer.
 *
 * One pre-LayerNorm GPT block, forward and backward, on one GPU with a *logical* tp_size:
 *
 *   ln1 = LN(x; g1, b1)
 *   qkv = ln1 W_qkv^T + b_qkv        column-parallel: each shard owns whole heads
 *   o   = causal softmax attention per head (scale 1/sqrt(d), softmax in fp32)
 *   h1  = x + b_o + sum_t o_t W_o,t^T     row-parallel: shard partials summed on-device
 *   ln2 = LN(h1; g2, b2)
 *   a   = GeLU(ln2 W1^T + b1)         column-parallel
 *   y   = h1 + b2 + sum_t a_t W2,t^T      row-parallel
 *
 * Variants (launch flags on the trdm.cn page, section 3.3): swiglu = 1 gives the MLP
 * a = silu(gate) * up with [gate | up] = ln2 W1^T + b1 (fc1 has 2*ffn outputs, each shard its
 * own gate and up halves); disable_bias_linear = 1 drops b_qkv, b_o, b1 and b2.
 * sequence_parallel = 1 (the second-brain-czx page's sequence parallelism): x, y, dx, dy and
 * the LayerNorm / residual activations are split along the sequence, shard t owning
 * positions t*s/p .. (t+1)*s/p - 1 of every sequence, laid out shard-major [p][b][s/p][h];
 * the all-gather before QKV / fc1 and the reduce-scatter after out-proj / fc2 are realised
 * as the row order in which the GEMMs read and write those tensors.
 *
 * Sources: the page "Megatron-LM 3D并行原理与万亿参数训练实战指南" (trdm.cn), section 2.1
 * (tensor parallelism: W_q/W_k/W_v split by output columns with x broadcast and no
 * communication; W_o split by input rows with partial outputs summed by AllReduce), section 3.2
 * (LayerNorm statistics global over hidden; hidden and heads divisible by tp_size; softmax in
 * fp32), section 3.3 (GeLU is the default activation); and the page "Megatron-LM：NVIDIA大模型
 * 训练框架" (second-brain-czx), section "张量并行" (ColumnParallelLinear with
 * gather_output=False feeding RowParallelLinear with input_is_parallel=True). The pages give no
 * formulas; the readings taken (LN eps 1e-5 inside the square root with biased variance, exact
 * erf GeLU, biases of row-parallel layers added once after the shard sum, two LNs and two
 * residuals) are documented with the oracle.
 *
 * Conventions
 *   - Row-major everywhere. Weights are nn.Linear style [out, in]; y = x W^T + b.
 *   - Packed per-shard weights (column split = block of output rows, row split = block of
 *     input columns):
 *         w_qkv [p][3][H/p][d][h]   b_qkv [p][3][H/p][d]
 *         w_o   [p][h][h/p]         b_o   [h]
 *         w1    [p][f/p][h]         b1    [p][f/p]
 *         (swiglu: w1 [p][2][f/p][h], b1 [p][2][f/p]: shard t's gate rows, then its up rows)
 *         w2    [p][h][f/p]         b2    [h]
 *         ln1_g, ln1_b, ln2_g, ln2_b [h]
 *   - x, y, dx, dy: [b, s, h], tokens flattened as T = b*s with s fastest (sequence_parallel:
 *     [p][b][s/p][h]; so are the regions ln1, h1, ln2, their statistics, dln2, dh1, dln1).
 *   - dtype MGT_BF16: activations, weights and biases are bf16; LN gamma/beta are fp32.
 *     dtype MGT_F32: everything fp32. All gradients of parameters are written in fp32 and
 *     OVERWRITTEN (not accumulated); dx is in the activation dtype.
 *   - All device pointers are owned by the caller. The handle owns host state (config,
 *     derived sizes) and a few CUDA objects: optional profiling events, and the backward's
 *     second stream with its fork/join events (created by the first mgt_layer_bwd). A handle
 *     binds to the device current at its first fwd/bwd call; a call from another device
 *     returns MGT_EUNSUPPORTED. Calls are asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = legacy default stream).
 *   - The library never allocates device memory. `saved` (written by fwd, read by bwd) and
 *     `workspace` are caller buffers of the sizes mgt_layer_sizes reports, 256-byte aligned.
 *     The first 256 bytes of `workspace` hold the device status word: zero the workspace once
 *     after allocating it; device errors accumulate there until mgt_layer_get_error reads and
 *     clears them.
 *
 * The same block split over real tensor-parallel ranks (one shard per rank, the four shard
 * sums done by a caller-provided all-reduce) is the mgt_tp_rank_* API at the end of this file.
 *
 * Errors: synchronous validation returns MGT_EINVAL / MGT_EUNSUPPORTED without touching the
 * GPU; a failed launch returns MGT_ECUDA; a device-side bounded wait that runs out records
 * MGT_ETIMEOUT in the status word (read by mgt_layer_get_error). Nothing aborts or traps.
 */
#ifndef MGT_LAYER_H
#define MGT_LAYER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mgt_status {
  MGT_OK = 0,
  MGT_EINVAL = 1,        /* bad sizes, null pointers, divisibility (h%p, H%p, h%H, f%p) */
  MGT_EUNSUPPORTED = 2,  /* dtype, head_dim, alignment outside what the kernels implement */
  MGT_ECUDA = 3,         /* a CUDA runtime/driver call or kernel launch failed */
  MGT_ETIMEOUT = 4,      /* a device-side bounded wait gave up (see mgt_layer_get_error) */
  MGT_ENOMEM = 5         /* a caller buffer is smaller than required */
} mgt_status;

typedef enum mgt_dtype { MGT_F32 = 0, MGT_BF16 = 1 } mgt_dtype;

/* Layer shape and numerics. Mirrors TransformerConfig(hidden_size, num_attention_heads,
 * ffn_hidden_size, seq_length) plus micro-batch and the logical tensor-parallel size.
 * Valid: all sizes > 0; hidden % heads == 0; hidden % tp_size == 0; heads % tp_size == 0;
 * ffn % tp_size == 0; head_dim in {64, 128} for bf16, <= 64 for f32; for bf16 also
 * hidden/tp_size and ffn/tp_size multiples of 64. causal must be 1 (the GPT mask);
 * recompute_attn is accepted for either value -- attention probabilities are never stored,
 * the backward always recomputes them from the saved log-sum-exp. swiglu and
 * disable_bias_linear are 0 or 1 (a zero-filled tail keeps the GeLU layer with biases);
 * gelu_tanh has no effect with swiglu. sequence_parallel is 0 or 1 and needs seq % tp_size
 * == 0 and, for bf16, (seq / tp_size) % 128 == 0. */
typedef struct mgt_layer_config {
  int32_t hidden;
  int32_t heads;
  int32_t ffn;
  int32_t seq;
  int32_t micro_batch;
  int32_t tp_size;
  int32_t dtype;          /* mgt_dtype */
  int32_t causal;         /* must be 1 */
  float ln_eps;           /* LayerNorm epsilon, added to the biased variance */
  int32_t recompute_attn; /* informational; see above */
  int32_t gelu_tanh;      /* 0: exact erf GeLU; 1: tanh approximation */
  int32_t swiglu;         /* 0: GeLU MLP; 1: SwiGLU, a = silu(gate) * up (fc1: 2*ffn outputs) */
  int32_t disable_bias_linear; /* 1: no biases in QKV, out-proj, fc1, fc2 (b_* may be NULL) */
  int32_t sequence_parallel;   /* 1: sequence-sharded [p][b][s/p][h] LN/residual regions */
} mgt_layer_config;

/* Parameters (device pointers, packed layouts above). With disable_bias_linear the four b_*
 * pointers are ignored and may be NULL; likewise their gradients. */
typedef struct mgt_layer_params {
  const void *ln1_g, *ln1_b, *w_qkv, *b_qkv, *w_o, *b_o;
  const void *ln2_g, *ln2_b, *w1, *b1, *w2, *b2;
} mgt_layer_params;

/* Parameter gradients (device pointers, fp32, same packed layouts). */
typedef struct mgt_layer_grads {
  void *ln1_g, *ln1_b, *w_qkv, *b_qkv, *w_o, *b_o;
  void *ln2_g, *ln2_b, *w1, *b1, *w2, *b2;
} mgt_layer_grads;

typedef struct mgt_layer mgt_layer; /* opaque handle, host memory only */

/* Validate `cfg` and create a handle. Host only: makes no CUDA call. On error *out = NULL. */
mgt_status mgt_layer_init(const mgt_layer_config* cfg, mgt_layer** out);

/* Bytes the caller must provide for `saved` (fwd -> bwd activations) and `workspace`. */
mgt_status mgt_layer_sizes(const mgt_layer* layer, size_t* saved_bytes, size_t* workspace_bytes);

/* Where each intermediate lives, for inspection and tests. `region` is an mgt_region value;
 * regions below 64 are offsets into `saved`, regions from 64 up are offsets into `workspace`.
 * Element types: ACT = activation dtype, F32 = float. Shapes use T = b*s. */
typedef enum mgt_region {
  MGT_SAVED_LN1 = 0,        /* ACT [T, h]          LN1 output                          */
  MGT_SAVED_LN1_MEAN = 1,   /* F32 [T]                                                 */
  MGT_SAVED_LN1_RSTD = 2,   /* F32 [T]             1/sqrt(var + eps)                   */
  MGT_SAVED_QKV = 3,        /* ACT [T][p][3][H/p][d]                                   */
  MGT_SAVED_ATTN_O = 4,     /* ACT [T][p][H/p][d]  attention output (= [T, h])         */
  MGT_SAVED_ATTN_LSE = 5,   /* F32 [b][H][s]       natural-log sum of exp of scores    */
  MGT_SAVED_H1 = 6,         /* ACT [T, h]          first residual stream               */
  MGT_SAVED_LN2 = 7,        /* ACT [T, h]                                              */
  MGT_SAVED_LN2_MEAN = 8,   /* F32 [T]                                                 */
  MGT_SAVED_LN2_RSTD = 9,   /* F32 [T]                                                 */
  MGT_SAVED_FC1_U = 10,     /* ACT [T][p][f/p]     u, the fc1 pre-activation (bias included);
                               swiglu: ACT [T][p][2][f/p], u = [gate | up]              */
  MGT_SAVED_FC1_A = 11,     /* ACT [T][p][f/p]     GeLU(u) (swiglu: silu(gate) * up)   */
  MGT_SAVED_COUNT = 12,
  MGT_WS_STATUS = 64,       /* int32 device status word (first 256 bytes)              */
  MGT_WS_DU = 65,           /* ACT [T, f]   dL/du (swiglu: [T][p][2][f/p], d gate | d up) */
  MGT_WS_DLN2 = 66,         /* ACT [T, h]   dL/d ln2 (shard contributions summed)      */
  MGT_WS_DH1 = 67,          /* ACT [T, h]   dL/d h1                                    */
  MGT_WS_DO = 68,           /* ACT [T, h]   dL/d attention output                      */
  MGT_WS_DQKV = 69,         /* ACT [T, 3h]  dL/d qkv (packed like qkv)                 */
  MGT_WS_DLN1 = 70,         /* ACT [T, h]   dL/d ln1                                   */
  MGT_WS_ATTN_D = 71,       /* F32 [b][H][s] rowsum(dO * O)                            */
  MGT_WS_DQ_ACC = 72,       /* I32 [T, h]   fixed-point dQ accumulator of the attention
                               backward, then per-head scaling data (bf16 layers with
                               head_dim 128; 0 bytes otherwise)                         */
  MGT_WS_LN_PARTIAL = 73,   /* F32 [slices][3][h] LayerNorm dgamma/dbeta/residual-grad partial sums */
  MGT_WS_COUNT = 74
} mgt_region;
mgt_status mgt_layer_region(const mgt_layer* layer, int region, size_t* offset, size_t* bytes);

/* Forward. Reads x [b,s,h]; writes y [b,s,h] and every region of `saved`.
 * Launch order on `stream`: LN1, QKV GEMM(+bias), attention, out-proj GEMM (+shard sum,
 * +b_o, +x), LN2, fc1 GEMM (+b1, GeLU; stores a and u; swiglu: each tile holds a
 * shard's gate and up columns for the same outputs and stores a and [gate | up]), fc2 GEMM
 * (+shard sum, +b2, +h1). */
mgt_status mgt_layer_fwd(mgt_layer* layer, const mgt_layer_params* params, const void* x,
                         void* y, void* saved, void* workspace, void* stream);

/* Backward. Reads x, saved (from the matching fwd) and dy; writes dx and every gradient in
 * `grads` (fp32, overwritten). Uses `workspace` for intermediate gradients.
 * Ordering: all work is ordered after what `stream` held at the call, and everything the call
 * writes is complete before later work on `stream` runs. Inside, the weight-gradient GEMMs
 * and the bias column sums run on a second stream of the handle (forked from `stream` by
 * events after the launch that produces their inputs, joined back at the end) so that they
 * overlap the data-gradient chain; under stream capture this is a fork/join in the graph.
 * The first call creates that stream and its events on the current device: make it outside
 * a stream capture. With profiling on (mgt_layer_profile) everything runs on `stream`. */
mgt_status mgt_layer_bwd(mgt_layer* layer, const mgt_layer_params* params, const void* x,
                         const void* saved, const void* dy, void* dx, const mgt_layer_grads* grads,
                         void* workspace, void* stream);

/* Synchronise `stream`, read and clear the device status word in `workspace`.
 * Returns MGT_OK, MGT_ETIMEOUT (a bounded wait gave up) or MGT_ECUDA. */
mgt_status mgt_layer_get_error(mgt_layer* layer, void* workspace, void* stream);

/* Per-kernel timing with CUDA events recorded around every launch of this handle
 * (enable = 1 creates the events and needs a GPU; 0 stops recording). */
typedef struct mgt_kernel_stat {
  char name[32];     /* kernel family, e.g. "gemm_tc", "attn_fwd", "ln_fwd"         */
  int64_t launches;  /* launches recorded                                          */
  double ms;         /* summed device time of those launches                       */
  double flops;      /* summed algorithmic FLOPs (dense contractions)              */
  double bytes;      /* summed algorithmic HBM bytes (memory-bound kernels)        */
} mgt_kernel_stat;
mgt_status mgt_layer_profile(mgt_layer* layer, int enable);
/* Synchronises the recorded events, folds them into per-family totals, copies up to `cap`
 * entries to `out`, sets *n, and resets the totals. */
mgt_status mgt_layer_profile_read(mgt_layer* layer, mgt_kernel_stat* out, int cap, int* n);

void mgt_layer_destroy(mgt_layer* layer);
const char* mgt_status_string(mgt_status s);

/* Plain bf16 GEMM on the tensor-core path used inside the layer, exported for unit tests:
 *   C[m, n] = sum_k A(m, k) * B(n, k),  C fp32 row-major with leading dimension ldc.
 * A(m, k) = A[m*lda + k] if a_mn_major == 0, else A[k*lda + m]; likewise B(n, k) with
 * b_mn_major. lda/ldb in elements, multiples of 8; pointers 16-byte aligned; M, N, K >= 1.
 * `status` is an int32 device word (zeroed by the caller) that receives timeout codes. */
mgt_status mgt_gemm_bf16(int32_t M, int32_t N, int32_t K, int32_t a_mn_major,
                         int32_t b_mn_major, const void* A, int64_t lda, const void* B,
                         int64_t ldb, float* C, int64_t ldc, int32_t* status, void* stream);

/* FP8 (e4m3) with per-tensor scaling. The page "把大模型训练“摁”到规模化：NVIDIA Megatron-LM /
 * Megatron Core 上手与理解" (section 0) lists FP8 among Megatron Core's mixed precisions and the
 * trdm.cn page's inference section enables it (--enable-fp8); neither gives a recipe. Here:
 *
 * mgt_fp8_quantize: amax = max |x| over n elements of x (dtype MGT_F32 or MGT_BF16), then
 *   q[i] = e4m3(x[i] * s), s = 448 / amax (1 if amax == 0), rounded to nearest even and
 *   saturated to +-448 (the largest finite e4m3); scales (device, 2 floats) receives
 *   {amax, amax / 448} (the second, 1 if amax == 0, is the dequantisation factor). q: n bytes,
 *   2-byte aligned. Asynchronous on `stream`; MGT_EINVAL for n < 1 or null pointers.
 *
 * mgt_gemm_fp8: C[m, n] = (sum_k A[m*lda + k] * B[n*ldb + k]) * a_scales[1] * b_scales[1]
 *   with A [M][K], B [N][K] e4m3 bytes (both K-major), products accumulated in fp32 on the
 *   tensor cores (tcgen05 kind::f8f6f4); C row-major with leading dimension ldc in c_dtype
 *   (MGT_F32 or MGT_BF16, round to nearest even). K, lda, ldb multiples of 16; ldc a
 *   multiple of 4 (f32) or 8 (bf16); pointers 16-byte aligned; `status` an int32 device word
 *   (zeroed by the caller) that receives timeout codes. MGT_EUNSUPPORTED when the alignment
 *   rules fail. */
mgt_status mgt_fp8_quantize(int32_t dtype, int64_t n, const void* x, uint8_t* q, float* scales,
                            void* stream);
mgt_status mgt_gemm_fp8(int32_t M, int32_t N, int32_t K, const uint8_t* A, int64_t lda,
                        const uint8_t* B, int64_t ldb, const float* a_scales,
                        const float* b_scales, void* C, int32_t c_dtype, int64_t ldc,
                        int32_t* status, void* stream);

/* Failure-path probe (diagnostics and tests; no counterpart in the pages). Launches one thread
 * that waits on a device barrier nothing ever arrives on, through the same bounded wait that
 * every pipelined kernel of this library uses; after limit_ns (0 < limit_ns <= 1e9) it gives
 * up, records a non-zero code in the int32 device word `status` and returns. Demonstrates that a
 * device wait which runs out ends in a readable status, not a hang or trap, and that the context
 * stays usable. Point `status` at a layer's status word (mgt_layer_status_word) to make
 * mgt_layer_get_error report MGT_ETIMEOUT. */
mgt_status mgt_debug_bounded_wait(int64_t limit_ns, int32_t* status, void* stream);

/* Numerics probe (tests; no counterpart in the pages): y[i] = 2^x[i] for n floats: path 0 =
 * the hardware approximation (ex2.approx) that the attention kernels use for the softmax
 * probabilities, path 1 = an alternative polynomial evaluated on the FMA pipe (relative
 * error below 7.5e-5 for -125 <= x <= 127; inputs below -125 give 2^-125), which the kernels
 * do not use because it made none of their loops faster on B200. x, y device
 * pointers; asynchronous on `stream`; MGT_EINVAL for n < 0, null pointers or another path. */
mgt_status mgt_debug_exp2(int32_t path, int64_t n, const float* x, float* y, void* stream);

/* Device address of the status word inside `workspace` (the first bytes of the workspace). */
mgt_status mgt_layer_status_word(mgt_layer* layer, void* workspace, int32_t** word);

/* LayerNorm backward that allocates nothing -- the pages have no counterpart; it exists for
 * callers that cannot call cudaMalloc where they run the backward (frameworks that own all
 * device memory through their own pool allocator, hot loops where an allocation would
 * synchronise the device). Computes, for `rows` rows of width h,
 *   dx = dres + rstd * (g - mean(g) - xhat * mean(g * xhat)),  g = dy * gamma,
 *   dgamma = sum_rows dy * xhat,  dbeta = sum_rows dy,  xhat = (x - mean) * rstd,
 * i.e. the LayerNorm backward of mgt_layer_bwd. dtype: MGT_BF16 (dy, dres, x, dx bf16) or
 * MGT_F32; gamma, mean, rstd, dgamma, dbeta fp32. dres may be NULL. h must be a multiple of 8
 * (bf16) or 4 (f32) and at most 16384 (bf16) / 8192 (f32), else MGT_EUNSUPPORTED.
 * Alignment: dy, dres, x, dx and gamma 16-byte aligned; mean, rstd, dgamma, dbeta 4-byte
 * aligned; otherwise MGT_EUNSUPPORTED before anything is launched.
 * Its per-block partial sums live in a fixed 4 MiB array of the library's own device memory,
 * held on every GPU that loads the library until the process exits. The first call on each
 * device looks up that array's device address (cudaGetSymbolAddress) and keeps it for the
 * life of the process: make that first call before any stream capture, and do not reset the
 * device (cudaDeviceReset) after it. All calls share the array: calls that overlap on the GPU
 * (other streams, other threads) race on it, so serialise them. The kernels it launches wait
 * on nothing on the device, so there is no timeout to report. Allocates no memory. */
mgt_status mgt_layernorm_bwd_noalloc(int32_t dtype, int64_t rows, int32_t h, const void* dy,
                                     const void* dres, const void* x, const float* gamma,
                                     const float* mean, const float* rstd, void* dx,
                                     float* dgamma, float* dbeta, void* stream);

/* ---------------------------------------------------------------------------------------
 * One rank of a real tensor-parallel group. The page "Megatron-LM 3D并行原理与万亿参数训练实战指南"
 * (trdm.cn), section 2.1, sums the row-parallel layers' partial outputs across the ranks with
 * an AllReduce; the backward's two reductions (the gradients of the replicated inputs of the
 * column-parallel layers) are its adjoint. A rank holds shard `rank` of the packed parameters:
 * w_qkv [3][H/p][d][h], b_qkv [3][H/p][d], w_o [h][h/p], w1 [f/p][h] (swiglu: [2][f/p][h]),
 * b1 [f/p] ([2][f/p]), w2 [h][f/p], and ln1_g, ln1_b, b_o, ln2_g, ln2_b, b2 whole; gradients
 * have the same shapes (fp32). x, dy are the whole [b, s, h] on every rank; y, dx come out
 * whole on every rank.
 *
 * The caller provides the reduction: `allreduce(buf, count, user, stream)` must replace the
 * `count` fp32 values at device address `buf` by their sum over all ranks, ordered on
 * `stream` (work already on `stream` has produced this rank's values; work enqueued after the
 * callback returns reads the sum), and return MGT_OK. It is called 2 times per forward
 * (out-proj and fc2 partials) and 2 times per backward (dln2 and dln1 contributions) --
 * once per row band with mgt_tp_rank_set_bands -- always inside the workspace region reported
 * by mgt_tp_rank_partial, in the same order on every rank. bf16 layers only; sequence
 * parallelism is not supported here (MGT_EUNSUPPORTED). Everything runs on `stream`, except
 * the banded exchanges (below). */
typedef mgt_status (*mgt_allreduce_fn)(float* buf, int64_t count, void* user, void* stream);
typedef struct mgt_tp_rank mgt_tp_rank; /* opaque handle, host memory only */

/* Validate `cfg` (as mgt_layer_init) and 0 <= rank < tp_size; create the rank's handle.
 * Host only. */
mgt_status mgt_tp_rank_init(const mgt_layer_config* cfg, int32_t rank, mgt_tp_rank** out);
mgt_status mgt_tp_rank_sizes(const mgt_tp_rank* r, size_t* saved_bytes, size_t* workspace_bytes);
/* Offset and size in `workspace` of the fp32 [T, h] buffer the reductions run on. */
mgt_status mgt_tp_rank_partial(const mgt_tp_rank* r, size_t* offset, size_t* bytes);
/* Row bands of each shard sum (1 <= bands <= 16; default 1; MGT_EINVAL otherwise). With one
 * band, the callback gets the whole [T, h] partial once per sum, on `stream`, after the
 * partial GEMM (and, in the backward, after the weight-gradient GEMM enqueued behind it).
 * With more, the partial GEMM runs over consecutive row bands (an even split of T rounded up
 * to multiples of 128 rows) and the callback is made once per band, right after that band's
 * GEMM is enqueued, with `buf` = the band's first row of the partial buffer, `count` = its
 * rows * h, and `stream` = the rank's communication stream (created by the first such call on
 * the bound device): work enqueued there runs after the band's partial is written, and
 * `stream` waits for every band's exchange before the sum is used. An asynchronous collective
 * (NCCL) therefore exchanges band i while band i+1 is being computed -- the overlap of
 * communication with the row-parallel GEMM (--tp-comm-overlap on the vampireachao.github.io
 * page). Every rank must use the same number of bands. */
mgt_status mgt_tp_rank_set_bands(mgt_tp_rank* r, int32_t bands);
mgt_status mgt_tp_rank_fwd(mgt_tp_rank* r, const mgt_layer_params* shard, const void* x, void* y,
                           void* saved, void* workspace, mgt_allreduce_fn allreduce, void* user,
                           void* stream);
mgt_status mgt_tp_rank_bwd(mgt_tp_rank* r, const mgt_layer_params* shard, const void* x,
                           const void* saved, const void* dy, void* dx,
                           const mgt_layer_grads* grads, void* workspace,
                           mgt_allreduce_fn allreduce, void* user, void* stream);
void mgt_tp_rank_destroy(mgt_tp_rank* r);

#ifdef __cplusplus
}
#endif
#endif /* MGT_LAYER_H */
