// Internal declarations shared by the kernel translation units and the C-ABI host code.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace mgt {

// Kernel launch, with programmatic stream serialization when `programmatic`: the kernel's CTAs
// may then be scheduled as soon as the previous kernel of `s` has no CTA left, while that
// grid completes and flushes its writes, run their set-up, and wait inside the kernel
// (grid_dependency_wait) for that kernel's results. Only kernels that call
// grid_dependency_wait before touching global memory may be launched this way. A launch whose
// stream predecessor produces none of its inputs (a weight gradient on the backward's second
// stream) stays plain.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(bool programmatic, void (*kern)(KArgs...), dim3 grid,
                                 dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = programmatic ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Device status codes written into the caller's status word (first failure wins).
enum DeviceError : int {
  kErrNone = 0,
  kErrTimeoutProducer = 0x100,  // TMA producer waited too long for a free stage
  kErrTimeoutMma = 0x101,       // MMA issuer waited too long for data or a free accumulator
  kErrTimeoutEpilogue = 0x102,  // epilogue waited too long for an accumulator
  kErrTimeoutDrain = 0x103,     // unwinding after a timeout waited too long
  kErrTimeoutAttn = 0x110,
  kErrTimeoutLn = 0x120,        // a LayerNorm row ring waited too long for a bulk copy
  kErrTimeoutProbe = 0x1F0,     // the bounded-wait probe (mgt_debug_bounded_wait) gave up
};

// Epilogue applied to each fp32 accumulator tile of the GEMM.
enum Epilogue : int {
  kEpiStoreF32 = 0,  // out (fp32) = acc                     (weight gradients)
  kEpiBf16 = 1,      // out (act) = acc [+ bias] [+ residual] (QKV, out-proj, fc2, dgrads)
  kEpiGelu = 2,      // u = acc + bias; out = GeLU(u), out2 = u (fc1)
  kEpiDGelu = 3,     // out = acc * GeLU'(aux), aux = u        (fc2 dgrad -> du)
  // SwiGLU fc1 (GLU tiles): group ng holds Ng outputs; B rows ng*2Ng + n (gate) and
  // ng*2Ng + Ng + n (up) feed output (m, ng*Ng + n). out[m*ldc + ng*Ng + n] = silu(g) * u;
  // out2[m*ldc2 + ng*2Ng + n] = g, out2[... + Ng] = u (g, u include the bias, indexed like
  // the B rows). Pair kernel only, K-major operands.
  kEpiSwiglu = 4,
  // SwiGLU backward on the fc2 dgrad: acc = dA(m, ng*Ng + n); aux = [g | u] as stored above
  // (row stride ld_aux); out[m*ldc + ng*2Ng + n] = dA * u * silu'(g), out[... + Ng] =
  // dA * silu(g).
  kEpiDSwiglu = 5,
};

// One GEMM  C[m, col] = sum_{kg < KG} sum_{kk < Kg} A(m, kg, kk) * B(ng, n, kg, kk)
// over tiles (ng < NG, m < M, n < Ng), col = ng*Ng + n. Operands are described by 3-D TMA
// tensor maps built on the host (bf16 path) or by strides (fp32 SIMT path):
//   A K-major : A[m*lda + kg*Kg + kk]              tensor map dims {Kg, KG, M}
//   A M-major : A[(kg*Kg + kk)*lda + m]            tensor map dims {M, Kg*KG, 1}
//   B K-major : B[kg*b_kgs + n*ldb + kk]           tensor map dims {Kg, Ng, KG}
//   B N-major : B[ng*b_ngs + (kg*Kg + kk)*ldb + n] tensor map dims {Ng, Kg*KG, NG}
// Output element (m, col) lives at out[(col / out_ng) * out_gs + m * ldc + col % out_ng].
struct GemmArgs {
  int M, Ng, NG, Kg, KG;
  int a_mn, b_mn;                       // operand majorness (0 = K-major)
  // SIMT path only (fp32): raw operand pointers and strides in elements.
  const void* A; long long lda;
  const void* B; long long ldb, b_kgs, b_ngs;
  // Epilogue.
  int epi;
  void* out; long long ldc; int out_ng; long long out_gs;
  void* out2;                           // kEpiGelu: u (same addressing as out)
  long long ldc2;                       // kEpiSwiglu: row stride of out2
  const void* bias;                     // indexed by col; nullable
  const void* res; long long ldr;       // residual, res[m*ldr + col]; nullable
  const void* aux; long long ld_aux;    // kEpiDGelu: u[m*ld_aux + col]
  int gelu_tanh;
  int* err;                             // device status word
  // Sequence-parallel layout: token m (= batch * seq + position) of an operand or output held
  // shard-major lives at row seq_row(m) (see below). a_sp / b_sp remap A's / B's token
  // coordinate (M of a K-major A; K of an MN-major A or B), out_sp the output rows and the
  // residual rows read with them. Needs the shard length a multiple of 128.
  int a_sp, b_sp, out_sp;
  int sp_seq, sp_len, sp_b;             // sequence length, positions per shard, micro-batch
  // FP8 (f8 = 1): A and B are e4m3 bytes, both K-major; the accumulator is multiplied by
  // (*a_scale) * (*b_scale) (device scalars: the operands' dequantisation factors) before the
  // epilogue. Only kEpiStoreF32 and kEpiBf16, one group, no K groups.
  int f8;
  const float* a_scale;
  const float* b_scale;
  // Tile order (set by the launcher): 1 = N fastest within a group, 0 = M fastest.
  int n_fast;
  // 1: plain launch; 0: programmatic stream serialization (see launch_kernel)
  int plain_launch;
};


// Row of token m in the sequence-parallel layout [p][b][s/p]: shard t = pos / (s/p) owns
// positions t*s/p .. of every sequence.
__host__ __device__ __forceinline__ int seq_row(const GemmArgs& a, int m) {
  const int bb = m / a.sp_seq, pos = m - bb * a.sp_seq;
  const int t = pos / a.sp_len;
  return (t * a.sp_b + bb) * a.sp_len + (pos - t * a.sp_len);
}

// seq_row along one sweep of a token coordinate k (K of an MN-major operand): a shard chunk
// of sp_len consecutive tokens lies in one sequence and one shard, so seq_row(k) - k is
// constant over it and one division per chunk replaces two per k step. `end` starts at 0.
struct SeqCursor {
  int end, off;
  __host__ __device__ __forceinline__ int row(const GemmArgs& a, int k) {
    if (k >= end || k < end - a.sp_len) {
      off = seq_row(a, k) - k;
      end = (k / a.sp_len + 1) * a.sp_len;
    }
    return k + off;
  }
};

// 3-D bf16 tensor map (128-byte swizzle, zero fill out of bounds); strides in elements.
bool make_tensor_map_bf16_3d(CUtensorMap* m, const void* base, const uint64_t dims[3],
                             const uint64_t strides[2], const uint32_t box[3]);
// 3-D int32 tensor map without swizzle (row-major boxes); strides in elements.
bool make_tensor_map_i32_3d(CUtensorMap* m, const void* base, const uint64_t dims[3],
                            const uint64_t strides[2], const uint32_t box[3]);

// tcgen05 / TMA GEMM for bf16 operands (fp32 accumulate in tensor memory).
// Builds the tensor maps from the pointers in `args` (A, B, strides) and launches a persistent
// kernel with one CTA per SM. Returns a CUDA error code.
cudaError_t launch_gemm_tc(const GemmArgs& args, int num_sms, cudaStream_t stream);
// The FP8 path of the CTA-pair kernel (args.f8 semantics; e4m3 A [M][K], B [N][K]).
cudaError_t launch_gemm_fp8(const GemmArgs& args, int num_sms, cudaStream_t stream);
// Plain FFMA GEMM with the same semantics for fp32 operands.
cudaError_t launch_gemm_simt_f32(const GemmArgs& args, cudaStream_t stream);

// LayerNorm over the last dimension. dtype: 0 fp32, 1 bf16 (x, y); stats and params fp32.
// err: device status word for bounded-wait timeouts (may be null).
cudaError_t launch_ln_fwd(int dtype, long long rows, int h, float eps, const void* x,
                          const float* gamma, const float* beta, void* y, float* mean,
                          float* rstd, int* err, cudaStream_t stream);
// dx = dres + LN'^T(dy); dgamma, dbeta and (if dres_sum and dres are given) dres_sum =
// sum over rows of dres, through per-slice partials in `partial`, which must hold
// nblk * (dres_sum ? 3 : 2) * h floats; at most nblk slices are used.
int ln_bwd_blocks(long long rows, int num_sms);
cudaError_t launch_ln_bwd(int dtype, long long rows, int h, const void* dy, const void* dres,
                          const void* x, const float* gamma, const float* mean,
                          const float* rstd, void* dx, float* partial, int nblk,
                          float* dgamma, float* dbeta, float* dres_sum, int* err,
                          cudaStream_t stream);

// FP8 quantisation with a per-tensor scale: amax = max |x| over n elements (dtype 0 fp32,
// 1 bf16), then q = e4m3(x * 448 / amax) with round-to-nearest-even and saturation, and
// scale_out = {amax, amax / 448} (the second is the dequantisation factor).
cudaError_t launch_fp8_quantize(int dtype, long long n, const void* x, uint8_t* q,
                                float* scale_out, cudaStream_t stream);

// Device-side failure-path probe (see mgt_debug_bounded_wait).
// y[i] = 2^x[i] through the attention kernels' exponential: path 0 the special-function unit
// (ex2.approx), path 1 the polynomial on the FMA pipe (exp2_poly_pair), pairs (i, i+1).
cudaError_t launch_exp2_probe(int path, long long n, const float* x, float* y,
                              cudaStream_t stream);
cudaError_t launch_bounded_wait_probe(int* status, unsigned long long limit_ns,
                                      cudaStream_t stream);

// Column sums of a [rows, cols] activation matrix into fp32 (bias gradients), deterministic
// (fixed-order additions; one launch, no scratch memory).
cudaError_t launch_colsum(int dtype, long long rows, int cols, const void* x, float* out,
                          bool programmatic,
                          cudaStream_t stream);

// Causal attention over packed qkv [T][p][3][H/p][d]; O [T][p][H/p][d]; lse [b][H][s].
struct AttnArgs {
  int b, s, H, d, p;
  const void* qkv; void* o; float* lse;
  const void* dO; float* Dsum; void* dqkv;
  int* err;
  // Single-kernel backward (head_dim 128; null dq_fix selects the two-kernel backward):
  //   dq_fix   int32 [T][H][d]: dQ accumulated in fixed point (integer adds are associative,
  //            so the sum does not depend on the order in which key blocks arrive)
  //   dq_bound float [b*H][4*ceil(s/128)][3]: per 32-token chunk, max |K|, max |V row|^2,
  //            max |dO row|^2, from which every partial sum of dQ is bounded
  //   dq_exp   int32 [b*H]: the power of two that scales each head's dQ to fixed point
  //   dq_stat  float [b*H][2][ceil(s/128)*128]: -lse*log2(e) and -D per query, padded past s
  //            with -inf and 0 (the softmax reads them as they are, no bounds checks)
  int32_t* dq_fix;
  float* dq_bound;
  int32_t* dq_exp;
  float* dq_stat;
};
// Bytes of the single-kernel backward's dQ scratch (dq_fix, dq_exp, dq_bound) and where each
// part starts, for b sequences of s tokens, H heads of 128.
struct DqScratch {
  size_t fix_off, exp_off, bound_off, stat_off, bytes;
};
inline DqScratch dq_scratch_layout(long long b, long long s, long long H) {
  DqScratch r;
  const long long nchunk = (s + 127) / 128;
  r.fix_off = 0;
  r.exp_off = (size_t)b * s * H * 128 * 4;
  r.bound_off = r.exp_off + (((size_t)b * H * 4 + 255) / 256) * 256;
  r.stat_off = r.bound_off + (((size_t)b * H * nchunk * 4 * 3 * 4 + 255) / 256) * 256;
  r.bytes = r.stat_off + (size_t)b * H * 2 * nchunk * 128 * 4;
  return r;
}
cudaError_t launch_attn_fwd(int dtype, const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_attn_fwd_tc(const AttnArgs& a, cudaStream_t stream);  // bf16, d in {64, 128}
// bf16 backward on tcgen05. With a.dq_fix (head_dim 128): D = rowsum(dO * O), the bounds of
// dQ and a zeroed fixed-point dQ accumulator, then one key-stationary kernel computing dK, dV
// and adding dQ, then the dQ conversion to bf16. Otherwise: dQ kernel (which also writes
// a.Dsum) then dK/dV kernel.
cudaError_t launch_attn_bwd_tc(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_attn_bwd(int dtype, const AttnArgs& a, cudaStream_t stream);

}  // namespace mgt
