// One tensor-parallel rank of the layer: the rank holds shard `rank` of the packed parameters
// and computes only that shard; the four shard sums of the layer are all-reduces that the
// caller provides as a callback (NCCL, or a test harness). The page "Megatron-LM
// 3D并行原理与万亿参数训练实战指南" (trdm.cn), section 2.1, places the AllReduce after the
// row-parallel layer (out-proj and fc2 partial outputs); the backward's two (the dln2 and
// dln1 contributions of the column-parallel layers, whose input is replicated) are its
// adjoint.
//
// Per reduction: the partial GEMM writes fp32 [T, h] into the workspace, the callback sums
// it over the ranks in place (ordered on the stream), and a small kernel adds the bias and
// the residual (forward) or casts to the activation type (backward). With row bands
// (mgt_tp_rank_set_bands) the partial GEMM runs band by band and each band is handed to the
// callback on a communication stream as soon as its GEMM is enqueued, so the exchange of one
// band overlaps the GEMM of the next (the page's --tp-comm-overlap). Everything else reuses
// the single-GPU kernels with one shard: H/p heads, f/p MLP columns.
#include <cstring>
#include <new>

#include "mgt_device.cuh"
#include "mgt_internal.h"
#include "mgt_layer.h"

namespace mgt {
namespace {

constexpr int kMaxLnSlices = 148;  // LayerNorm backward partial rows (one block per SM)
constexpr int kMaxBands = 16;      // row bands per shard sum

// out[i] = bf16(part[i] + bias[i % h] + res[i]); bias and res may be null. Eight elements per
// thread step (h is a multiple of 8, every pointer 16-byte aligned).
__global__ void __launch_bounds__(256) sum_epilogue_kernel(long long n8, int h,
                                                           const float* __restrict__ part,
                                                           const __nv_bfloat16* __restrict__ bias,
                                                           const __nv_bfloat16* __restrict__ res,
                                                           __nv_bfloat16* __restrict__ out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 p0 = reinterpret_cast<const float4*>(part)[2 * i];
    const float4 p1 = reinterpret_cast<const float4*>(part)[2 * i + 1];
    float v[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    if (bias) {
      const uint4 bw = reinterpret_cast<const uint4*>(bias)[(i * 8 % h) / 8];
      const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] += bf16_lo(bb[j]);
        v[2 * j + 1] += bf16_hi(bb[j]);
      }
    }
    if (res) {
      const uint4 rw = reinterpret_cast<const uint4*>(res)[i];
      const uint32_t rr[4] = {rw.x, rw.y, rw.z, rw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] += bf16_lo(rr[j]);
        v[2 * j + 1] += bf16_hi(rr[j]);
      }
    }
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    reinterpret_cast<uint4*>(out)[i] = w;
  }
}

cudaError_t sum_epilogue(long long n, int h, const float* part, const void* bias,
                         const void* res, void* out, int num_sms, cudaStream_t s) {
  const long long n8 = n / 8;
  long long blocks = (n8 + 255) / 256;
  if (blocks > 8LL * num_sms) blocks = 8LL * num_sms;
  sum_epilogue_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      n8, h, part, reinterpret_cast<const __nv_bfloat16*>(bias),
      reinterpret_cast<const __nv_bfloat16*>(res), reinterpret_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

struct Reg {
  size_t off, bytes;
};

enum SavedReg { S_LN1, S_MU1, S_RS1, S_QKV, S_O, S_LSE, S_H1, S_LN2, S_MU2, S_RS2, S_AUX, S_A,
                S_COUNT };
enum WsReg { W_STATUS, W_PART, W_DU, W_DLN2, W_DH1, W_DO, W_DQKV, W_DLN1, W_D, W_LNP,
             W_DQACC, W_COUNT };

GemmArgs base(int M, int N, int K) {
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = M; a.Ng = N; a.NG = 1; a.Kg = K; a.KG = 1;
  a.out_ng = N;
  return a;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace mgt

using namespace mgt;

struct mgt_tp_rank {
  mgt_layer_config cfg;
  int rank, T, h, H, d, p, hl, Hl, fl, f1l, nblk;
  Reg saved[S_COUNT], ws[W_COUNT];
  size_t saved_bytes = 0, ws_bytes = 0;
  int num_sms = 0;
  int device = -1;
  // Row bands of each shard sum (1: one exchange after the whole partial GEMM, on the
  // caller's stream). With more, the exchanges run on `comm`, each ordered after its band's
  // GEMM by ev_ready[i]; ev_done joins the last one back into the caller's stream.
  int bands = 1;
  cudaStream_t comm = nullptr;
  cudaEvent_t ev_ready[kMaxBands] = {};
  cudaEvent_t ev_done = nullptr;
};

namespace {

void place(Reg* r, int n, const size_t* bytes, size_t* total) {
  size_t off = 0;
  for (int i = 0; i < n; ++i) {
    r[i].off = off;
    r[i].bytes = bytes[i];
    off += (bytes[i] + 255) / 256 * 256;
  }
  *total = off;
}

char* at(void* base, const Reg& r) { return static_cast<char*>(base) + r.off; }
const char* at(const void* base, const Reg& r) { return static_cast<const char*>(base) + r.off; }

// bound to the device current at the first call, like the layer handle
mgt_status ensure(mgt_tp_rank* R) {
  int dev = 0, n = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MGT_ECUDA;
  if (R->num_sms > 0) return dev == R->device ? MGT_OK : MGT_EUNSUPPORTED;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return MGT_ECUDA;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return MGT_EUNSUPPORTED;
  R->num_sms = n;
  R->device = dev;
  return MGT_OK;
}

// Shard parameter (or gradient) pointers: every one set and 16-byte aligned, the four linear
// biases excepted without them.
mgt_status check_ptrs(const mgt_tp_rank* R, const void* const* q) {
  for (int i = 0; i < 12; ++i) {
    const bool is_bias = i == 3 || i == 5 || i == 9 || i == 11;
    if (is_bias && R->cfg.disable_bias_linear) continue;
    if (!q[i]) return MGT_EINVAL;
    if (!al16(q[i])) return MGT_EUNSUPPORTED;
  }
  return MGT_OK;
}

#define TP_TRY(expr)                              \
  do {                                            \
    cudaError_t _e = (expr);                      \
    if (_e != cudaSuccess) return MGT_ECUDA;      \
  } while (0)
#define TP_TRY_ST(expr)                           \
  do {                                            \
    mgt_status _s = (expr);                       \
    if (_s != MGT_OK) return _s;                  \
  } while (0)

// The communication stream and its events, created on the first banded call on the bound
// device; on a failure everything created so far is released and the next call tries again.
cudaError_t ensure_comm(mgt_tp_rank* R) {
  if (R->comm) return cudaSuccess;
  cudaStream_t comm = nullptr;
  cudaEvent_t ev[kMaxBands + 1] = {};
  cudaError_t e = cudaStreamCreateWithFlags(&comm, cudaStreamNonBlocking);
  for (int i = 0; i <= kMaxBands && e == cudaSuccess; ++i)
    e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
  if (e != cudaSuccess) {
    for (auto& x : ev)
      if (x) cudaEventDestroy(x);
    if (comm) cudaStreamDestroy(comm);
    return e;
  }
  for (int i = 0; i < kMaxBands; ++i) R->ev_ready[i] = ev[i];
  R->ev_done = ev[kMaxBands];
  R->comm = comm;
  return cudaSuccess;
}

// Rows per band: an even split of T rounded up to whole 128-row tiles.
int band_rows(const mgt_tp_rank* R) {
  const int per = (R->T + R->bands - 1) / R->bands;
  return (per + 127) / 128 * 128;
}

// First half of a shard sum. `a` is the partial GEMM over all T rows (K-major A at `A` with
// `lda` elements per row, fp32 output `part` [T, h]). One band: the GEMM only (the exchange
// follows in reduce_end, on the caller's stream). Several bands: each band's GEMM, then that
// band's exchange on the communication stream, ordered after the GEMM by an event, so band
// i's exchange overlaps band i+1's GEMM.
mgt_status reduce_begin(mgt_tp_rank* R, GemmArgs a, const void* A, long long lda, float* part,
                        mgt_allreduce_fn allreduce, void* user, cudaStream_t s) {
  if (R->bands == 1) {
    a.A = A;
    a.out = part;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
    return MGT_OK;
  }
  TP_TRY(ensure_comm(R));
  const int per = band_rows(R);
  for (int i = 0, r0 = 0; r0 < R->T; ++i, r0 += per) {
    const int rows = R->T - r0 < per ? R->T - r0 : per;
    GemmArgs b = a;
    b.M = rows;
    b.A = static_cast<const __nv_bfloat16*>(A) + (long long)r0 * lda;
    b.out = part + (long long)r0 * R->h;
    TP_TRY(launch_gemm_tc(b, R->num_sms, s));
    TP_TRY(cudaEventRecord(R->ev_ready[i], s));
    TP_TRY(cudaStreamWaitEvent(R->comm, R->ev_ready[i], 0));
    TP_TRY_ST(allreduce(part + (long long)r0 * R->h, (int64_t)rows * R->h, user, R->comm));
  }
  return MGT_OK;
}

// Second half: one band -- the exchange of the whole partial on the caller's stream; several
// -- the caller's stream waits for the last band's exchange (the communication stream runs
// them in order).
mgt_status reduce_end(mgt_tp_rank* R, float* part, mgt_allreduce_fn allreduce, void* user,
                      cudaStream_t s) {
  if (R->bands == 1) {
    TP_TRY_ST(allreduce(part, (int64_t)R->T * R->h, user, s));
    return MGT_OK;
  }
  TP_TRY(cudaEventRecord(R->ev_done, R->comm));
  TP_TRY(cudaStreamWaitEvent(s, R->ev_done, 0));
  return MGT_OK;
}

}  // namespace

extern "C" {

mgt_status mgt_tp_rank_set_bands(mgt_tp_rank* R, int32_t bands) {
  if (!R || bands < 1 || bands > kMaxBands) return MGT_EINVAL;
  R->bands = bands;
  return MGT_OK;
}

mgt_status mgt_tp_rank_init(const mgt_layer_config* cfg, int32_t rank, mgt_tp_rank** out) {
  if (!out) return MGT_EINVAL;
  *out = nullptr;
  if (!cfg) return MGT_EINVAL;
  // the whole layer's configuration must be valid on its own
  mgt_layer* tmp = nullptr;
  mgt_status st = mgt_layer_init(cfg, &tmp);
  if (st != MGT_OK) return st;
  mgt_layer_destroy(tmp);
  if (rank < 0 || rank >= cfg->tp_size) return MGT_EINVAL;
  if (cfg->dtype != MGT_BF16 || cfg->sequence_parallel) return MGT_EUNSUPPORTED;
  mgt_tp_rank* R = new (std::nothrow) mgt_tp_rank();
  if (!R) return MGT_ENOMEM;
  R->cfg = *cfg;
  R->rank = rank;
  R->T = cfg->seq * cfg->micro_batch;
  R->h = cfg->hidden;
  R->H = cfg->heads;
  R->d = cfg->hidden / cfg->heads;
  R->p = cfg->tp_size;
  R->hl = cfg->hidden / cfg->tp_size;
  R->Hl = cfg->heads / cfg->tp_size;
  R->fl = cfg->ffn / cfg->tp_size;
  R->f1l = (cfg->swiglu ? 2 : 1) * R->fl;
  R->nblk = R->T < kMaxLnSlices ? R->T : kMaxLnSlices;
  const size_t T = R->T, h = R->h, e = 2;
  const size_t lse = (size_t)cfg->micro_batch * R->Hl * cfg->seq * 4;
  const size_t sb[S_COUNT] = {T * h * e, T * 4, T * 4, T * 3 * R->hl * e, T * R->hl * e, lse,
                              T * h * e, T * h * e, T * 4, T * 4, T * R->f1l * e,
                              T * R->fl * e};
  const size_t wb[W_COUNT] = {256, T * h * 4, T * R->f1l * e, T * h * e, T * h * e,
                              T * R->hl * e, T * 3 * R->hl * e, T * h * e, lse,
                              (size_t)R->nblk * 3 * h * 4,
                              // fixed-point dQ accumulator and its scaling data
                              R->d == 128 ? dq_scratch_layout(cfg->micro_batch, cfg->seq,
                                                              R->Hl).bytes
                                          : 0};
  place(R->saved, S_COUNT, sb, &R->saved_bytes);
  place(R->ws, W_COUNT, wb, &R->ws_bytes);
  *out = R;
  return MGT_OK;
}

mgt_status mgt_tp_rank_sizes(const mgt_tp_rank* R, size_t* saved_bytes, size_t* workspace_bytes) {
  if (!R) return MGT_EINVAL;
  if (saved_bytes) *saved_bytes = R->saved_bytes;
  if (workspace_bytes) *workspace_bytes = R->ws_bytes;
  return MGT_OK;
}

mgt_status mgt_tp_rank_partial(const mgt_tp_rank* R, size_t* offset, size_t* bytes) {
  if (!R) return MGT_EINVAL;
  if (offset) *offset = R->ws[W_PART].off;
  if (bytes) *bytes = R->ws[W_PART].bytes;
  return MGT_OK;
}

void mgt_tp_rank_destroy(mgt_tp_rank* R) {
  if (!R) return;
  if (R->comm) {
    cudaStreamSynchronize(R->comm);
    for (auto& e : R->ev_ready)
      if (e) cudaEventDestroy(e);
    if (R->ev_done) cudaEventDestroy(R->ev_done);
    cudaStreamDestroy(R->comm);
  }
  delete R;
}

mgt_status mgt_tp_rank_fwd(mgt_tp_rank* R, const mgt_layer_params* P, const void* x, void* y,
                           void* saved, void* workspace, mgt_allreduce_fn allreduce, void* user,
                           void* stream) {
  if (!R || !P || !x || !y || !saved || !workspace || !allreduce) return MGT_EINVAL;
  const void* ptrs[] = {P->ln1_g, P->ln1_b, P->w_qkv, P->b_qkv, P->w_o, P->b_o,
                        P->ln2_g, P->ln2_b, P->w1, P->b1, P->w2, P->b2};
  TP_TRY_ST(check_ptrs(R, ptrs));
  if (!al16(x) || !al16(y) || ((uintptr_t)saved & 255) || ((uintptr_t)workspace & 255))
    return MGT_EUNSUPPORTED;
  TP_TRY_ST(ensure(R));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = R->T, h = R->h, hl = R->hl, fl = R->fl;
  const bool nb = R->cfg.disable_bias_linear, sw = R->cfg.swiglu;
  int* err = reinterpret_cast<int*>(at(workspace, R->ws[W_STATUS]));
  float* part = reinterpret_cast<float*>(at(workspace, R->ws[W_PART]));
  char* ln1 = at(saved, R->saved[S_LN1]);
  float* mu1 = reinterpret_cast<float*>(at(saved, R->saved[S_MU1]));
  float* rs1 = reinterpret_cast<float*>(at(saved, R->saved[S_RS1]));
  char* qkv = at(saved, R->saved[S_QKV]);
  char* O = at(saved, R->saved[S_O]);
  float* lse = reinterpret_cast<float*>(at(saved, R->saved[S_LSE]));
  char* h1 = at(saved, R->saved[S_H1]);
  char* ln2 = at(saved, R->saved[S_LN2]);
  float* mu2 = reinterpret_cast<float*>(at(saved, R->saved[S_MU2]));
  float* rs2 = reinterpret_cast<float*>(at(saved, R->saved[S_RS2]));
  char* aux = at(saved, R->saved[S_AUX]);
  char* act = at(saved, R->saved[S_A]);
  // LN1 (replicated rows), QKV of this rank's heads, attention over them
  TP_TRY(launch_ln_fwd(1, T, h, R->cfg.ln_eps, x, (const float*)P->ln1_g,
                       (const float*)P->ln1_b, ln1, mu1, rs1, err, s));
  {
    GemmArgs a = base(T, 3 * hl, h);
    a.A = ln1; a.lda = h; a.B = P->w_qkv; a.ldb = h;
    a.epi = kEpiBf16; a.out = qkv; a.ldc = 3 * hl; a.bias = nb ? nullptr : P->b_qkv;
    a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  }
  {
    AttnArgs a{R->cfg.micro_batch, R->cfg.seq, R->Hl, R->d, 1, qkv, O, lse,
               nullptr, nullptr, nullptr, err};
    TP_TRY(launch_attn_fwd(1, a, s));
  }
  // out-proj partial -> all-reduce -> h1 = x + b_o + sum
  {
    GemmArgs a = base(T, h, hl);
    a.lda = hl; a.B = P->w_o; a.ldb = hl;
    a.epi = kEpiStoreF32; a.ldc = h; a.err = err;
    TP_TRY_ST(reduce_begin(R, a, O, hl, part, allreduce, user, s));
  }
  TP_TRY_ST(reduce_end(R, part, allreduce, user, s));
  TP_TRY(sum_epilogue((long long)T * h, h, part, nb ? nullptr : P->b_o, x, h1, R->num_sms, s));
  // LN2, fc1 of this rank's columns (+ activation)
  TP_TRY(launch_ln_fwd(1, T, h, R->cfg.ln_eps, h1, (const float*)P->ln2_g,
                       (const float*)P->ln2_b, ln2, mu2, rs2, err, s));
  if (sw) {
    GemmArgs a = base(T, fl, h);
    a.A = ln2; a.lda = h; a.B = P->w1; a.ldb = h;
    a.epi = kEpiSwiglu; a.out = act; a.ldc = fl; a.out2 = aux; a.ldc2 = 2LL * fl;
    a.bias = nb ? nullptr : P->b1; a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  } else {
    GemmArgs a = base(T, fl, h);
    a.A = ln2; a.lda = h; a.B = P->w1; a.ldb = h;
    a.epi = kEpiGelu; a.out = act; a.out2 = aux; a.ldc = fl; a.bias = nb ? nullptr : P->b1;
    a.gelu_tanh = R->cfg.gelu_tanh; a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  }
  // fc2 partial -> all-reduce -> y = h1 + b2 + sum
  {
    GemmArgs a = base(T, h, fl);
    a.lda = fl; a.B = P->w2; a.ldb = fl;
    a.epi = kEpiStoreF32; a.ldc = h; a.err = err;
    TP_TRY_ST(reduce_begin(R, a, act, fl, part, allreduce, user, s));
  }
  TP_TRY_ST(reduce_end(R, part, allreduce, user, s));
  TP_TRY(sum_epilogue((long long)T * h, h, part, nb ? nullptr : P->b2, h1, y, R->num_sms, s));
  return MGT_OK;
}

mgt_status mgt_tp_rank_bwd(mgt_tp_rank* R, const mgt_layer_params* P, const void* x,
                           const void* saved, const void* dy, void* dx, const mgt_layer_grads* G,
                           void* workspace, mgt_allreduce_fn allreduce, void* user,
                           void* stream) {
  if (!R || !P || !G || !x || !saved || !dy || !dx || !workspace || !allreduce)
    return MGT_EINVAL;
  const void* ptrs[] = {P->ln1_g, P->ln1_b, P->w_qkv, P->b_qkv, P->w_o, P->b_o,
                        P->ln2_g, P->ln2_b, P->w1, P->b1, P->w2, P->b2};
  const void* gptrs[] = {G->ln1_g, G->ln1_b, G->w_qkv, G->b_qkv, G->w_o, G->b_o,
                         G->ln2_g, G->ln2_b, G->w1, G->b1, G->w2, G->b2};
  TP_TRY_ST(check_ptrs(R, ptrs));
  TP_TRY_ST(check_ptrs(R, gptrs));
  if (!al16(x) || !al16(dy) || !al16(dx) || ((uintptr_t)saved & 255) ||
      ((uintptr_t)workspace & 255))
    return MGT_EUNSUPPORTED;
  TP_TRY_ST(ensure(R));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = R->T, h = R->h, hl = R->hl, fl = R->fl, f1l = R->f1l;
  const bool nb = R->cfg.disable_bias_linear, sw = R->cfg.swiglu;
  int* err = reinterpret_cast<int*>(at(workspace, R->ws[W_STATUS]));
  float* part = reinterpret_cast<float*>(at(workspace, R->ws[W_PART]));
  const char* ln1 = at(saved, R->saved[S_LN1]);
  const float* mu1 = reinterpret_cast<const float*>(at(saved, R->saved[S_MU1]));
  const float* rs1 = reinterpret_cast<const float*>(at(saved, R->saved[S_RS1]));
  const char* qkv = at(saved, R->saved[S_QKV]);
  const char* O = at(saved, R->saved[S_O]);
  const float* lse = reinterpret_cast<const float*>(at(saved, R->saved[S_LSE]));
  const char* h1 = at(saved, R->saved[S_H1]);
  const char* ln2 = at(saved, R->saved[S_LN2]);
  const float* mu2 = reinterpret_cast<const float*>(at(saved, R->saved[S_MU2]));
  const float* rs2 = reinterpret_cast<const float*>(at(saved, R->saved[S_RS2]));
  const char* aux = at(saved, R->saved[S_AUX]);
  const char* act = at(saved, R->saved[S_A]);
  char* du = at(workspace, R->ws[W_DU]);
  char* dln2 = at(workspace, R->ws[W_DLN2]);
  char* dh1 = at(workspace, R->ws[W_DH1]);
  char* dO = at(workspace, R->ws[W_DO]);
  char* dqkv = at(workspace, R->ws[W_DQKV]);
  char* dln1 = at(workspace, R->ws[W_DLN1]);
  float* Dsum = reinterpret_cast<float*>(at(workspace, R->ws[W_D]));
  float* lnp = reinterpret_cast<float*>(at(workspace, R->ws[W_LNP]));
  // fc2: du = (dy W2_t) * act'(u) (the activation backward in the dgrad epilogue); dW2_t
  {
    GemmArgs a = base(T, fl, h);
    a.b_mn = 1; a.A = dy; a.lda = h; a.B = P->w2; a.ldb = fl;
    a.epi = sw ? kEpiDSwiglu : kEpiDGelu; a.out = du; a.ldc = f1l; a.aux = aux;
    a.ld_aux = f1l; a.gelu_tanh = R->cfg.gelu_tanh; a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  }
  {
    GemmArgs a = base(h, fl, T);
    a.a_mn = 1; a.b_mn = 1; a.A = dy; a.lda = h; a.B = act; a.ldb = fl;
    a.epi = kEpiStoreF32; a.out = G->w2; a.ldc = fl; a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  }
  // fc1: db1_t, dln2 partial -> all-reduce -> bf16, dW1_t
  if (!nb) TP_TRY(launch_colsum(1, T, f1l, du, (float*)G->b1, true, s));
  {
    GemmArgs a = base(T, h, f1l);
    a.b_mn = 1; a.lda = f1l; a.B = P->w1; a.ldb = h;
    a.epi = kEpiStoreF32; a.ldc = h; a.err = err;
    TP_TRY_ST(reduce_begin(R, a, du, f1l, part, allreduce, user, s));
  }
  {
    GemmArgs a = base(f1l, h, T);
    a.a_mn = 1; a.b_mn = 1; a.A = du; a.lda = f1l; a.B = ln2; a.ldb = h;
    a.epi = kEpiStoreF32; a.out = G->w1; a.ldc = h; a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  }
  TP_TRY_ST(reduce_end(R, part, allreduce, user, s));
  TP_TRY(sum_epilogue((long long)T * h, h, part, nullptr, nullptr, dln2, R->num_sms, s));
  // LN2 backward (replicated): dh1 = dy + LN2'(dln2); the dres sum is db2
  TP_TRY(launch_ln_bwd(1, T, h, dln2, dy, h1, (const float*)P->ln2_g, mu2, rs2, dh1, lnp,
                       R->nblk, (float*)G->ln2_g, (float*)G->ln2_b,
                       nb ? nullptr : (float*)G->b2, err, s));
  // out-proj: dO_t = dh1 W_o,t; dW_o,t
  {
    GemmArgs a = base(T, hl, h);
    a.b_mn = 1; a.A = dh1; a.lda = h; a.B = P->w_o; a.ldb = hl;
    a.epi = kEpiBf16; a.out = dO; a.ldc = hl; a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  }
  {
    GemmArgs a = base(h, hl, T);
    a.a_mn = 1; a.b_mn = 1; a.A = dh1; a.lda = h; a.B = O; a.ldb = hl;
    a.epi = kEpiStoreF32; a.out = G->w_o; a.ldc = hl; a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  }
  // attention backward over this rank's heads
  {
    AttnArgs a{R->cfg.micro_batch, R->cfg.seq, R->Hl, R->d, 1, qkv, (void*)O, (float*)lse,
               dO, Dsum, dqkv, err};
    if (R->ws[W_DQACC].bytes) {
      char* base = at(workspace, R->ws[W_DQACC]);
      const DqScratch q = dq_scratch_layout(R->cfg.micro_batch, R->cfg.seq, R->Hl);
      a.dq_fix = reinterpret_cast<int32_t*>(base + q.fix_off);
      a.dq_exp = reinterpret_cast<int32_t*>(base + q.exp_off);
      a.dq_bound = reinterpret_cast<float*>(base + q.bound_off);
      a.dq_stat = reinterpret_cast<float*>(base + q.stat_off);
    }
    TP_TRY(launch_attn_bwd(1, a, s));
  }
  // QKV: db_qkv_t, dln1 partial -> all-reduce -> bf16, dW_qkv,t
  if (!nb) TP_TRY(launch_colsum(1, T, 3 * hl, dqkv, (float*)G->b_qkv, true, s));
  {
    GemmArgs a = base(T, h, 3 * hl);
    a.b_mn = 1; a.lda = 3 * hl; a.B = P->w_qkv; a.ldb = h;
    a.epi = kEpiStoreF32; a.ldc = h; a.err = err;
    TP_TRY_ST(reduce_begin(R, a, dqkv, 3 * hl, part, allreduce, user, s));
  }
  {
    GemmArgs a = base(3 * hl, h, T);
    a.a_mn = 1; a.b_mn = 1; a.A = dqkv; a.lda = 3 * hl; a.B = ln1; a.ldb = h;
    a.epi = kEpiStoreF32; a.out = G->w_qkv; a.ldc = h; a.err = err;
    TP_TRY(launch_gemm_tc(a, R->num_sms, s));
  }
  TP_TRY_ST(reduce_end(R, part, allreduce, user, s));
  TP_TRY(sum_epilogue((long long)T * h, h, part, nullptr, nullptr, dln1, R->num_sms, s));
  // LN1 backward (replicated): dx = dh1 + LN1'(dln1); the dres sum is db_o
  TP_TRY(launch_ln_bwd(1, T, h, dln1, dh1, x, (const float*)P->ln1_g, mu1, rs1, dx, lnp,
                       R->nblk, (float*)G->ln1_g, (float*)G->ln1_b,
                       nb ? nullptr : (float*)G->b_o, err, s));
  return MGT_OK;
}

}  // extern "C"
