// C ABI of the tensor-parallel GPT layer: validation, buffer layout, and the launch sequence of
// the forward and backward passes. Host code only; every step of the layer runs in the
// kernels of gemm_tc.cu, attn.cu and ln_misc.cu.
//
// The logical tensor-parallel shards follow the partitioning on the trdm.cn page, section 2.1,
// and the ColumnParallelLinear / RowParallelLinear pairing on the second-brain-czx page
// ("张量并行"): QKV and fc1 are column-parallel (one GEMM over the packed rows of every shard:
// the shards' output blocks are independent), out-proj and fc2 are row-parallel (the GEMM's K
// loop runs over the shards, so the shard partials are summed in the accumulator, which is what
// the AllReduce after RowParallelLinear computes). In the backward pass the column-parallel
// layers' input gradient is the sum of the shards' contributions (x was broadcast); that sum is
// again the K loop of the dgrad GEMM.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/mgt_layer.h"
#include "mgt_internal.h"

using namespace mgt;

namespace {

// LayerNorm backward blocks, each writing one partial row of dgamma/dbeta (and the residual
// gradient's column sum): one per SM on 148 SMs. A block's bulk-copy row ring keeps enough
// bytes in flight on its own, and half the partial rows of two per SM take 7 us per step off
// the two fixed-order parameter reduces.
constexpr int kMaxLnBlocks = 148;

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Region {
  size_t off = 0, bytes = 0;
};

struct ProfEntry {
  const char* family;
  double flops, bytes;
  cudaEvent_t start, stop;
};

struct Family {
  std::string name;
  int64_t launches = 0;
  double ms = 0, flops = 0, bytes = 0;
};

}  // namespace

struct mgt_layer {
  mgt_layer_config cfg;
  int T, h, H, d, f, p;
  int esz;  // activation element size
  Region saved[MGT_SAVED_COUNT];
  Region ws[MGT_WS_COUNT - 64];
  size_t saved_bytes = 0, ws_bytes = 0;
  int num_sms = 0;
  int device = -1;  // the device the handle is bound to (at its first call)
  // second stream of the backward (weight gradients) and its fork / join events
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork[4] = {};
  cudaEvent_t ev_join = nullptr;
  // profiling
  bool prof = false;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_next = 0;
  std::vector<ProfEntry> pending;
  std::vector<Family> fams;
};

namespace {

mgt_status validate(const mgt_layer_config* c) {
  if (!c) return MGT_EINVAL;
  if (c->hidden <= 0 || c->heads <= 0 || c->ffn <= 0 || c->seq <= 0 || c->micro_batch <= 0 ||
      c->tp_size <= 0)
    return MGT_EINVAL;
  if (c->hidden % c->heads || c->hidden % c->tp_size || c->heads % c->tp_size ||
      c->ffn % c->tp_size)
    return MGT_EINVAL;
  if (!(c->ln_eps >= 0.f)) return MGT_EINVAL;
  if (c->swiglu != 0 && c->swiglu != 1) return MGT_EINVAL;
  if (c->disable_bias_linear != 0 && c->disable_bias_linear != 1) return MGT_EINVAL;
  if (c->sequence_parallel != 0 && c->sequence_parallel != 1) return MGT_EINVAL;
  if (c->sequence_parallel && c->seq % c->tp_size) return MGT_EINVAL;
  // sequence-parallel tiles: 128 tokens of a GEMM tile stay inside one shard's positions
  if (c->sequence_parallel && c->dtype == MGT_BF16 && (c->seq / c->tp_size) % 128)
    return MGT_EUNSUPPORTED;
  if (c->causal != 1) return MGT_EUNSUPPORTED;
  const long long T = (long long)c->seq * c->micro_batch;
  if (T > (1LL << 30) || (long long)c->ffn * 3 > (1LL << 30) || (long long)c->hidden * 3 > (1LL << 30))
    return MGT_EINVAL;
  const int d = c->hidden / c->heads;
  if (c->dtype == MGT_BF16) {
    if (d != 64 && d != 128) return MGT_EUNSUPPORTED;
    // K tiles of the row-parallel GEMMs must not straddle shards; 16-byte TMA strides.
    if ((c->hidden / c->tp_size) % 64 || (c->ffn / c->tp_size) % 64) return MGT_EUNSUPPORTED;
    if (c->hidden > 16384) return MGT_EUNSUPPORTED;
  } else if (c->dtype == MGT_F32) {
    if (d > 64 || c->hidden % 4 || c->ffn % 4 || c->hidden > 8192) return MGT_EUNSUPPORTED;
  } else {
    return MGT_EUNSUPPORTED;
  }
  return MGT_OK;
}

// fixed-point dQ accumulator and scaling data of the single-kernel attention backward (bf16,
// head_dim 128)
size_t dq_acc_bytes(const mgt_layer* L) {
  if (L->cfg.dtype != MGT_BF16 || L->d != 128) return 0;
  return dq_scratch_layout(L->cfg.micro_batch, L->cfg.seq, L->H).bytes;
}

void layout(mgt_layer* L) {
  const size_t T = L->T, h = L->h, f = L->f, e = L->esz;
  const size_t f1 = L->cfg.swiglu ? 2 * f : f;  // fc1 outputs: [gate | up] with SwiGLU
  const size_t bHs = (size_t)L->cfg.micro_batch * L->H * L->cfg.seq;
  size_t sz[MGT_SAVED_COUNT] = {T * h * e, T * 4, T * 4, T * 3 * h * e, T * h * e, bHs * 4,
                                T * h * e, T * h * e, T * 4, T * 4, T * f1 * e, T * f * e};
  size_t off = 0;
  for (int i = 0; i < MGT_SAVED_COUNT; ++i) {
    L->saved[i].off = off;
    L->saved[i].bytes = sz[i];
    off += align256(sz[i]);
  }
  L->saved_bytes = off;
  const size_t nblk = T < (size_t)kMaxLnBlocks ? T : (size_t)kMaxLnBlocks;
  size_t wsz[MGT_WS_COUNT - 64] = {256,
                                   T * f1 * e,
                                   T * h * e,
                                   T * h * e,
                                   T * h * e,
                                   T * 3 * h * e,
                                   T * h * e,
                                   bHs * 4,
                                   dq_acc_bytes(L),
                                   nblk * 3 * h * 4};
  off = 0;
  for (int i = 0; i < MGT_WS_COUNT - 64; ++i) {
    L->ws[i].off = off;
    L->ws[i].bytes = wsz[i];
    off += align256(wsz[i]);
  }
  L->ws_bytes = off;
}

inline char* sp(void* base, const Region& r) { return static_cast<char*>(base) + r.off; }
inline const char* sp(const void* base, const Region& r) {
  return static_cast<const char*>(base) + r.off;
}

// Runs one launch, bracketed by profiling events when enabled.
template <class F>
cudaError_t run(mgt_layer* L, const char* family, double flops, double bytes, cudaStream_t s,
                F&& fn) {
  if (!L->prof || L->ev_next + 2 > L->ev_pool.size()) return fn();
  ProfEntry e{family, flops, bytes, L->ev_pool[L->ev_next], L->ev_pool[L->ev_next + 1]};
  L->ev_next += 2;
  cudaEventRecord(e.start, s);
  cudaError_t r = fn();
  cudaEventRecord(e.stop, s);
  L->pending.push_back(e);
  return r;
}

GemmArgs gemm_base(int M, int Ng, int NG, int Kg, int KG) {
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = M; a.Ng = Ng; a.NG = NG; a.Kg = Kg; a.KG = KG;
  a.out_ng = Ng * NG;
  a.out_gs = 0;
  return a;
}

// `site` names the call ("gemm_tc/fc1_fwd", ...): profiling groups launches by this name.
// With sequence parallelism the row map of the shard-major layout is filled in here; the call
// sites set which operand or output lives in it (a_sp, b_sp, out_sp).
cudaError_t gemm(mgt_layer* L, const char* site, const GemmArgs& a_in, cudaStream_t s) {
  GemmArgs a = a_in;
  if (!L->cfg.sequence_parallel) {
    a.a_sp = a.b_sp = a.out_sp = 0;
  } else {
    a.sp_seq = L->cfg.seq;
    a.sp_len = L->cfg.seq / L->cfg.tp_size;
    a.sp_b = L->cfg.micro_batch;
  }
  // A SwiGLU fc1 tile computes a gate and an up product per output.
  const double flops = 2.0 * a.M * (double)a.Ng * a.NG * (double)a.Kg * a.KG *
                       (a.epi == kEpiSwiglu ? 2 : 1);
  if (L->cfg.dtype == MGT_BF16)
    return run(L, site, flops, 0, s, [&] { return launch_gemm_tc(a, L->num_sms, s); });
  return run(L, "gemm_simt", flops, 0, s, [&] { return launch_gemm_simt_f32(a, s); });
}

mgt_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MGT_OK;
  return MGT_ECUDA;
}

#define MGT_TRY(expr)                          \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return MGT_ECUDA;   \
  } while (0)

// The handle binds to the device current at its first call (its SM count, its backward
// stream); a later call from another device is rejected.
mgt_status ensure_device(mgt_layer* L) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MGT_ECUDA;
  if (L->num_sms > 0) return dev == L->device ? MGT_OK : MGT_EUNSUPPORTED;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return MGT_ECUDA;
  if (L->cfg.dtype == MGT_BF16) {
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) return MGT_EUNSUPPORTED;  // tcgen05 / TMA kernels are built for sm_100a
  }
  L->num_sms = n;
  L->device = dev;
  return MGT_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// The backward's second stream (non-blocking) and its events, created on first use; on a
// failure everything created so far is released and the next call tries again.
cudaError_t ensure_side_stream(mgt_layer* L) {
  if (L->side) return cudaSuccess;
  cudaStream_t side = nullptr;
  cudaEvent_t ev[5] = {};
  cudaError_t e = cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking);
  for (int i = 0; i < 5 && e == cudaSuccess; ++i)
    e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
  if (e != cudaSuccess) {
    for (auto& x : ev)
      if (x) cudaEventDestroy(x);
    if (side) cudaStreamDestroy(side);
    return e;
  }
  for (int i = 0; i < 4; ++i) L->ev_fork[i] = ev[i];
  L->ev_join = ev[4];
  L->side = side;
  return cudaSuccess;
}

// Every parameter (and gradient) pointer must be set and 16-byte aligned, except the four
// linear biases of a layer without them, which are ignored.
mgt_status check_param_ptrs(const mgt_layer* L, const void* const* q) {
  for (int i = 0; i < 12; ++i) {
    const bool is_bias = i == 3 || i == 5 || i == 9 || i == 11;  // b_qkv, b_o, b1, b2
    if (is_bias && L->cfg.disable_bias_linear) continue;
    if (!q[i]) return MGT_EINVAL;
    if (!aligned16(q[i])) return MGT_EUNSUPPORTED;
  }
  return MGT_OK;
}

}  // namespace

extern "C" {

const char* mgt_status_string(mgt_status s) {
  switch (s) {
    case MGT_OK: return "ok";
    case MGT_EINVAL: return "invalid argument";
    case MGT_EUNSUPPORTED: return "unsupported configuration";
    case MGT_ECUDA: return "CUDA error";
    case MGT_ETIMEOUT: return "device wait timed out";
    case MGT_ENOMEM: return "buffer too small";
  }
  return "unknown status";
}

mgt_status mgt_layer_init(const mgt_layer_config* cfg, mgt_layer** out) {
  if (!out) return MGT_EINVAL;
  *out = nullptr;
  mgt_status st = validate(cfg);
  if (st != MGT_OK) return st;
  mgt_layer* L = new (std::nothrow) mgt_layer();
  if (!L) return MGT_ENOMEM;
  L->cfg = *cfg;
  L->T = cfg->seq * cfg->micro_batch;
  L->h = cfg->hidden;
  L->H = cfg->heads;
  L->d = cfg->hidden / cfg->heads;
  L->f = cfg->ffn;
  L->p = cfg->tp_size;
  L->esz = cfg->dtype == MGT_BF16 ? 2 : 4;
  layout(L);
  *out = L;
  return MGT_OK;
}

mgt_status mgt_layer_sizes(const mgt_layer* L, size_t* saved_bytes, size_t* workspace_bytes) {
  if (!L) return MGT_EINVAL;
  if (saved_bytes) *saved_bytes = L->saved_bytes;
  if (workspace_bytes) *workspace_bytes = L->ws_bytes;
  return MGT_OK;
}

mgt_status mgt_layer_region(const mgt_layer* L, int region, size_t* offset, size_t* bytes) {
  if (!L) return MGT_EINVAL;
  Region r;
  if (region >= 0 && region < MGT_SAVED_COUNT)
    r = L->saved[region];
  else if (region >= 64 && region < MGT_WS_COUNT)
    r = L->ws[region - 64];
  else
    return MGT_EINVAL;
  if (offset) *offset = r.off;
  if (bytes) *bytes = r.bytes;
  return MGT_OK;
}

mgt_status mgt_layer_fwd(mgt_layer* L, const mgt_layer_params* P, const void* x, void* y,
                         void* saved, void* workspace, void* stream) {
  if (!L || !P || !x || !y || !saved || !workspace) return MGT_EINVAL;
  const void* ptrs[] = {P->ln1_g, P->ln1_b, P->w_qkv, P->b_qkv, P->w_o, P->b_o,
                        P->ln2_g, P->ln2_b, P->w1, P->b1, P->w2, P->b2};
  mgt_status st = check_param_ptrs(L, ptrs);
  if (st != MGT_OK) return st;
  if (!aligned16(x) || !aligned16(y) || ((uintptr_t)saved & 255) || ((uintptr_t)workspace & 255))
    return MGT_EUNSUPPORTED;
  st = ensure_device(L);
  if (st != MGT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = L->T, h = L->h, f = L->f, p = L->p, dt = L->cfg.dtype == MGT_BF16 ? 1 : 0;
  const int e = L->esz;
  int* err = reinterpret_cast<int*>(sp(workspace, L->ws[MGT_WS_STATUS - 64]));
  char* ln1 = sp(saved, L->saved[MGT_SAVED_LN1]);
  float* mu1 = reinterpret_cast<float*>(sp(saved, L->saved[MGT_SAVED_LN1_MEAN]));
  float* rs1 = reinterpret_cast<float*>(sp(saved, L->saved[MGT_SAVED_LN1_RSTD]));
  char* qkv = sp(saved, L->saved[MGT_SAVED_QKV]);
  char* O = sp(saved, L->saved[MGT_SAVED_ATTN_O]);
  float* lse = reinterpret_cast<float*>(sp(saved, L->saved[MGT_SAVED_ATTN_LSE]));
  char* h1 = sp(saved, L->saved[MGT_SAVED_H1]);
  char* ln2 = sp(saved, L->saved[MGT_SAVED_LN2]);
  float* mu2 = reinterpret_cast<float*>(sp(saved, L->saved[MGT_SAVED_LN2_MEAN]));
  float* rs2 = reinterpret_cast<float*>(sp(saved, L->saved[MGT_SAVED_LN2_RSTD]));
  char* u1 = sp(saved, L->saved[MGT_SAVED_FC1_U]);  // fc1 pre-activation u
  char* act = sp(saved, L->saved[MGT_SAVED_FC1_A]);
  const double ln_bytes = (double)T * h * 2 * e + 8.0 * h;
  const bool nb = L->cfg.disable_bias_linear;
  const void* b_qkv = nb ? nullptr : P->b_qkv;
  const void* b_o = nb ? nullptr : P->b_o;
  const void* b1 = nb ? nullptr : P->b1;
  const void* b2 = nb ? nullptr : P->b2;

  // 1. LN1
  MGT_TRY(run(L, "ln_fwd", 0, ln_bytes, s, [&] {
    return launch_ln_fwd(dt, T, h, L->cfg.ln_eps, x, (const float*)P->ln1_g,
                         (const float*)P->ln1_b, ln1, mu1, rs1, err, s);
  }));
  // 2. QKV, column-parallel: the packed [p][3][H/p][d] rows are the GEMM's N dimension.
  {
    GemmArgs a = gemm_base(T, 3 * h, 1, h, 1);
    a.A = ln1; a.lda = h; a.B = P->w_qkv; a.ldb = h;
    a.epi = kEpiBf16; a.out = qkv; a.ldc = 3 * h; a.bias = b_qkv; a.err = err;
    a.a_sp = 1;  // sequence parallel: the all-gather of ln1 is this row map
    MGT_TRY(gemm(L, "gemm_tc/qkv_fwd", a, s));
  }
  // 3. causal attention per head (each shard's heads are local)
  {
    AttnArgs a{L->cfg.micro_batch, L->cfg.seq, L->H, L->d, p, qkv, O, lse,
               nullptr, nullptr, nullptr, err};
    const double fl = 2.0 * L->cfg.micro_batch * (double)L->cfg.seq * L->cfg.seq * h;
    MGT_TRY(run(L, "attn_fwd", fl, 0, s, [&] { return launch_attn_fwd(dt, a, s); }));
  }
  // 4. out-proj, row-parallel: K loop over shards (A = O as [T][p][h/p], B = w_o [p][h][h/p]),
  //    partial sums add in the accumulator; + b_o once; + residual x.
  {
    GemmArgs a = gemm_base(T, h, 1, h / p, p);
    a.A = O; a.lda = h; a.B = P->w_o; a.ldb = h / p; a.b_kgs = (long long)h * (h / p);
    a.epi = kEpiBf16; a.out = h1; a.ldc = h; a.bias = b_o; a.res = x; a.ldr = h; a.err = err;
    a.out_sp = 1;  // sequence parallel: the reduce-scatter of the shard sum is this row map
    MGT_TRY(gemm(L, "gemm_tc/outproj_fwd", a, s));
  }
  // 5. LN2
  MGT_TRY(run(L, "ln_fwd", 0, ln_bytes, s, [&] {
    return launch_ln_fwd(dt, T, h, L->cfg.ln_eps, h1, (const float*)P->ln2_g,
                         (const float*)P->ln2_b, ln2, mu2, rs2, err, s);
  }));
  // 6. fc1, column-parallel, + b1, GeLU (stores a = GeLU(u) and u for the backward).
  //    SwiGLU: shard t's gate and up rows go to the two halves of one tile; the epilogue stores
  //    a = silu(gate) * up and [gate | up] for the backward.
  if (L->cfg.swiglu) {
    GemmArgs a = gemm_base(T, f / p, p, h, 1);
    a.A = ln2; a.lda = h; a.B = P->w1; a.ldb = h;
    a.epi = kEpiSwiglu; a.out = act; a.ldc = f; a.out2 = u1; a.ldc2 = 2LL * f; a.bias = b1;
    a.err = err; a.a_sp = 1;
    MGT_TRY(gemm(L, "gemm_tc/fc1_fwd", a, s));
  } else {
    GemmArgs a = gemm_base(T, f, 1, h, 1);
    a.A = ln2; a.lda = h; a.B = P->w1; a.ldb = h;
    a.epi = kEpiGelu; a.out = act; a.out2 = u1; a.ldc = f; a.bias = b1;
    a.gelu_tanh = L->cfg.gelu_tanh; a.err = err; a.a_sp = 1;
    MGT_TRY(gemm(L, "gemm_tc/fc1_fwd", a, s));
  }
  // 7. fc2, row-parallel with shard sum, + b2, + residual h1
  {
    GemmArgs a = gemm_base(T, h, 1, f / p, p);
    a.A = act; a.lda = f; a.B = P->w2; a.ldb = f / p; a.b_kgs = (long long)h * (f / p);
    a.epi = kEpiBf16; a.out = y; a.ldc = h; a.bias = b2; a.res = h1; a.ldr = h; a.err = err;
    a.out_sp = 1;
    MGT_TRY(gemm(L, "gemm_tc/fc2_fwd", a, s));
  }
  return MGT_OK;
}

mgt_status mgt_layer_bwd(mgt_layer* L, const mgt_layer_params* P, const void* x,
                         const void* saved, const void* dy, void* dx, const mgt_layer_grads* G,
                         void* workspace, void* stream) {
  if (!L || !P || !x || !saved || !dy || !dx || !G || !workspace) return MGT_EINVAL;
  const void* ptrs[] = {P->ln1_g, P->ln1_b, P->w_qkv, P->b_qkv, P->w_o, P->b_o,
                        P->ln2_g, P->ln2_b, P->w1, P->b1, P->w2, P->b2};
  const void* gptrs[] = {G->ln1_g, G->ln1_b, G->w_qkv, G->b_qkv, G->w_o, G->b_o,
                         G->ln2_g, G->ln2_b, G->w1, G->b1, G->w2, G->b2};
  mgt_status st = check_param_ptrs(L, ptrs);
  if (st == MGT_OK) st = check_param_ptrs(L, gptrs);
  if (st != MGT_OK) return st;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || ((uintptr_t)saved & 255) ||
      ((uintptr_t)workspace & 255))
    return MGT_EUNSUPPORTED;
  st = ensure_device(L);
  if (st != MGT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = L->T, h = L->h, f = L->f, p = L->p, dt = L->cfg.dtype == MGT_BF16 ? 1 : 0;
  const int e = L->esz;
  int* err = reinterpret_cast<int*>(sp(workspace, L->ws[MGT_WS_STATUS - 64]));
  const char* ln1 = sp(saved, L->saved[MGT_SAVED_LN1]);
  const float* mu1 = reinterpret_cast<const float*>(sp(saved, L->saved[MGT_SAVED_LN1_MEAN]));
  const float* rs1 = reinterpret_cast<const float*>(sp(saved, L->saved[MGT_SAVED_LN1_RSTD]));
  const char* qkv = sp(saved, L->saved[MGT_SAVED_QKV]);
  const char* O = sp(saved, L->saved[MGT_SAVED_ATTN_O]);
  const float* lse = reinterpret_cast<const float*>(sp(saved, L->saved[MGT_SAVED_ATTN_LSE]));
  const char* h1 = sp(saved, L->saved[MGT_SAVED_H1]);
  const char* ln2 = sp(saved, L->saved[MGT_SAVED_LN2]);
  const float* mu2 = reinterpret_cast<const float*>(sp(saved, L->saved[MGT_SAVED_LN2_MEAN]));
  const float* rs2 = reinterpret_cast<const float*>(sp(saved, L->saved[MGT_SAVED_LN2_RSTD]));
  const char* u1 = sp(saved, L->saved[MGT_SAVED_FC1_U]);
  const char* act = sp(saved, L->saved[MGT_SAVED_FC1_A]);
  char* du = sp(workspace, L->ws[MGT_WS_DU - 64]);
  char* dln2 = sp(workspace, L->ws[MGT_WS_DLN2 - 64]);
  char* dh1 = sp(workspace, L->ws[MGT_WS_DH1 - 64]);
  char* dO = sp(workspace, L->ws[MGT_WS_DO - 64]);
  char* dqkv = sp(workspace, L->ws[MGT_WS_DQKV - 64]);
  char* dln1 = sp(workspace, L->ws[MGT_WS_DLN1 - 64]);
  float* Dsum = reinterpret_cast<float*>(sp(workspace, L->ws[MGT_WS_ATTN_D - 64]));
  float* part = reinterpret_cast<float*>(sp(workspace, L->ws[MGT_WS_LN_PARTIAL - 64]));
  const int nblk = T < kMaxLnBlocks ? T : kMaxLnBlocks;
  // Weight gradients and bias column sums feed nothing else in the backward: they run on a
  // second stream `w`, forked after the launch that produces their inputs and joined into `s`
  // at the end, so their tiles fill the SMs that the data-gradient chain's last partial waves
  // leave idle. With profiling on, every launch stays on `s` and is timed alone.
  const bool two = !L->prof;
  if (two) MGT_TRY(ensure_side_stream(L));
  cudaStream_t w = two ? L->side : s;
  auto fork = [&](int k) -> cudaError_t {
    if (!two) return cudaSuccess;
    cudaError_t r = cudaEventRecord(L->ev_fork[k], s);
    return r == cudaSuccess ? cudaStreamWaitEvent(w, L->ev_fork[k], 0) : r;
  };
  // joins `w` into `s` on every return path once the first fork has been made
  struct Join {
    mgt_layer* L;
    cudaStream_t s, w;
    bool on = false;
    ~Join() {
      if (on && cudaEventRecord(L->ev_join, w) == cudaSuccess) cudaStreamWaitEvent(s, L->ev_join, 0);
    }
  } join{L, s, w};
  auto colsum = [&](const void* src, int cols, void* out) {
    return run(L, "colsum", 0, (double)T * cols * e + 4.0 * cols, w,
               [&] { return launch_colsum(dt, T, cols, src, (float*)out, !two, w); });
  };
  const double lnb_bytes = (double)T * h * 6 * e + 3.0 * nblk * h * 4 * 2;
  const bool nb = L->cfg.disable_bias_linear, sw = L->cfg.swiglu;
  const int f1 = sw ? 2 * f : f;  // fc1 output columns (gate and up with SwiGLU)

  // B1. fc2: dgrad fused with GeLU' -> du (SwiGLU: with the SwiGLU backward -> d[gate | up]),
  //     wgrad (db2 = sum dy comes with the LN2 backward)
  MGT_TRY(fork(0));  // dy and the saved activation a are ready
  join.on = two;
  {
    GemmArgs a = gemm_base(T, f / p, p, h, 1);  // N grouped by shard
    a.b_mn = 1; a.A = dy; a.lda = h; a.B = P->w2; a.ldb = f / p;
    a.b_ngs = (long long)h * (f / p);
    a.epi = sw ? kEpiDSwiglu : kEpiDGelu; a.out = du; a.ldc = f1; a.aux = u1; a.ld_aux = f1;
    a.gelu_tanh = L->cfg.gelu_tanh; a.err = err;
    a.a_sp = 1;  // dy is sequence-parallel: its all-gather (adjoint of the reduce-scatter)
    MGT_TRY(gemm(L, "gemm_tc/fc2_dgrad", a, s));
  }
  {
    GemmArgs a = gemm_base(h, f, 1, T, 1);
    a.a_mn = 1; a.b_mn = 1; a.A = dy; a.lda = h; a.B = act; a.ldb = f;
    a.epi = kEpiStoreF32; a.out = G->w2; a.ldc = f / p; a.out_ng = f / p;
    a.plain_launch = two;  // the side stream's predecessor is not an input
    a.out_gs = (long long)h * (f / p); a.err = err; a.a_sp = 1;
    MGT_TRY(gemm(L, "gemm_tc/fc2_wgrad", a, w));
  }
  MGT_TRY(fork(1));  // du is ready (fc2 dgrad)
  // B3. fc1: db1, dgrad (sum over shards = K loop over all fc1 outputs), wgrad
  if (!nb) MGT_TRY(colsum(du, f1, G->b1));
  {
    GemmArgs a = gemm_base(T, h, 1, f1, 1);
    a.b_mn = 1; a.A = du; a.lda = f1; a.B = P->w1; a.ldb = h;
    a.epi = kEpiBf16; a.out = dln2; a.ldc = h; a.err = err;
    a.out_sp = 1;  // the reduce-scatter of dln2 (adjoint of the all-gather of ln2)
    MGT_TRY(gemm(L, "gemm_tc/fc1_dgrad", a, s));
  }
  {
    GemmArgs a = gemm_base(f1, h, 1, T, 1);
    a.a_mn = 1; a.b_mn = 1; a.A = du; a.lda = f1; a.B = ln2; a.ldb = h;
    a.epi = kEpiStoreF32; a.out = G->w1; a.ldc = h; a.err = err; a.b_sp = 1;
    a.plain_launch = two;  // the side stream's predecessor is not an input
    MGT_TRY(gemm(L, "gemm_tc/fc1_wgrad", a, w));
  }
  // B4. LN2 backward + residual gradient dy -> dh1
  MGT_TRY(run(L, "ln_bwd", 0, lnb_bytes, s, [&] {
    // dres = dy, so the residual-gradient sum it also returns is db2
    return launch_ln_bwd(dt, T, h, dln2, dy, h1, (const float*)P->ln2_g, mu2, rs2, dh1, part,
                         nblk, (float*)G->ln2_g, (float*)G->ln2_b,
                         nb ? nullptr : (float*)G->b2, err, s);
  }));
  MGT_TRY(fork(2));  // dh1 is ready
  // B5. out-proj: dgrad (N grouped by shard) -> dO, wgrad (db_o = sum dh1 comes with LN1 bwd)
  {
    GemmArgs a = gemm_base(T, h / p, p, h, 1);
    a.b_mn = 1; a.A = dh1; a.lda = h; a.B = P->w_o; a.ldb = h / p;
    a.b_ngs = (long long)h * (h / p);
    a.epi = kEpiBf16; a.out = dO; a.ldc = h; a.err = err; a.a_sp = 1;
    MGT_TRY(gemm(L, "gemm_tc/outproj_dgrad", a, s));
  }
  {
    GemmArgs a = gemm_base(h, h, 1, T, 1);
    a.a_mn = 1; a.b_mn = 1; a.A = dh1; a.lda = h; a.B = O; a.ldb = h; a.a_sp = 1;
    a.epi = kEpiStoreF32; a.out = G->w_o; a.ldc = h / p; a.out_ng = h / p;
    a.plain_launch = two;  // the side stream's predecessor is not an input
    a.out_gs = (long long)h * (h / p); a.err = err;
    MGT_TRY(gemm(L, "gemm_tc/outproj_wgrad", a, w));
  }
  // B6. attention backward (probabilities recomputed from the saved log-sum-exp)
  {
    AttnArgs a{L->cfg.micro_batch, L->cfg.seq, L->H, L->d, p, qkv, (void*)O, (float*)lse,
               dO, Dsum, dqkv, err};
    if (L->ws[MGT_WS_DQ_ACC - 64].bytes) {
      char* base = sp(workspace, L->ws[MGT_WS_DQ_ACC - 64]);
      const DqScratch q = dq_scratch_layout(L->cfg.micro_batch, L->cfg.seq, L->H);
      a.dq_fix = reinterpret_cast<int32_t*>(base + q.fix_off);
      a.dq_exp = reinterpret_cast<int32_t*>(base + q.exp_off);
      a.dq_bound = reinterpret_cast<float*>(base + q.bound_off);
      a.dq_stat = reinterpret_cast<float*>(base + q.stat_off);
    }
    const double fl = 2.5 * 2.0 * L->cfg.micro_batch * (double)L->cfg.seq * L->cfg.seq * h;  // model FLOPs incl. one recompute of S
    MGT_TRY(run(L, "attn_bwd", fl, 0, s, [&] { return launch_attn_bwd(dt, a, s); }));
  }
  MGT_TRY(fork(3));  // dqkv is ready
  // B7. QKV: db_qkv, dgrad (sum over shards = K loop over 3h), wgrad
  if (!nb) MGT_TRY(colsum(dqkv, 3 * h, G->b_qkv));
  {
    GemmArgs a = gemm_base(T, h, 1, 3 * h, 1);
    a.b_mn = 1; a.A = dqkv; a.lda = 3 * h; a.B = P->w_qkv; a.ldb = h;
    a.epi = kEpiBf16; a.out = dln1; a.ldc = h; a.err = err; a.out_sp = 1;
    MGT_TRY(gemm(L, "gemm_tc/qkv_dgrad", a, s));
  }
  {
    GemmArgs a = gemm_base(3 * h, h, 1, T, 1);
    a.a_mn = 1; a.b_mn = 1; a.A = dqkv; a.lda = 3 * h; a.B = ln1; a.ldb = h;
    a.epi = kEpiStoreF32; a.out = G->w_qkv; a.ldc = h; a.err = err; a.b_sp = 1;
    a.plain_launch = two;  // the side stream's predecessor is not an input
    MGT_TRY(gemm(L, "gemm_tc/qkv_wgrad", a, w));
  }
  // B8. LN1 backward + residual gradient dh1 -> dx
  MGT_TRY(run(L, "ln_bwd", 0, lnb_bytes, s, [&] {
    // dres = dh1, so the residual-gradient sum it also returns is db_o
    return launch_ln_bwd(dt, T, h, dln1, dh1, x, (const float*)P->ln1_g, mu1, rs1, dx, part,
                         nblk, (float*)G->ln1_g, (float*)G->ln1_b,
                         nb ? nullptr : (float*)G->b_o, err, s);
  }));
  return MGT_OK;
}

mgt_status mgt_layer_get_error(mgt_layer* L, void* workspace, void* stream) {
  if (!L || !workspace) return MGT_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MGT_ECUDA;
  int word = 0;
  int* dev = reinterpret_cast<int*>(sp(workspace, L->ws[MGT_WS_STATUS - 64]));
  if (cudaMemcpy(&word, dev, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MGT_ECUDA;
  if (word != 0) {
    if (cudaMemset(dev, 0, sizeof(int)) != cudaSuccess) return MGT_ECUDA;
    return MGT_ETIMEOUT;
  }
  return cudaGetLastError() == cudaSuccess ? MGT_OK : MGT_ECUDA;
}

mgt_status mgt_layer_profile(mgt_layer* L, int enable) {
  if (!L) return MGT_EINVAL;
  if (enable && L->ev_pool.empty()) {
    L->ev_pool.resize(8192);
    for (auto& ev : L->ev_pool)
      if (cudaEventCreate(&ev) != cudaSuccess) return MGT_ECUDA;
  }
  L->prof = enable != 0;
  return MGT_OK;
}

mgt_status mgt_layer_profile_read(mgt_layer* L, mgt_kernel_stat* out, int cap, int* n) {
  if (!L || !n) return MGT_EINVAL;
  for (auto& e : L->pending) {
    if (cudaEventSynchronize(e.stop) != cudaSuccess) return MGT_ECUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, e.start, e.stop) != cudaSuccess) return MGT_ECUDA;
    Family* fam = nullptr;
    for (auto& fm : L->fams)
      if (fm.name == e.family) fam = &fm;
    if (!fam) {
      L->fams.push_back(Family{e.family});
      fam = &L->fams.back();
    }
    fam->launches += 1;
    fam->ms += ms;
    fam->flops += e.flops;
    fam->bytes += e.bytes;
  }
  L->pending.clear();
  L->ev_next = 0;
  int k = 0;
  for (auto& fm : L->fams) {
    if (k >= cap || !out) break;
    std::memset(&out[k], 0, sizeof(mgt_kernel_stat));
    std::snprintf(out[k].name, sizeof(out[k].name), "%s", fm.name.c_str());
    out[k].launches = fm.launches;
    out[k].ms = fm.ms;
    out[k].flops = fm.flops;
    out[k].bytes = fm.bytes;
    ++k;
  }
  *n = k;
  L->fams.clear();
  return MGT_OK;
}

void mgt_layer_destroy(mgt_layer* L) {
  if (!L) return;
  for (auto& ev : L->ev_pool) cudaEventDestroy(ev);
  for (auto& ev : L->ev_fork)
    if (ev) cudaEventDestroy(ev);
  if (L->ev_join) cudaEventDestroy(L->ev_join);
  if (L->side) cudaStreamDestroy(L->side);
  delete L;
}

mgt_status mgt_debug_bounded_wait(int64_t limit_ns, int32_t* status, void* stream) {
  if (!status || limit_ns <= 0 || limit_ns > 1000000000LL) return MGT_EINVAL;
  return cuda_status(launch_bounded_wait_probe(reinterpret_cast<int*>(status),
                                               (unsigned long long)limit_ns,
                                               static_cast<cudaStream_t>(stream)));
}

mgt_status mgt_debug_exp2(int32_t path, int64_t n, const float* x, float* y, void* stream) {
  if (n < 0 || (n && (!x || !y)) || (path != 0 && path != 1)) return MGT_EINVAL;
  if (n == 0) return MGT_OK;
  return cuda_status(launch_exp2_probe(path, n, x, y, static_cast<cudaStream_t>(stream)));
}

mgt_status mgt_layer_status_word(mgt_layer* L, void* workspace, int32_t** word) {
  if (!L || !workspace || !word) return MGT_EINVAL;
  *word = reinterpret_cast<int32_t*>(sp(workspace, L->ws[MGT_WS_STATUS - 64]));
  return MGT_OK;
}

mgt_status mgt_gemm_bf16(int32_t M, int32_t N, int32_t K, int32_t a_mn_major, int32_t b_mn_major,
                         const void* A, int64_t lda, const void* B, int64_t ldb, float* C,
                         int64_t ldc, int32_t* status, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0 || !A || !B || !C || !status) return MGT_EINVAL;
  if (lda % 8 || ldb % 8 || !aligned16(A) || !aligned16(B) || !aligned16(C) || ldc % 4)
    return MGT_EUNSUPPORTED;
  if (lda < (a_mn_major ? M : K) || ldb < (b_mn_major ? N : K) || ldc < N) return MGT_EINVAL;
  int dev = 0, nsm = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MGT_ECUDA;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return MGT_EUNSUPPORTED;
  GemmArgs a = gemm_base(M, N, 1, K, 1);
  a.a_mn = a_mn_major ? 1 : 0; a.b_mn = b_mn_major ? 1 : 0;
  a.A = A; a.lda = lda; a.B = B; a.ldb = ldb;
  a.epi = kEpiStoreF32; a.out = C; a.ldc = ldc; a.err = status;
  return cuda_status(launch_gemm_tc(a, nsm, static_cast<cudaStream_t>(stream)));
}

mgt_status mgt_fp8_quantize(int32_t dtype, int64_t n, const void* x, uint8_t* q, float* scales,
                            void* stream) {
  if (n < 1 || !x || !q || !scales) return MGT_EINVAL;
  if (dtype != MGT_F32 && dtype != MGT_BF16) return MGT_EUNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(q) & 1) return MGT_EUNSUPPORTED;
  return cuda_status(launch_fp8_quantize(dtype == MGT_BF16 ? 1 : 0, n, x, q, scales,
                                         static_cast<cudaStream_t>(stream)));
}

mgt_status mgt_gemm_fp8(int32_t M, int32_t N, int32_t K, const uint8_t* A, int64_t lda,
                        const uint8_t* B, int64_t ldb, const float* a_scales,
                        const float* b_scales, void* C, int32_t c_dtype, int64_t ldc,
                        int32_t* status, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0 || !A || !B || !C || !a_scales || !b_scales || !status)
    return MGT_EINVAL;
  if (c_dtype != MGT_F32 && c_dtype != MGT_BF16) return MGT_EUNSUPPORTED;
  if (lda < K || ldb < K || ldc < N) return MGT_EINVAL;
  // TMA: 16-byte aligned bases and row strides; the K coordinate steps by 128 bytes.
  if (K % 16 || lda % 16 || ldb % 16 || ldc % (c_dtype == MGT_F32 ? 4 : 8) || !aligned16(A) ||
      !aligned16(B) || !aligned16(C))
    return MGT_EUNSUPPORTED;
  int dev = 0, nsm = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MGT_ECUDA;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return MGT_EUNSUPPORTED;
  GemmArgs a = gemm_base(M, N, 1, K, 1);
  a.A = A; a.lda = lda; a.B = B; a.ldb = ldb;
  a.f8 = 1; a.a_scale = a_scales + 1; a.b_scale = b_scales + 1;
  a.epi = c_dtype == MGT_F32 ? kEpiStoreF32 : kEpiBf16;
  a.out = C; a.ldc = ldc; a.err = status;
  return cuda_status(launch_gemm_fp8(a, nsm, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
