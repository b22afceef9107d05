// Causal multi-head attention, forward and backward, on the packed qkv of the column-parallel
// QKV projection: qkv [T][p][3][H/p][d]. Each logical shard owns whole heads, so every head's
// softmax is local (the trdm.cn page, section 2.1: column-split Q/K/V let each shard compute its
// heads without communication). Softmax arithmetic is fp32 (section 3.2,
// attention_softmax_in_fp32). Scale 1/sqrt(d); key j visible to query i iff j <= i.
//
// bf16 path: forward and backward run on tcgen05 (attn_tc.cu). The backward recomputes the
// probabilities from the saved log-sum-exp (the page's section 4.1 recompute).
// fp32 path: plain per-row kernels (tiny shapes only).
#include "mgt_device.cuh"

namespace mgt {
namespace {

// ============================================================================ fp32 kernels
// One thread per (batch, head, query): online softmax over keys 0..i.
template <int DMAX>
__global__ void attn_fwd_f32_kernel(AttnArgs a) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= a.b * a.H * a.s) return;
  const int i = idx % a.s, n = (idx / a.s) % a.H, b = idx / (a.s * a.H);
  const int hp = a.H / a.p, t = n / hp, j = n % hp, d = a.d;
  const long long ld = 3LL * a.H * d;
  const float* base = reinterpret_cast<const float*>(a.qkv) + (long long)b * a.s * ld +
                      (long long)t * 3 * hp * d + (long long)j * d;
  const float* q = base + (long long)i * ld;
  const float* k = base + (long long)hp * d;
  const float* v = base + 2LL * hp * d;
  const float scale = rsqrtf((float)d);
  float o[DMAX];
  for (int c = 0; c < d; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int jj = 0; jj <= i; ++jj) {
    float sdot = 0.f;
    for (int c = 0; c < d; ++c) sdot += q[c] * k[(long long)jj * ld + c];
    sdot *= scale;
    const float mn = fmaxf(m, sdot);
    const float alpha = expf(m - mn), pj = expf(sdot - mn);
    l = l * alpha + pj;
    for (int c = 0; c < d; ++c) o[c] = o[c] * alpha + pj * v[(long long)jj * ld + c];
    m = mn;
  }
  float* orow = reinterpret_cast<float*>(a.o) + ((long long)b * a.s + i) * a.H * d + n * d;
  for (int c = 0; c < d; ++c) orow[c] = o[c] / l;
  a.lse[((long long)b * a.H + n) * a.s + i] = m + logf(l);
}

// One thread per (batch, head, query i): P_ij recomputed from lse; dq_i accumulated locally;
// dk_j, dv_j scattered with atomics into the zeroed fp32 dqkv.
template <int DMAX>
__global__ void attn_bwd_f32_kernel(AttnArgs a) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= a.b * a.H * a.s) return;
  const int i = idx % a.s, n = (idx / a.s) % a.H, b = idx / (a.s * a.H);
  const int hp = a.H / a.p, t = n / hp, j = n % hp, d = a.d;
  const long long ld = 3LL * a.H * d;
  const long long off = (long long)b * a.s * ld + (long long)t * 3 * hp * d + (long long)j * d;
  const float* base = reinterpret_cast<const float*>(a.qkv) + off;
  float* dbase = reinterpret_cast<float*>(a.dqkv) + off;
  const float* q = base + (long long)i * ld;
  const float* k = base + (long long)hp * d;
  const float* v = base + 2LL * hp * d;
  const long long orow = ((long long)b * a.s + i) * a.H * d + n * d;
  const float* o = reinterpret_cast<const float*>(a.o) + orow;
  const float* dO = reinterpret_cast<const float*>(a.dO) + orow;
  const float scale = rsqrtf((float)d);
  const float lse = a.lse[((long long)b * a.H + n) * a.s + i];
  float D = 0.f;
  for (int c = 0; c < d; ++c) D += dO[c] * o[c];
  float dq[DMAX];
  for (int c = 0; c < d; ++c) dq[c] = 0.f;
  for (int jj = 0; jj <= i; ++jj) {
    float sdot = 0.f, dp = 0.f;
    for (int c = 0; c < d; ++c) {
      sdot += q[c] * k[(long long)jj * ld + c];
      dp += dO[c] * v[(long long)jj * ld + c];
    }
    const float p = expf(sdot * scale - lse);
    const float ds = p * (dp - D);
    for (int c = 0; c < d; ++c) {
      dq[c] += ds * k[(long long)jj * ld + c];
      atomicAdd(dbase + (long long)hp * d + (long long)jj * ld + c, ds * scale * q[c]);
      atomicAdd(dbase + 2LL * hp * d + (long long)jj * ld + c, p * dO[c]);
    }
  }
  for (int c = 0; c < d; ++c) dbase[(long long)i * ld + c] = dq[c] * scale;
}

}  // namespace

cudaError_t launch_attn_fwd(int dtype, const AttnArgs& a, cudaStream_t s) {
  if (dtype == 0) {
    const int total = a.b * a.H * a.s;
    attn_fwd_f32_kernel<64><<<(total + 127) / 128, 128, 0, s>>>(a);
    return cudaGetLastError();
  }
  return launch_attn_fwd_tc(a, s);  // tcgen05 kernel (attn_tc.cu)
}

cudaError_t launch_attn_bwd(int dtype, const AttnArgs& a, cudaStream_t s) {
  if (dtype == 0) {
    const long long T = (long long)a.b * a.s;
    cudaError_t e = cudaMemsetAsync(a.dqkv, 0, sizeof(float) * T * 3 * a.H * a.d, s);
    if (e != cudaSuccess) return e;
    const int total = a.b * a.H * a.s;
    attn_bwd_f32_kernel<64><<<(total + 127) / 128, 128, 0, s>>>(a);
    return cudaGetLastError();
  }
  return launch_attn_bwd_tc(a, s);  // dQ (with D) then dK/dV kernels on tcgen05 (attn_tc.cu)
}


}  // namespace mgt
