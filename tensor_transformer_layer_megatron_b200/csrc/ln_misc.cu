// Memory-bound kernels: LayerNorm forward/backward, column sums (bias gradients), and the
// fp32 SIMT GEMM used by the fp32 layer.
//
// LayerNorm statistics are taken over the whole hidden row: the trdm.cn page, section 3.2,
// requires the normalisation statistics to agree across the tensor-parallel group; the LN input
// is replicated on every shard under the column/row split, so each shard's statistics already
// are the global ones. The page's section 4.2 motivates one fused kernel per LayerNorm (launch
// overhead of unfused norms at short sequences).
#include "mgt_device.cuh"

namespace mgt {
namespace {

// ---------------------------------------------------------------------------- vector I/O
// VEC elements per 16-byte access: 8 for bf16, 4 for fp32.
template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = bf16_lo(ww[j]);
      v[2 * j + 1] = bf16_hi(ww[j]);
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = w;
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float (&v)[4]) {
    const float4 w = *reinterpret_cast<const float4*>(p);
    v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
  }
  __device__ static void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();  // protect `red` from the previous use
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) s += red[i];
  return s;
}

// ---------------------------------------------------------------------------- LN forward
// One CTA of NT threads per row; each thread keeps up to MAXV 16-byte vectors of the row in
// registers, so the row is read once: mean, then the centred second moment (two passes over
// registers, no cancellation), then the normalised, affine output.
template <typename T, int NT, int MAXV>
__global__ void __launch_bounds__(NT) ln_fwd_kernel(long long rows, int h, float eps,
                                                    const T* __restrict__ x,
                                                    const float* __restrict__ gamma,
                                                    const float* __restrict__ beta,
                                                    T* __restrict__ y, float* __restrict__ mean,
                                                    float* __restrict__ rstd) {
  constexpr int V = Vec<T>::N;
  __shared__ float red[NT / 32];
  const long long row = blockIdx.x;
  const T* xr = x + row * h;
  const int nvec = h / V;
  float v[MAXV][V];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = threadIdx.x + i * NT;
    if (vi < nvec) {
      Vec<T>::load(xr + vi * V, v[i]);
#pragma unroll
      for (int j = 0; j < V; ++j) s += v[i][j];
    }
  }
  const float mu = block_sum<NT>(s, red) / h;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = threadIdx.x + i * NT;
    if (vi < nvec) {
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const float c = v[i][j] - mu;
        q += c * c;
      }
    }
  }
  const float var = block_sum<NT>(q, red) / h;
  const float rs = rsqrtf(var + eps);
  T* yr = y + row * h;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = threadIdx.x + i * NT;
    if (vi < nvec) {
      float o[V];
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int c = vi * V + j;
        o[j] = (v[i][j] - mu) * rs * __ldg(gamma + c) + __ldg(beta + c);
      }
      Vec<T>::store(yr + vi * V, o);
    }
  }
  if (threadIdx.x == 0) {
    mean[row] = mu;
    rstd[row] = rs;
  }
}

// ---------------------------------------------------------------------------- LN backward
// CTA b handles rows b, b+grid, ...; thread columns are fixed, so each thread accumulates its
// columns' dgamma = sum dy*xhat and dbeta = sum dy across its rows in registers and writes one
// partial row per CTA. dx = rstd*(g - mean(g) - xhat*mean(g*xhat)) + dres with g = dy*gamma.
// The second pass re-reads x and dy (an L1/L2 hit) instead of holding them in registers.
template <typename T, int NT, int MAXV>
__global__ void __launch_bounds__(NT) ln_bwd_kernel(long long rows, int h,
                                                    const T* __restrict__ dy,
                                                    const T* __restrict__ dres,
                                                    const T* __restrict__ x,
                                                    const float* __restrict__ gamma,
                                                    const float* __restrict__ mean,
                                                    const float* __restrict__ rstd,
                                                    T* __restrict__ dx,
                                                    float* __restrict__ partial) {
  constexpr int V = Vec<T>::N;
  __shared__ float red[NT / 32];
  const int nvec = h / V;
  float dg[MAXV][V], db[MAXV][V];
#pragma unroll
  for (int i = 0; i < MAXV; ++i)
#pragma unroll
    for (int j = 0; j < V; ++j) dg[i][j] = db[i][j] = 0.f;

  for (long long row = blockIdx.x; row < rows; row += gridDim.x) {
    const float mu = mean[row], rs = rstd[row];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int vi = threadIdx.x + i * NT;
      if (vi < nvec) {
        float xv[V], dv[V];
        Vec<T>::load(x + row * h + vi * V, xv);
        Vec<T>::load(dy + row * h + vi * V, dv);
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const float xh = (xv[j] - mu) * rs;
          const float g = dv[j] * __ldg(gamma + vi * V + j);
          s1 += g;
          s2 += g * xh;
          dg[i][j] += dv[j] * xh;
          db[i][j] += dv[j];
        }
      }
    }
    const float m1 = block_sum<NT>(s1, red) / h;
    const float m2 = block_sum<NT>(s2, red) / h;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int vi = threadIdx.x + i * NT;
      if (vi < nvec) {
        float xv[V], dv[V], r[V], o[V];
        Vec<T>::load(x + row * h + vi * V, xv);
        Vec<T>::load(dy + row * h + vi * V, dv);
        if (dres) {
          Vec<T>::load(dres + row * h + vi * V, r);
        } else {
#pragma unroll
          for (int j = 0; j < V; ++j) r[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const float xh = (xv[j] - mu) * rs;
          const float g = dv[j] * __ldg(gamma + vi * V + j);
          o[j] = rs * (g - m1 - xh * m2) + r[j];
        }
        Vec<T>::store(dx + row * h + vi * V, o);
      }
    }
  }
  float* pg = partial + (long long)blockIdx.x * 2 * h;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = threadIdx.x + i * NT;
    if (vi < nvec) {
#pragma unroll
      for (int j = 0; j < V; ++j) {
        pg[vi * V + j] = dg[i][j];
        pg[h + vi * V + j] = db[i][j];
      }
    }
  }
}

// dgamma[c] = sum_b partial[b][0][c]; dbeta[c] = sum_b partial[b][1][c] (fixed order).
__global__ void ln_param_reduce_kernel(int h, int nblk, const float* __restrict__ partial,
                                       float* __restrict__ dgamma, float* __restrict__ dbeta) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= 2 * h) return;
  const int which = c / h, col = c % h;
  float s = 0.f;
  for (int b = 0; b < nblk; ++b) s += partial[(long long)b * 2 * h + which * h + col];
  (which ? dbeta : dgamma)[col] = s;
}

// ---------------------------------------------------------------------------- column sums
// out[c] = sum_r x[r, c]. Block = 32 x 8 threads covering 32*VEC columns; blockIdx.y splits
// the rows; partial sums are combined with fp32 atomics into a zeroed `out`.
template <typename T>
__global__ void __launch_bounds__(256) colsum_kernel(long long rows, int cols,
                                                     const T* __restrict__ x,
                                                     float* __restrict__ out, long long rows_per) {
  constexpr int V = Vec<T>::N;
  __shared__ float red[8][32 * V + 1];
  const int c0 = (blockIdx.x * 32 + threadIdx.x) * V;
  const long long r0 = blockIdx.y * rows_per;
  const long long r1 = min(rows, r0 + rows_per);
  float acc[V];
#pragma unroll
  for (int j = 0; j < V; ++j) acc[j] = 0.f;
  if (c0 < cols) {
    for (long long r = r0 + threadIdx.y; r < r1; r += 8) {
      float v[V];
      Vec<T>::load(x + r * cols + c0, v);
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] += v[j];
    }
  }
#pragma unroll
  for (int j = 0; j < V; ++j) red[threadIdx.y][threadIdx.x * V + j] = acc[j];
  __syncthreads();
  const int t = threadIdx.y * 32 + threadIdx.x;
  for (int cc = t; cc < 32 * V; cc += 256) {
    const int col = blockIdx.x * 32 * V + cc;
    if (col < cols) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) s += red[k][cc];
      atomicAdd(out + col, s);
    }
  }
}

// ---------------------------------------------------------------------------- fp32 GEMM
// One thread per output element; exact GemmArgs semantics (see mgt_internal.h). Used for the
// fp32 layer only, where the sizes are tiny and 1e-4 relative accuracy rules out TF32.
__global__ void gemm_simt_f32_kernel(const GemmArgs a) {
  const long long total = (long long)a.NG * a.M * a.Ng;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int ng = (int)(idx / ((long long)a.M * a.Ng));
  const long long r = idx - (long long)ng * a.M * a.Ng;
  const int m = (int)(r / a.Ng), n = (int)(r % a.Ng);
  const float* A = reinterpret_cast<const float*>(a.A);
  const float* B = reinterpret_cast<const float*>(a.B);
  float acc = 0.f;
  for (int kg = 0; kg < a.KG; ++kg) {
    for (int kk = 0; kk < a.Kg; ++kk) {
      const long long k = (long long)kg * a.Kg + kk;
      const float av = a.a_mn ? A[k * a.lda + m] : A[(long long)m * a.lda + k];
      const float bv = a.b_mn ? B[(long long)ng * a.b_ngs + k * a.ldb + n]
                              : B[(long long)kg * a.b_kgs + (long long)n * a.ldb + kk];
      acc = fmaf(av, bv, acc);
    }
  }
  const int col = ng * a.Ng + n;
  const long long off = (long long)(col / a.out_ng) * a.out_gs + (long long)m * a.ldc +
                        col % a.out_ng;
  float* out = reinterpret_cast<float*>(a.out);
  const float* bias = reinterpret_cast<const float*>(a.bias);
  switch (a.epi) {
    case kEpiStoreF32: out[off] = acc; break;
    case kEpiBf16: {
      if (bias) acc += bias[col];
      if (a.res) acc += reinterpret_cast<const float*>(a.res)[(long long)m * a.ldr + col];
      out[off] = acc;
      break;
    }
    case kEpiGelu: {
      if (bias) acc += bias[col];
      reinterpret_cast<float*>(a.out2)[off] = acc;
      out[off] = gelu_f(acc, a.gelu_tanh);
      break;
    }
    case kEpiDGelu: {
      const float u = reinterpret_cast<const float*>(a.aux)[(long long)m * a.ld_aux + col];
      out[off] = acc * gelu_grad_f(u, a.gelu_tanh);
      break;
    }
  }
}

template <typename T, int NT, int MAXV>
cudaError_t ln_fwd_inst(long long rows, int h, float eps, const void* x, const float* g,
                        const float* b, void* y, float* mean, float* rstd, cudaStream_t s) {
  ln_fwd_kernel<T, NT, MAXV><<<(unsigned)rows, NT, 0, s>>>(
      rows, h, eps, reinterpret_cast<const T*>(x), g, b, reinterpret_cast<T*>(y), mean, rstd);
  return cudaGetLastError();
}

template <typename T, int NT, int MAXV>
cudaError_t ln_bwd_inst(long long rows, int h, const void* dy, const void* dres, const void* x,
                        const float* g, const float* mean, const float* rstd, void* dx,
                        float* partial, int nblk, cudaStream_t s) {
  ln_bwd_kernel<T, NT, MAXV><<<nblk, NT, 0, s>>>(
      rows, h, reinterpret_cast<const T*>(dy), reinterpret_cast<const T*>(dres),
      reinterpret_cast<const T*>(x), g, mean, rstd, reinterpret_cast<T*>(dx), partial);
  return cudaGetLastError();
}

}  // namespace

// Threads per row: enough 16-byte vectors per thread to cover h (forward: up to 256 threads
// x 8 vectors; backward: up to 512 threads x 4 vectors). bf16: h <= 16384; fp32: h <= 8192.
cudaError_t launch_ln_fwd(int dtype, long long rows, int h, float eps, const void* x,
                          const float* gamma, const float* beta, void* y, float* mean,
                          float* rstd, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int V = dtype ? 8 : 4;
  const int nvec = h / V;
  if (nvec <= 32 * 2)
    return dtype ? ln_fwd_inst<__nv_bfloat16, 32, 2>(rows, h, eps, x, gamma, beta, y, mean, rstd, s)
                 : ln_fwd_inst<float, 32, 2>(rows, h, eps, x, gamma, beta, y, mean, rstd, s);
  if (nvec <= 128 * 4)
    return dtype ? ln_fwd_inst<__nv_bfloat16, 128, 4>(rows, h, eps, x, gamma, beta, y, mean, rstd, s)
                 : ln_fwd_inst<float, 128, 4>(rows, h, eps, x, gamma, beta, y, mean, rstd, s);
  return dtype ? ln_fwd_inst<__nv_bfloat16, 256, 8>(rows, h, eps, x, gamma, beta, y, mean, rstd, s)
               : ln_fwd_inst<float, 256, 8>(rows, h, eps, x, gamma, beta, y, mean, rstd, s);
}

int ln_bwd_blocks(long long rows, int num_sms) {
  long long n = 2LL * num_sms;
  if (n > rows) n = rows;
  return n < 1 ? 1 : (int)n;
}

cudaError_t launch_ln_bwd(int dtype, long long rows, int h, const void* dy, const void* dres,
                          const void* x, const float* gamma, const float* mean,
                          const float* rstd, void* dx, float* partial, int nblk, float* dgamma,
                          float* dbeta, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int V = dtype ? 8 : 4;
  const int nvec = h / V;
  cudaError_t e;
  if (nvec <= 32 * 2)
    e = dtype ? ln_bwd_inst<__nv_bfloat16, 32, 2>(rows, h, dy, dres, x, gamma, mean, rstd, dx, partial, nblk, s)
              : ln_bwd_inst<float, 32, 2>(rows, h, dy, dres, x, gamma, mean, rstd, dx, partial, nblk, s);
  else if (nvec <= 128 * 4)
    e = dtype ? ln_bwd_inst<__nv_bfloat16, 128, 4>(rows, h, dy, dres, x, gamma, mean, rstd, dx, partial, nblk, s)
              : ln_bwd_inst<float, 128, 4>(rows, h, dy, dres, x, gamma, mean, rstd, dx, partial, nblk, s);
  else
    e = dtype ? ln_bwd_inst<__nv_bfloat16, 512, 4>(rows, h, dy, dres, x, gamma, mean, rstd, dx, partial, nblk, s)
              : ln_bwd_inst<float, 512, 4>(rows, h, dy, dres, x, gamma, mean, rstd, dx, partial, nblk, s);
  if (e != cudaSuccess) return e;
  ln_param_reduce_kernel<<<(2 * h + 255) / 256, 256, 0, s>>>(h, nblk, partial, dgamma, dbeta);
  return cudaGetLastError();
}

cudaError_t launch_colsum(int dtype, long long rows, int cols, const void* x, float* out,
                          cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * cols, s);
  if (e != cudaSuccess || rows <= 0) return e;
  const int V = dtype ? 8 : 4;
  const int cb = (cols + 32 * V - 1) / (32 * V);
  long long splits = (2 * 148 + cb - 1) / cb;  // aim for >= 2 blocks per SM
  if (splits > (rows + 7) / 8) splits = (rows + 7) / 8;
  if (splits < 1) splits = 1;
  const long long rows_per = (rows + splits - 1) / splits;
  dim3 grid(cb, (unsigned)splits), block(32, 8);
  if (dtype)
    colsum_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
        rows, cols, reinterpret_cast<const __nv_bfloat16*>(x), out, rows_per);
  else
    colsum_kernel<float><<<grid, block, 0, s>>>(rows, cols, reinterpret_cast<const float*>(x),
                                                 out, rows_per);
  return cudaGetLastError();
}

cudaError_t launch_gemm_simt_f32(const GemmArgs& a, cudaStream_t s) {
  const long long total = (long long)a.NG * a.M * a.Ng;
  if (total <= 0) return cudaSuccess;
  gemm_simt_f32_kernel<<<(unsigned)((total + 127) / 128), 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mgt
