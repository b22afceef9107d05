// Memory-bound kernels: LayerNorm forward/backward, column sums (bias gradients), and the
// fp32 SIMT GEMM used by the fp32 layer.
//
// LayerNorm statistics are taken over the whole hidden row: the trdm.cn page, section 3.2,
// requires the normalisation statistics to agree across the tensor-parallel group; the LN input
// is replicated on every shard under the column/row split, so each shard's statistics already
// are the global ones. The page's section 4.2 motivates one fused kernel per LayerNorm (launch
// overhead of unfused norms at short sequences).
#include <mutex>

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
  __device__ static void unpack(const uint4& w, float (&v)[8]) {
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
  __device__ static void unpack(const uint4& w, float (&v)[4]) {
    v[0] = __uint_as_float(w.x); v[1] = __uint_as_float(w.y);
    v[2] = __uint_as_float(w.z); v[3] = __uint_as_float(w.w);
  }
  __device__ static void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

// V consecutive fp32 parameters (gamma or beta) with 16-byte loads; the column index is a
// multiple of V, so the address is 16-byte aligned.
template <int V>
__device__ __forceinline__ void load_param(const float* __restrict__ p, int c, float (&v)[V]) {
#pragma unroll
  for (int j = 0; j < V; j += 4) {
    const float4 w = __ldg(reinterpret_cast<const float4*>(p + c + j));
    v[j] = w.x; v[j + 1] = w.y; v[j + 2] = w.z; v[j + 3] = w.w;
  }
}

// ---------------------------------------------------------------------------- row groups
// A row is owned by a group of W warps (W*32 threads); a 256-thread CTA holds 8/W groups. Sums
// over the row are warp shuffles, then (W > 1) a named barrier private to the group, so groups
// that process different numbers of rows never wait on each other.
template <int W>
__device__ __forceinline__ float group_sum(float v, float* red, int grp, int wg) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if constexpr (W == 1) {
    return v;
  } else {
    const int lane = threadIdx.x & 31;
    if (lane == 0) red[grp * W + wg] = v;
    asm volatile("bar.sync %0, %1;" ::"r"(grp + 1), "r"(W * 32) : "memory");
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < W; ++i) s += red[grp * W + i];
    asm volatile("bar.sync %0, %1;" ::"r"(grp + 1), "r"(W * 32) : "memory");  // red reusable
    return s;
  }
}

// ---------------------------------------------------------------------------- LN forward
// Each group reads its row once into registers (up to VPL 16-byte vectors per thread), takes
// the mean, then the centred second moment (two passes over registers, no cancellation), and
// writes the normalised, affine output.
template <typename T, int W, int VPL>
__global__ void __launch_bounds__(256) ln_fwd_kernel(long long rows, int h, float eps,
                                                     const T* __restrict__ x,
                                                     const float* __restrict__ gamma,
                                                     const float* __restrict__ beta,
                                                     T* __restrict__ y, float* __restrict__ mean,
                                                     float* __restrict__ rstd) {
  constexpr int V = Vec<T>::N, G = 8 / W, GT = 32 * W;
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, grp = warp / W, wg = warp % W;
  const int t = wg * 32 + (threadIdx.x & 31);
  const long long row = (long long)blockIdx.x * G + grp;
  const bool valid = row < rows;
  const int nvec = h / V;
  const T* xr = x + (valid ? row : 0) * h;
  float v[VPL][V];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = t + i * GT;
    if (valid && vi < nvec) {
      Vec<T>::load(xr + vi * V, v[i]);
#pragma unroll
      for (int j = 0; j < V; ++j) s += v[i][j];
    }
  }
  const float mu = group_sum<W>(s, red, grp, wg) / h;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = t + i * GT;
    if (valid && vi < nvec) {
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const float c = v[i][j] - mu;
        q += c * c;
      }
    }
  }
  const float var = group_sum<W>(q, red, grp, wg) / h;
  const float rs = rsqrtf(var + eps);
  if (!valid) return;
  T* yr = y + row * h;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = t + i * GT;
    if (vi < nvec) {
      float o[V], gv[V], bv[V];
      load_param<V>(gamma, vi * V, gv);
      load_param<V>(beta, vi * V, bv);
#pragma unroll
      for (int j = 0; j < V; ++j) o[j] = (v[i][j] - mu) * rs * gv[j] + bv[j];
      Vec<T>::store(yr + vi * V, o);
    }
  }
  if (t == 0) {
    mean[row] = mu;
    rstd[row] = rs;
  }
}

// ---------------------------------------------------------------------------- LN backward
// dx for one row per group, every row in flight at once (no accumulators across rows):
//   g = dy*gamma, dx = rstd*(g - mean(g) - xhat*mean(g*xhat)) + dres.
template <typename T, int W, int VPL>
__global__ void __launch_bounds__(256) ln_bwd_dx_kernel(long long rows, int h,
                                                        const T* __restrict__ dy,
                                                        const T* __restrict__ dres,
                                                        const T* __restrict__ x,
                                                        const float* __restrict__ gamma,
                                                        const float* __restrict__ mean,
                                                        const float* __restrict__ rstd,
                                                        T* __restrict__ dx) {
  constexpr int V = Vec<T>::N, G = 8 / W, GT = 32 * W;
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, grp = warp / W, wg = warp % W;
  const int t = wg * 32 + (threadIdx.x & 31);
  const long long row = (long long)blockIdx.x * G + grp;
  const bool valid = row < rows;
  const long long r = valid ? row : 0;
  const int nvec = h / V;
  const float mu = mean[r], rs = rstd[r];
  float xh[VPL][V], g[VPL][V];
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = t + i * GT;
    if (valid && vi < nvec) {
      float xv[V], dv[V], gv[V];
      Vec<T>::load(x + r * h + vi * V, xv);
      Vec<T>::load(dy + r * h + vi * V, dv);
      load_param<V>(gamma, vi * V, gv);
#pragma unroll
      for (int j = 0; j < V; ++j) {
        xh[i][j] = (xv[j] - mu) * rs;
        g[i][j] = dv[j] * gv[j];
        s1 += g[i][j];
        s2 += g[i][j] * xh[i][j];
      }
    }
  }
  const float m1 = group_sum<W>(s1, red, grp, wg) / h;
  const float m2 = group_sum<W>(s2, red, grp, wg) / h;
  if (!valid) return;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = t + i * GT;
    if (vi < nvec) {
      float rv[V], o[V];
      if (dres) {
        Vec<T>::load(dres + r * h + vi * V, rv);
      } else {
#pragma unroll
        for (int j = 0; j < V; ++j) rv[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < V; ++j) o[j] = rs * (g[i][j] - m1 - xh[i][j] * m2) + rv[j];
      Vec<T>::store(dx + r * h + vi * V, o);
    }
  }
}

// dx and the parameter partials in one pass over x, dy and dres (rows up to 512 16-byte vectors).
// The block walks a contiguous slice of rows one row at a time with all 256 threads (thread t
// owns the column vectors t, t + 256, ...), loading the next row's x, dy, dres and statistics
// while it reduces the current one. Every column belongs to one thread, so dgamma = sum dy*xhat,
// dbeta = sum dy and (NSUM = 3) sum dres accumulate in registers and leave as one partial row
// set per block, partial[slice][NSUM][h], for ln_param_reduce_kernel (fixed order).
template <typename T, int VPL, int NSUM>
__global__ void __launch_bounds__(256, 2) ln_bwd_fused_kernel(long long rows, int h,
                                                           const T* __restrict__ dy,
                                                           const T* __restrict__ dres,
                                                           const T* __restrict__ x,
                                                           const float* __restrict__ gamma,
                                                           const float* __restrict__ mean,
                                                           const float* __restrict__ rstd,
                                                           T* __restrict__ dx,
                                                           float* __restrict__ partial,
                                                           long long rows_per) {
  constexpr int V = Vec<T>::N;
  __shared__ float2 red[2][8];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int nvec = h / V;
  const long long r0 = (long long)blockIdx.x * rows_per;
  const long long r1 = min(rows, r0 + rows_per);
  const float inv_h = 1.f / (float)h;
  // gamma is re-read (from L1) at each use rather than held: registers go to the accumulators
  // and the prefetched row.
  float ag[VPL][V], ab[VPL][V], ar[VPL][V];
#pragma unroll
  for (int i = 0; i < VPL; ++i)
#pragma unroll
    for (int j = 0; j < V; ++j) ag[i][j] = ab[i][j] = ar[i][j] = 0.f;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  uint4 cx[VPL], cd[VPL], cr[VPL];
  float cmu = 0.f, crs = 0.f;
  auto load_row = [&](long long r, uint4 (&px)[VPL], uint4 (&pd)[VPL], uint4 (&pr)[VPL],
                      float& mu, float& rs) {
    mu = mean[r];
    rs = rstd[r];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = t + i * 256;
      const bool ok = vi < nvec;
      px[i] = ok ? *reinterpret_cast<const uint4*>(x + r * h + vi * V) : zero;
      pd[i] = ok ? *reinterpret_cast<const uint4*>(dy + r * h + vi * V) : zero;
      pr[i] = (ok && dres) ? *reinterpret_cast<const uint4*>(dres + r * h + vi * V) : zero;
    }
  };
  if (r0 < r1) load_row(r0, cx, cd, cr, cmu, crs);
  int par = 0;
  for (long long r = r0; r < r1; ++r, par ^= 1) {
    uint4 nx[VPL], nd[VPL], nr[VPL];
    float nmu = 0.f, nrs = 0.f;
    if (r + 1 < r1) load_row(r + 1, nx, nd, nr, nmu, nrs);
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = t + i * 256;
      float xv[V], dv[V], gv[V];
      Vec<T>::unpack(cx[i], xv);
      Vec<T>::unpack(cd[i], dv);
      if (vi < nvec) {
        load_param<V>(gamma, vi * V, gv);
      } else {
#pragma unroll
        for (int j = 0; j < V; ++j) gv[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const float xh = (xv[j] - cmu) * crs, g = dv[j] * gv[j];
        s1 += g;
        s2 += g * xh;
        ag[i][j] += dv[j] * xh;
        ab[i][j] += dv[j];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    // Two buffers by row parity: a buffer is rewritten two rows later, after every thread has
    // passed the next row's barrier and so has finished reading it.
    if (lane == 0) red[par][warp] = make_float2(s1, s2);
    __syncthreads();
    float S1 = 0.f, S2 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 v = red[par][k];
      S1 += v.x;
      S2 += v.y;
    }
    const float m1 = S1 * inv_h, m2 = S2 * inv_h;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = t + i * 256;
      if (vi < nvec) {
        float xv[V], dv[V], rv[V], gv[V], o[V];
        Vec<T>::unpack(cx[i], xv);
        Vec<T>::unpack(cd[i], dv);
        Vec<T>::unpack(cr[i], rv);
        load_param<V>(gamma, vi * V, gv);
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const float xh = (xv[j] - cmu) * crs, g = dv[j] * gv[j];
          o[j] = crs * (g - m1 - xh * m2) + rv[j];
          if constexpr (NSUM == 3) ar[i][j] += rv[j];
        }
        Vec<T>::store(dx + r * h + vi * V, o);
      }
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      cx[i] = nx[i];
      cd[i] = nd[i];
      cr[i] = nr[i];
    }
    cmu = nmu;
    crs = nrs;
  }
  float* pg = partial + (long long)blockIdx.x * NSUM * h;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = t + i * 256;
    if (vi < nvec) {
#pragma unroll
      for (int j = 0; j < V; j += 4) {
        *reinterpret_cast<float4*>(pg + vi * V + j) =
            make_float4(ag[i][j], ag[i][j + 1], ag[i][j + 2], ag[i][j + 3]);
        *reinterpret_cast<float4*>(pg + h + vi * V + j) =
            make_float4(ab[i][j], ab[i][j + 1], ab[i][j + 2], ab[i][j + 3]);
        if constexpr (NSUM == 3)
          *reinterpret_cast<float4*>(pg + 2 * h + vi * V + j) =
              make_float4(ar[i][j], ar[i][j + 1], ar[i][j + 2], ar[i][j + 3]);
      }
    }
  }
}

// ---------------------------------------------------------------------------- row rings
// Rows of 256 to 1024 16-byte vectors stream through a ring of S shared-memory stages filled
// by plain bulk copies (cp.async.bulk, one mbarrier per stage): one thread keeps up to S rows
// of every input in flight per block while all 256 threads reduce the current row, so far
// more bytes are in flight per SM than the registers of a row-per-group kernel can hold.
// Thread t owns the vectors t, t + 256, ... of every row. Every wait is bounded; on a timeout
// the block records it, waits (bounded) for its copies in flight and leaves.
constexpr int kRingStages = 4;

// Wait for the copies of local rows [i, min(n, i + S)) that are still in flight.
template <int S>
__device__ __forceinline__ void ring_drain(uint64_t* full, long long i, long long n, int* err) {
  for (long long j = i; j < n && j < i + S; ++j)
    mbar_wait(&full[j % S], (uint32_t)((j / S) & 1), err, kErrTimeoutDrain, nullptr);
}

// LayerNorm forward, one row per block iteration; rows r = blockIdx.x + i * gridDim.x. gamma
// and beta of the thread's columns are loaded once per block.
template <typename T, int VPL, int S>
__global__ void __launch_bounds__(256) ln_fwd_ring_kernel(long long rows, int h, float eps,
                                                          const T* __restrict__ x,
                                                          const float* __restrict__ gamma,
                                                          const float* __restrict__ beta,
                                                          T* __restrict__ y,
                                                          float* __restrict__ mean,
                                                          float* __restrict__ rstd, int* err) {
  grid_dependency_wait();
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[S];
  __shared__ float red[2][8];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int nvec = h / V;
  const uint32_t row_bytes = (uint32_t)h * sizeof(T);
  const long long nloc =
      (long long)blockIdx.x < rows ? (rows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (t == 0) {
    for (int k = 0; k < S; ++k) mbar_init(&full[k], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](long long i) {
    const int st = (int)(i % S);
    const long long r = blockIdx.x + i * gridDim.x;
    mbar_arrive_expect_tx(&full[st], row_bytes);
    bulk_load_1d(ring + (size_t)st * row_bytes, x + r * h, row_bytes, &full[st]);
  };
  if (t == 0)
    for (long long i = 0; i < S && i < nloc; ++i) issue(i);
  float gv[VPL][V], bv[VPL][V];
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int vi = t + k * 256;
    if (vi < nvec) {
      load_param<V>(gamma, vi * V, gv[k]);
      load_param<V>(beta, vi * V, bv[k]);
    } else {
#pragma unroll
      for (int j = 0; j < V; ++j) gv[k][j] = bv[k][j] = 0.f;
    }
  }
  const float inv_h = 1.f / (float)h;
  for (long long i = 0; i < nloc; ++i) {
    const int st = (int)(i % S);
    const bool ok = mbar_wait(&full[st], (uint32_t)((i / S) & 1), err, kErrTimeoutLn, nullptr);
    const uint4* src = reinterpret_cast<const uint4*>(ring + (size_t)st * row_bytes);
    float v[VPL][V];
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = t + k * 256;
      if (ok && vi < nvec) {
        Vec<T>::unpack(src[vi], v[k]);
#pragma unroll
        for (int j = 0; j < V; ++j) sum += v[k][j];
      } else {
#pragma unroll
        for (int j = 0; j < V; ++j) v[k][j] = 0.f;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) red[0][warp] = sum;
    if (__syncthreads_or(!ok)) {
      if (t == 0) ring_drain<S>(full, i, nloc, err);
      return;
    }
    // every thread has read this stage (before the barrier): refill it
    if (t == 0 && i + S < nloc) issue(i + S);
    float mu = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) mu += red[0][w];
    mu *= inv_h;
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      if (t + k * 256 < nvec) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const float c = v[k][j] - mu;
          q += c * c;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if (lane == 0) red[1][warp] = q;
    __syncthreads();
    float var = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) var += red[1][w];
    const float rs = rsqrtf(var * inv_h + eps);
    const long long r = blockIdx.x + i * gridDim.x;
    T* yr = y + r * h;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = t + k * 256;
      if (vi < nvec) {
        float o[V];
#pragma unroll
        for (int j = 0; j < V; ++j) o[j] = (v[k][j] - mu) * rs * gv[k][j] + bv[k][j];
        Vec<T>::store(yr + vi * V, o);
      }
    }
    if (t == 0) {
      mean[r] = mu;
      rstd[r] = rs;
    }
  }
}

// LayerNorm backward over a contiguous slice of rows per block (rows_per each): dx per row and
// the parameter partials of the slice, as ln_bwd_fused_kernel, with x, dy and dres streamed
// through the ring (one stage = the three rows) instead of prefetched into registers. Rows are
// taken two at a time: the two rows' sums are reduced together, behind one block barrier, so
// the shuffle chains and the barrier of one row overlap the other's (a row alone left the SM
// mostly waiting on that chain). Each row's sums and each column's partial sums are formed in
// the same order as one row at a time, so the results do not depend on the pairing.
template <typename T, int VPL, int NSUM, int S>
__global__ void __launch_bounds__(256, 1) ln_bwd_ring_kernel(long long rows, int h,
                                                          const T* __restrict__ dy,
                                                          const T* __restrict__ dres,
                                                          const T* __restrict__ x,
                                                          const float* __restrict__ gamma,
                                                          const float* __restrict__ mean,
                                                          const float* __restrict__ rstd,
                                                          T* __restrict__ dx,
                                                          float* __restrict__ partial,
                                                          long long rows_per, int* err) {
  grid_dependency_wait();
  static_assert(S % 2 == 0, "rows are taken in pairs of stages");
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[S];
  __shared__ float4 red[2][8];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int nvec = h / V;
  const uint32_t row_bytes = (uint32_t)h * sizeof(T);
  const uint32_t stage_bytes = (dres ? 3u : 2u) * row_bytes;
  const long long r0 = (long long)blockIdx.x * rows_per;
  const long long r1 = min(rows, r0 + rows_per);
  const long long nloc = r1 > r0 ? r1 - r0 : 0;
  if (t == 0) {
    for (int k = 0; k < S; ++k) mbar_init(&full[k], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](long long i) {
    const int st = (int)(i % S);
    const long long r = r0 + i;
    uint8_t* dst = ring + (size_t)st * stage_bytes;
    mbar_arrive_expect_tx(&full[st], stage_bytes);
    bulk_load_1d(dst, x + r * h, row_bytes, &full[st]);
    bulk_load_1d(dst + row_bytes, dy + r * h, row_bytes, &full[st]);
    if (dres) bulk_load_1d(dst + 2 * row_bytes, dres + r * h, row_bytes, &full[st]);
  };
  if (t == 0)
    for (long long i = 0; i < S && i < nloc; ++i) issue(i);
  const float inv_h = 1.f / (float)h;
  float ag[VPL][V], ab[VPL][V], ar[VPL][V];
#pragma unroll
  for (int k = 0; k < VPL; ++k)
#pragma unroll
    for (int j = 0; j < V; ++j) ag[k][j] = ab[k][j] = ar[k][j] = 0.f;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  float cmu[2], crs[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    cmu[q] = q < nloc ? mean[r0 + q] : 0.f;
    crs[q] = q < nloc ? rstd[r0 + q] : 0.f;
  }
  int par = 0;
  for (long long i = 0; i < nloc; i += 2, par ^= 1) {
    const long long r = r0 + i;
    const bool two = i + 1 < nloc;  // the slice's last row may come alone
    float nmu[2], nrs[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      nmu[q] = i + 2 + q < nloc ? mean[r + 2 + q] : 0.f;
      nrs[q] = i + 2 + q < nloc ? rstd[r + 2 + q] : 0.f;
    }
    bool ok = mbar_wait(&full[i % S], (uint32_t)((i / S) & 1), err, kErrTimeoutLn, nullptr);
    if (two && ok)
      ok = mbar_wait(&full[(i + 1) % S], (uint32_t)(((i + 1) / S) & 1), err, kErrTimeoutLn,
                     nullptr);
    uint4 cx[2][VPL], cd[2][VPL], cr[2][VPL];
    float s1[2] = {0.f, 0.f}, s2[2] = {0.f, 0.f};
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = t + k * 256;
      float gv[V];
      if (vi < nvec) {
        load_param<V>(gamma, vi * V, gv);
      } else {
#pragma unroll
        for (int j = 0; j < V; ++j) gv[j] = 0.f;
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint4* sx =
            reinterpret_cast<const uint4*>(ring + (size_t)((i + q) % S) * stage_bytes);
        const uint4* sd = sx + row_bytes / 16;
        const uint4* sr = sd + row_bytes / 16;
        const bool in = ok && vi < nvec && (q == 0 || two);
        cx[q][k] = in ? sx[vi] : zero;
        cd[q][k] = in ? sd[vi] : zero;
        cr[q][k] = (in && dres) ? sr[vi] : zero;
        float xv[V], dv[V];
        Vec<T>::unpack(cx[q][k], xv);
        Vec<T>::unpack(cd[q][k], dv);
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const float xh = (xv[j] - cmu[q]) * crs[q], g = dv[j] * gv[j];
          s1[q] += g;
          s2[q] += g * xh;
          ag[k][j] += dv[j] * xh;  // a missing second row has dy = 0: it adds nothing
          ab[k][j] += dv[j];
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1[0] += __shfl_xor_sync(0xffffffffu, s1[0], o);
      s2[0] += __shfl_xor_sync(0xffffffffu, s2[0], o);
      s1[1] += __shfl_xor_sync(0xffffffffu, s1[1], o);
      s2[1] += __shfl_xor_sync(0xffffffffu, s2[1], o);
    }
    // Two buffers by pair parity: a buffer is rewritten two pairs later, after every thread
    // has passed the next pair's barrier and so has finished reading it.
    if (lane == 0) red[par][warp] = make_float4(s1[0], s2[0], s1[1], s2[1]);
    if (__syncthreads_or(!ok)) {
      if (t == 0) ring_drain<S>(full, i, nloc, err);
      return;
    }
    if (t == 0) {  // both stages have been read into registers: refill them
      if (i + S < nloc) issue(i + S);
      if (i + 1 + S < nloc) issue(i + 1 + S);
    }
    float S1[2] = {0.f, 0.f}, S2[2] = {0.f, 0.f};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const float4 v = red[par][w];
      S1[0] += v.x;
      S2[0] += v.y;
      S1[1] += v.z;
      S2[1] += v.w;
    }
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = t + k * 256;
      if (vi < nvec) {
        float gv[V];
        load_param<V>(gamma, vi * V, gv);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q == 1 && !two) break;
          const float m1 = S1[q] * inv_h, m2 = S2[q] * inv_h;
          float xv[V], dv[V], rv[V], o[V];
          Vec<T>::unpack(cx[q][k], xv);
          Vec<T>::unpack(cd[q][k], dv);
          Vec<T>::unpack(cr[q][k], rv);
#pragma unroll
          for (int j = 0; j < V; ++j) {
            const float xh = (xv[j] - cmu[q]) * crs[q], g = dv[j] * gv[j];
            o[j] = crs[q] * (g - m1 - xh * m2) + rv[j];
            if constexpr (NSUM == 3) ar[k][j] += rv[j];
          }
          Vec<T>::store(dx + (r + q) * h + vi * V, o);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      cmu[q] = nmu[q];
      crs[q] = nrs[q];
    }
  }
  float* pg = partial + (long long)blockIdx.x * NSUM * h;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int vi = t + k * 256;
    if (vi < nvec) {
#pragma unroll
      for (int j = 0; j < V; j += 4) {
        *reinterpret_cast<float4*>(pg + vi * V + j) =
            make_float4(ag[k][j], ag[k][j + 1], ag[k][j + 2], ag[k][j + 3]);
        *reinterpret_cast<float4*>(pg + h + vi * V + j) =
            make_float4(ab[k][j], ab[k][j + 1], ab[k][j + 2], ab[k][j + 3]);
        if constexpr (NSUM == 3)
          *reinterpret_cast<float4*>(pg + 2 * h + vi * V + j) =
              make_float4(ar[k][j], ar[k][j + 1], ar[k][j + 2], ar[k][j + 3]);
      }
    }
  }
}

// Partial dgamma = sum dy*xhat and dbeta = sum dy over one slice of rows, and with NSUM = 3 also
// sum dres (the residual gradient: a bias gradient of the layer for free, as the LayerNorm
// backward reads it anyway). Block = 32 x 8 threads covering 32*VEC columns; blockIdx.y is the
// slice; the 8 row lanes are combined in shared memory and written to partial[slice][NSUM][h]
// (no atomics: deterministic).
template <typename T, int NSUM>
__global__ void __launch_bounds__(256) ln_bwd_param_kernel(long long rows, int h,
                                                           const T* __restrict__ dy,
                                                           const T* __restrict__ x,
                                                           const T* __restrict__ dres,
                                                           const float* __restrict__ mean,
                                                           const float* __restrict__ rstd,
                                                           float* __restrict__ partial,
                                                           long long rows_per) {
  constexpr int V = Vec<T>::N;
  __shared__ float red[NSUM][8][32 * V + 1];
  const int c0 = (blockIdx.x * 32 + threadIdx.x) * V;
  const long long r0 = blockIdx.y * rows_per;
  const long long r1 = min(rows, r0 + rows_per);
  float ag[V], ab[V], ar[V];
#pragma unroll
  for (int j = 0; j < V; ++j) ag[j] = ab[j] = ar[j] = 0.f;
  if (c0 < h) {
    long long r = r0 + threadIdx.y;
    for (; r + 8 < r1; r += 16) {  // two independent rows in flight per thread
      float x0[V], d0[V], x1[V], d1[V];
      Vec<T>::load(x + r * h + c0, x0);
      Vec<T>::load(dy + r * h + c0, d0);
      Vec<T>::load(x + (r + 8) * h + c0, x1);
      Vec<T>::load(dy + (r + 8) * h + c0, d1);
      const float mu0 = mean[r], rs0 = rstd[r], mu1 = mean[r + 8], rs1 = rstd[r + 8];
#pragma unroll
      for (int j = 0; j < V; ++j) {
        ag[j] += d0[j] * ((x0[j] - mu0) * rs0) + d1[j] * ((x1[j] - mu1) * rs1);
        ab[j] += d0[j] + d1[j];
      }
      if constexpr (NSUM == 3) {
        float e0[V], e1[V];
        Vec<T>::load(dres + r * h + c0, e0);
        Vec<T>::load(dres + (r + 8) * h + c0, e1);
#pragma unroll
        for (int j = 0; j < V; ++j) ar[j] += e0[j] + e1[j];
      }
    }
    for (; r < r1; r += 8) {
      float x0[V], d0[V];
      Vec<T>::load(x + r * h + c0, x0);
      Vec<T>::load(dy + r * h + c0, d0);
      const float mu0 = mean[r], rs0 = rstd[r];
#pragma unroll
      for (int j = 0; j < V; ++j) {
        ag[j] += d0[j] * ((x0[j] - mu0) * rs0);
        ab[j] += d0[j];
      }
      if constexpr (NSUM == 3) {
        float e0[V];
        Vec<T>::load(dres + r * h + c0, e0);
#pragma unroll
        for (int j = 0; j < V; ++j) ar[j] += e0[j];
      }
    }
  }
#pragma unroll
  for (int j = 0; j < V; ++j) {
    red[0][threadIdx.y][threadIdx.x * V + j] = ag[j];
    red[1][threadIdx.y][threadIdx.x * V + j] = ab[j];
    if constexpr (NSUM == 3) red[2][threadIdx.y][threadIdx.x * V + j] = ar[j];
  }
  __syncthreads();
  float* pg = partial + (long long)blockIdx.y * NSUM * h;
  const int t = threadIdx.y * 32 + threadIdx.x;
  for (int cc = t; cc < NSUM * 32 * V; cc += 256) {
    const int which = cc / (32 * V), cl = cc % (32 * V);
    const int col = blockIdx.x * 32 * V + cl;
    if (col < h) {
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) sum += red[which][k][cl];
      pg[which * h + col] = sum;
    }
  }
}

// dgamma[c] = sum_b partial[b][0][c], dbeta[c] = sum_b partial[b][1][c] and, when the partials
// carry a third row, dres_sum[c] = sum_b partial[b][2][c]. Block = 32 columns x 8 slices of the
// partial rows; fixed summation order.
__global__ void __launch_bounds__(256) ln_param_reduce_kernel(int h, int nblk, int nsum,
                                                              const float* __restrict__ partial,
                                                              float* __restrict__ dgamma,
                                                              float* __restrict__ dbeta,
                                                              float* __restrict__ dres_sum) {
  grid_dependency_wait();
  __shared__ float red[8][33];
  const int c = blockIdx.x * 32 + (threadIdx.x & 31);
  const int sl = threadIdx.x >> 5;
  float s = 0.f;
  if (c < nsum * h) {
    // eight loads in flight per thread; the additions keep the order b = sl, sl + 8, ...
    const long long step = (long long)nsum * h;
    int b = sl;
    for (; b + 56 < nblk; b += 64) {
      float p[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) p[u] = __ldg(partial + (b + 8 * u) * step + c);
#pragma unroll
      for (int u = 0; u < 8; ++u) s += p[u];
    }
    for (; b < nblk; b += 8) s += __ldg(partial + b * step + c);
  }
  red[sl][threadIdx.x & 31] = s;
  __syncthreads();
  if (sl == 0 && c < nsum * h) {
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) tot += red[k][threadIdx.x & 31];
    float* out = c < h ? dgamma : (c < 2 * h ? dbeta : dres_sum);
    out[c % h] = tot;
  }
}

// ---------------------------------------------------------------------------- column sums
// out[c] = sum_r x[r, c] in one launch. A cluster of kColsumSlices CTAs along y covers one
// stripe of 32*VEC columns; CTA y of the cluster takes the y-th slice of the rows. Thread (x, t)
// takes rows t, t + 8, ... of the slice, kColsumBatch 16-byte loads in flight at a time (rows
// past the slice read as zeros); the eight row groups of the CTA are added in order into a
// per-column slice sum in shared memory, and after a cluster barrier CTA 0 adds the slices'
// sums, read from the other CTAs' shared memory, in rank order. Every addition has a fixed
// order, so the result does not depend on scheduling.
constexpr int kColsumSlices = 8;
constexpr int kColsumBatch = 8;
__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
template <typename T>
__global__ void __cluster_dims__(1, kColsumSlices, 1) __launch_bounds__(256, 4)
    colsum_kernel(long long rows, int cols, const T* __restrict__ x, float* __restrict__ out,
                  long long rows_per) {
  grid_dependency_wait();
  constexpr int V = Vec<T>::N;
  __shared__ float red[8][32 * V + 1];
  __shared__ float slice_sum[32 * V];
  const int c0 = (blockIdx.x * 32 + threadIdx.x) * V;
  const long long r0 = blockIdx.y * rows_per;
  const long long r1 = min(rows, r0 + rows_per);
  float acc[V];
#pragma unroll
  for (int j = 0; j < V; ++j) acc[j] = 0.f;
  if (c0 < cols) {
    for (long long r = r0 + threadIdx.y; r < r1; r += 8 * kColsumBatch) {
      uint4 w[kColsumBatch];
#pragma unroll
      for (int u = 0; u < kColsumBatch; ++u)
        w[u] = r + 8 * u < r1 ? __ldg(reinterpret_cast<const uint4*>(x + (r + 8 * u) * cols + c0))
                              : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < kColsumBatch; ++u) {
        float v[V];
        Vec<T>::unpack(w[u], v);
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] += v[j];
      }
    }
  }
#pragma unroll
  for (int j = 0; j < V; ++j) red[threadIdx.y][threadIdx.x * V + j] = acc[j];
  __syncthreads();
  const int t = threadIdx.y * 32 + threadIdx.x;
  for (int cc = t; cc < 32 * V; cc += 256) {
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) sum += red[k][cc];
    slice_sum[cc] = sum;
  }
  cluster_sync_all();  // every slice sum of the cluster is written
  if (cluster_ctarank() == 0) {
    for (int cc = t; cc < 32 * V; cc += 256) {
      const int col = blockIdx.x * 32 * V + cc;
      const uint32_t local = smem_u32(&slice_sum[cc]);
      float p[kColsumSlices];
#pragma unroll
      for (int q = 0; q < kColsumSlices; ++q) p[q] = ld_shared_cluster_f32(mapa_shared(local, q));
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < kColsumSlices; ++q) sum += p[q];
      if (col < cols) out[col] = sum;
    }
  }
  cluster_sync_all();  // no CTA leaves while CTA 0 may still read its shared memory
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
  float* out = reinterpret_cast<float*>(a.out);
  const float* bias = reinterpret_cast<const float*>(a.bias);
  // token indices of operands / outputs held in the sequence-parallel layout
  const int ma = a.a_sp ? seq_row(a, m) : m;
  const int mo = a.out_sp ? seq_row(a, m) : m;
  if (a.epi == kEpiSwiglu) {  // gate row ng*2Ng + n and up row + Ng of K-major B
    const long long rg = 2LL * ng * a.Ng + n, ru = rg + a.Ng;
    float g = 0.f, u = 0.f;
    for (int k = 0; k < a.Kg; ++k) {
      const float av = A[(long long)ma * a.lda + k];
      g = fmaf(av, B[rg * a.ldb + k], g);
      u = fmaf(av, B[ru * a.ldb + k], u);
    }
    if (bias) {
      g += bias[rg];
      u += bias[ru];
    }
    float sl, ds;
    silu_and_grad_f(g, sl, ds);
    out[(long long)m * a.ldc + (long long)ng * a.Ng + n] = sl * u;
    float* z = reinterpret_cast<float*>(a.out2) + (long long)m * a.ldc2;
    z[rg] = g;
    z[ru] = u;
    return;
  }
  float acc = 0.f;
  for (int kg = 0; kg < a.KG; ++kg) {
    for (int kk = 0; kk < a.Kg; ++kk) {
      const long long k = (long long)kg * a.Kg + kk;
      const long long kt_a = a.a_sp ? seq_row(a, (int)k) : k;  // token K of an MN-major A
      const long long kt_b = a.b_sp ? seq_row(a, (int)k) : k;  // token K of an MN-major B
      const float av = a.a_mn ? A[kt_a * a.lda + m] : A[(long long)ma * a.lda + k];
      const float bv = a.b_mn ? B[(long long)ng * a.b_ngs + kt_b * a.ldb + n]
                              : B[(long long)kg * a.b_kgs + (long long)n * a.ldb + kk];
      acc = fmaf(av, bv, acc);
    }
  }
  const int col = ng * a.Ng + n;
  const long long off = (long long)(col / a.out_ng) * a.out_gs + (long long)mo * a.ldc +
                        col % a.out_ng;
  switch (a.epi) {
    case kEpiStoreF32: out[off] = acc; break;
    case kEpiBf16: {
      if (bias) acc += bias[col];
      if (a.res) acc += reinterpret_cast<const float*>(a.res)[(long long)mo * a.ldr + col];
      out[off] = acc;
      break;
    }
    case kEpiGelu: {  // out = GeLU(u), out2 = u
      if (bias) acc += bias[col];
      reinterpret_cast<float*>(a.out2)[off] = acc;
      out[off] = gelu_f(acc, a.gelu_tanh);
      break;
    }
    case kEpiDGelu: {  // du = dA GeLU'(u), aux = u
      out[off] = acc * gelu_grad_f(reinterpret_cast<const float*>(a.aux)[(long long)m * a.ld_aux + col],
                                   a.gelu_tanh);
      break;
    }
    case kEpiDSwiglu: {  // acc = dA(m, ng*Ng + n); aux and out laid out [M][NG][2][Ng]
      const long long zo = 2LL * ng * a.Ng + n;
      const float* z = reinterpret_cast<const float*>(a.aux) + (long long)m * a.ld_aux;
      float sl, ds;
      silu_and_grad_f(z[zo], sl, ds);
      float* o = out + (long long)m * a.ldc;
      o[zo] = acc * z[zo + a.Ng] * ds;
      o[zo + a.Ng] = acc * sl;
      break;
    }
  }
}

template <typename T, int W, int VPL>
cudaError_t ln_fwd_inst(long long rows, int h, float eps, const void* x, const float* g,
                        const float* b, void* y, float* mean, float* rstd, cudaStream_t s) {
  const long long grid = (rows + (8 / W) - 1) / (8 / W);
  ln_fwd_kernel<T, W, VPL><<<(unsigned)grid, 256, 0, s>>>(
      rows, h, eps, reinterpret_cast<const T*>(x), g, b, reinterpret_cast<T*>(y), mean, rstd);
  return cudaGetLastError();
}

template <typename T, int W, int VPL>
cudaError_t ln_bwd_dx_inst(long long rows, int h, const void* dy, const void* dres,
                           const void* x, const float* g, const float* mean, const float* rstd,
                           void* dx, cudaStream_t s) {
  const long long grid = (rows + (8 / W) - 1) / (8 / W);
  ln_bwd_dx_kernel<T, W, VPL><<<(unsigned)grid, 256, 0, s>>>(
      rows, h, reinterpret_cast<const T*>(dy), reinterpret_cast<const T*>(dres),
      reinterpret_cast<const T*>(x), g, mean, rstd, reinterpret_cast<T*>(dx));
  return cudaGetLastError();
}

bool aligned16_ptr(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 1;
  return n;
}

// Blocks of a ring kernel resident per SM at `smem` bytes of dynamic shared memory (0 on
// failure); raises the kernel's dynamic shared-memory limit first. Cached per (kernel, smem).
template <typename K>
int ring_blocks_per_sm(K kern, size_t smem) {
  struct Entry {
    const void* fn;
    size_t smem;
    int bps;
  };
  static std::mutex mu;
  static Entry cache[32];
  static int used = 0;
  const void* fn = reinterpret_cast<const void*>(kern);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].fn == fn && cache[i].smem == smem) return cache[i].bps;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 256, smem) != cudaSuccess) return 0;
  if (used < 32) cache[used++] = Entry{fn, smem, n};
  return n;
}

template <typename T, int VPL>
cudaError_t ln_fwd_ring_inst(long long rows, int h, float eps, const void* x, const float* g,
                             const float* b, void* y, float* mean, float* rstd, int* err,
                             cudaStream_t s) {
  auto kern = ln_fwd_ring_kernel<T, VPL, kRingStages>;
  const size_t smem = (size_t)kRingStages * h * sizeof(T);
  const int bps = ring_blocks_per_sm(kern, smem);
  if (bps < 1) return cudaErrorInvalidConfiguration;
  long long grid = (long long)bps * device_sms();
  if (grid > rows) grid = rows;
  return launch_kernel(true, kern, dim3((unsigned)grid), dim3(256), smem, s, rows, h, eps,
                       reinterpret_cast<const T*>(x), g, b, reinterpret_cast<T*>(y), mean, rstd,
                       err);
}

// Row-group shapes: a row is spread over W warps with at most VPL 16-byte vectors per thread,
// so registers stay small and many rows are in flight. bf16: h <= 16384; fp32: h <= 8192.
// Rows of 256..1024 vectors (bf16 h = 2048..8192) go through the shared-memory ring instead.
template <typename T>
cudaError_t ln_fwd_dispatch(long long rows, int h, float eps, const void* x, const float* g,
                            const float* b, void* y, float* mean, float* rstd, int* err,
                            cudaStream_t s) {
  const int nvec = h / Vec<T>::N;
  if (nvec >= 256 && nvec <= 1024 && aligned16_ptr(x)) {
    if (nvec <= 256) return ln_fwd_ring_inst<T, 1>(rows, h, eps, x, g, b, y, mean, rstd, err, s);
    if (nvec <= 512) return ln_fwd_ring_inst<T, 2>(rows, h, eps, x, g, b, y, mean, rstd, err, s);
    return ln_fwd_ring_inst<T, 4>(rows, h, eps, x, g, b, y, mean, rstd, err, s);
  }
  if (nvec <= 64) return ln_fwd_inst<T, 1, 2>(rows, h, eps, x, g, b, y, mean, rstd, s);
  if (nvec <= 128) return ln_fwd_inst<T, 1, 4>(rows, h, eps, x, g, b, y, mean, rstd, s);
  if (nvec <= 256) return ln_fwd_inst<T, 2, 4>(rows, h, eps, x, g, b, y, mean, rstd, s);
  if (nvec <= 512) return ln_fwd_inst<T, 4, 4>(rows, h, eps, x, g, b, y, mean, rstd, s);
  if (nvec <= 1024) return ln_fwd_inst<T, 8, 4>(rows, h, eps, x, g, b, y, mean, rstd, s);
  return ln_fwd_inst<T, 8, 8>(rows, h, eps, x, g, b, y, mean, rstd, s);
}

// dgamma, dbeta (and dres_sum) from the per-block partial rows, in a fixed order.
cudaError_t launch_param_reduce(int h, long long slices, int nsum, const float* partial,
                                float* dgamma, float* dbeta, float* dres_sum, cudaStream_t s) {
  return launch_kernel(true, ln_param_reduce_kernel, dim3((nsum * h + 31) / 32), dim3(256), 0,
                       s, h, (int)slices, nsum, partial, dgamma, dbeta, dres_sum);
}

template <typename T>
cudaError_t ln_bwd_dispatch(long long rows, int h, const void* dy, const void* dres,
                            const void* x, const float* g, const float* mean, const float* rstd,
                            void* dx, float* partial, int nblk, float* dgamma, float* dbeta,
                            float* dres_sum, int* err, cudaStream_t s) {
  const int nvec = h / Vec<T>::N;
  const int nsum = (dres_sum && dres) ? 3 : 2;
  cudaError_t e;
  if (nvec <= 512) {  // one pass: dx and the parameter partials together
    long long slices = nblk < rows ? nblk : rows;
    const long long rows_per = (rows + slices - 1) / slices;
    slices = (rows + rows_per - 1) / rows_per;
    const T* pdy = reinterpret_cast<const T*>(dy);
    const T* pdr = reinterpret_cast<const T*>(dres);
    const T* px = reinterpret_cast<const T*>(x);
    T* pdx = reinterpret_cast<T*>(dx);
    const unsigned gs = (unsigned)slices;
    // The ring kernel's waits are bounded and report a run-out through `err`; a caller with
    // no status word gets the wait-free kernels, so a timeout can never go unreported.
    const bool ring = err && nvec >= 256 && aligned16_ptr(x) && aligned16_ptr(dy) &&
                      (!dres || aligned16_ptr(dres));
    if (ring) {
      // x, dy (and dres) rows streamed through the shared-memory ring
      const size_t smem = (size_t)kRingStages * (dres ? 3 : 2) * h * sizeof(T);
      auto launch = [&](auto kern) {
        if (ring_blocks_per_sm(kern, smem) < 1) return cudaErrorInvalidConfiguration;
        return launch_kernel(true, kern, dim3(gs), dim3(256), smem, s, rows, h, pdy, pdr, px,
                             g, mean, rstd, pdx, partial, rows_per, err);
      };
      if (nvec <= 256)
        e = nsum == 3 ? launch(ln_bwd_ring_kernel<T, 1, 3, kRingStages>)
                      : launch(ln_bwd_ring_kernel<T, 1, 2, kRingStages>);
      else
        e = nsum == 3 ? launch(ln_bwd_ring_kernel<T, 2, 3, kRingStages>)
                      : launch(ln_bwd_ring_kernel<T, 2, 2, kRingStages>);
      if (e != cudaSuccess) return e;
    } else if (nvec <= 256) {
      if (nsum == 3)
        ln_bwd_fused_kernel<T, 1, 3><<<gs, 256, 0, s>>>(rows, h, pdy, pdr, px, g, mean, rstd,
                                                        pdx, partial, rows_per);
      else
        ln_bwd_fused_kernel<T, 1, 2><<<gs, 256, 0, s>>>(rows, h, pdy, pdr, px, g, mean, rstd,
                                                        pdx, partial, rows_per);
    } else {
      if (nsum == 3)
        ln_bwd_fused_kernel<T, 2, 3><<<gs, 256, 0, s>>>(rows, h, pdy, pdr, px, g, mean, rstd,
                                                        pdx, partial, rows_per);
      else
        ln_bwd_fused_kernel<T, 2, 2><<<gs, 256, 0, s>>>(rows, h, pdy, pdr, px, g, mean, rstd,
                                                        pdx, partial, rows_per);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_param_reduce(h, slices, nsum, partial, dgamma, dbeta, dres_sum, s);
  }
  // Wider rows: a dx kernel, then a parameter-partial kernel over slices of rows.
  if (nvec <= 64)
    e = ln_bwd_dx_inst<T, 1, 2>(rows, h, dy, dres, x, g, mean, rstd, dx, s);
  else if (nvec <= 128)
    e = ln_bwd_dx_inst<T, 1, 4>(rows, h, dy, dres, x, g, mean, rstd, dx, s);
  else if (nvec <= 256)
    e = ln_bwd_dx_inst<T, 2, 4>(rows, h, dy, dres, x, g, mean, rstd, dx, s);
  else if (nvec <= 512)
    e = ln_bwd_dx_inst<T, 4, 4>(rows, h, dy, dres, x, g, mean, rstd, dx, s);
  else if (nvec <= 1024)
    e = ln_bwd_dx_inst<T, 8, 4>(rows, h, dy, dres, x, g, mean, rstd, dx, s);
  else
    e = ln_bwd_dx_inst<T, 8, 8>(rows, h, dy, dres, x, g, mean, rstd, dx, s);
  if (e != cudaSuccess) return e;
  // dgamma/dbeta partials: one partial row pair per slice of rows, at most nblk slices.
  const int cb = (h + 32 * Vec<T>::N - 1) / (32 * Vec<T>::N);
  long long slices = (4LL * 148 + cb - 1) / cb;
  if (slices > nblk) slices = nblk;
  if (slices > (rows + 15) / 16) slices = (rows + 15) / 16;
  if (slices < 1) slices = 1;
  const long long rows_per = (rows + slices - 1) / slices;
  slices = (rows + rows_per - 1) / rows_per;
  if (nsum == 3)
    ln_bwd_param_kernel<T, 3><<<dim3(cb, (unsigned)slices), dim3(32, 8), 0, s>>>(
        rows, h, reinterpret_cast<const T*>(dy), reinterpret_cast<const T*>(x),
        reinterpret_cast<const T*>(dres), mean, rstd, partial, rows_per);
  else
    ln_bwd_param_kernel<T, 2><<<dim3(cb, (unsigned)slices), dim3(32, 8), 0, s>>>(
        rows, h, reinterpret_cast<const T*>(dy), reinterpret_cast<const T*>(x), nullptr, mean,
        rstd, partial, rows_per);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_param_reduce(h, slices, nsum, partial, dgamma, dbeta, dres_sum, s);
}

}  // namespace

cudaError_t launch_ln_fwd(int dtype, long long rows, int h, float eps, const void* x,
                          const float* gamma, const float* beta, void* y, float* mean,
                          float* rstd, int* err, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  return dtype ? ln_fwd_dispatch<__nv_bfloat16>(rows, h, eps, x, gamma, beta, y, mean, rstd,
                                                err, s)
               : ln_fwd_dispatch<float>(rows, h, eps, x, gamma, beta, y, mean, rstd, err, s);
}

int ln_bwd_blocks(long long rows, int num_sms) {
  long long n = 2LL * num_sms;
  if (n > rows) n = rows;
  return n < 1 ? 1 : (int)n;
}

cudaError_t launch_ln_bwd(int dtype, long long rows, int h, const void* dy, const void* dres,
                          const void* x, const float* gamma, const float* mean,
                          const float* rstd, void* dx, float* partial, int nblk, float* dgamma,
                          float* dbeta, float* dres_sum, int* err, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  return dtype ? ln_bwd_dispatch<__nv_bfloat16>(rows, h, dy, dres, x, gamma, mean, rstd, dx,
                                                partial, nblk, dgamma, dbeta, dres_sum, err, s)
               : ln_bwd_dispatch<float>(rows, h, dy, dres, x, gamma, mean, rstd, dx, partial,
                                        nblk, dgamma, dbeta, dres_sum, err, s);
}

cudaError_t launch_colsum(int dtype, long long rows, int cols, const void* x, float* out,
                          bool programmatic,
                          cudaStream_t s) {
  if (rows <= 0) return cudaMemsetAsync(out, 0, sizeof(float) * cols, s);
  const int V = dtype ? 8 : 4;
  const int cb = (cols + 32 * V - 1) / (32 * V);
  const long long rows_per = (rows + kColsumSlices - 1) / kColsumSlices;
  dim3 grid(cb, kColsumSlices), block(32, 8);
  if (dtype)
    return launch_kernel(programmatic, colsum_kernel<__nv_bfloat16>, grid, block, 0, s, rows,
                         cols, reinterpret_cast<const __nv_bfloat16*>(x), out, rows_per);
  return launch_kernel(programmatic, colsum_kernel<float>, grid, block, 0, s, rows, cols,
                       reinterpret_cast<const float*>(x), out, rows_per);
}

// One thread waits on an mbarrier that nothing ever arrives on, through the same bounded
// wait every pipelined kernel uses: it gives up after limit_ns, records kErrTimeoutProbe in
// the status word and returns, leaving the context usable.
__global__ void bounded_wait_probe_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, status, kErrTimeoutProbe, nullptr, limit_ns);
}

__global__ void exp2_probe_kernel(int path, long long n, const float* x, float* y) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
  if (path == 1) {
    exp2_poly_pair(a, b);
  } else {
    a = ex2_approx(a);
    b = ex2_approx(b);
  }
  y[i] = a;
  if (i + 1 < n) y[i + 1] = b;
}

cudaError_t launch_exp2_probe(int path, long long n, const float* x, float* y, cudaStream_t s) {
  const long long pairs = (n + 1) / 2;
  exp2_probe_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, s>>>(path, n, x, y);
  return cudaGetLastError();
}

cudaError_t launch_bounded_wait_probe(int* status, unsigned long long limit_ns, cudaStream_t s) {
  bounded_wait_probe_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_gemm_simt_f32(const GemmArgs& a, cudaStream_t s) {
  const long long total = (long long)a.NG * a.M * a.Ng;
  if (total <= 0) return cudaSuccess;
  gemm_simt_f32_kernel<<<(unsigned)((total + 127) / 128), 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mgt
