// FP8 (e4m3) with a per-tensor scale: the precision that the page "把大模型训练“摁”到规模化：
// NVIDIA Megatron-LM / Megatron Core 上手与理解" (section 0) lists among Megatron Core's mixed
// precisions, and the trdm.cn page's inference section enables with --enable-fp8. The pages give
// no scaling recipe; the one used here is current per-tensor scaling: amax = max |x| over the
// tensor, q = e4m3(x * 448 / amax) (448 = largest finite e4m3), dequantisation factor
// amax / 448, products accumulated in fp32 by the tensor cores (gemm_tc.cu, F8 path).
#include "mgt_device.cuh"

namespace mgt {
namespace {

template <typename T>
__device__ __forceinline__ float load_f(const T* p, long long i);
template <>
__device__ __forceinline__ float load_f<float>(const float* p, long long i) {
  return p[i];
}
template <>
__device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p, long long i) {
  return __bfloat162float(p[i]);
}

// amax over n elements: grid-stride maxima of |x|, a block reduction, then one atomic max on
// the float's bit pattern (non-negative floats order like their bits) into a zeroed word.
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(long long n, const T* __restrict__ x,
                                                   unsigned int* __restrict__ amax_bits) {
  __shared__ float red[8];
  float m = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(load_f(x, i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) b = fmaxf(b, red[w]);
    atomicMax(amax_bits, __float_as_uint(b));
  }
}

// Two fp32 values to two e4m3 bytes (round to nearest even, saturating to +-448): the
// hardware conversion; lo lands in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// q[i] = e4m3(x[i] * s) with s = 448 / amax (1 if amax is 0), two elements per thread step;
// scales[1] = amax / 448 (1 if amax is 0), the dequantisation factor.
template <typename T>
__global__ void __launch_bounds__(256) cast_kernel(long long n, const T* __restrict__ x,
                                                   float* __restrict__ scales,
                                                   uint8_t* __restrict__ q) {
  const float amax = scales[0];
  const float s = amax > 0.f ? 448.f / amax : 1.f;
  const long long pairs = (n + 1) / 2;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < pairs;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = 2 * i;
    const float lo = load_f(x, e) * s;
    const float hi = e + 1 < n ? load_f(x, e + 1) * s : 0.f;
    const uint16_t w = e4m3x2(lo, hi);
    if (e + 1 < n) {
      *reinterpret_cast<uint16_t*>(q + e) = w;
    } else {
      q[e] = static_cast<uint8_t>(w & 0xffu);
    }
  }
}

__global__ void dequant_factor_kernel(float* scales) {
  const float amax = scales[0];
  scales[1] = amax > 0.f ? amax / 448.f : 1.f;
}

}  // namespace

cudaError_t launch_fp8_quantize(int dtype, long long n, const void* x, uint8_t* q,
                                float* scales, cudaStream_t s) {
  if (n <= 0) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(scales, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  const long long want = (n + 255) / 256;
  const unsigned blocks = (unsigned)(want < 4 * 148 ? want : 4 * 148);
  auto* bits = reinterpret_cast<unsigned int*>(scales);
  if (dtype)
    amax_kernel<<<blocks, 256, 0, s>>>(n, reinterpret_cast<const __nv_bfloat16*>(x), bits);
  else
    amax_kernel<<<blocks, 256, 0, s>>>(n, reinterpret_cast<const float*>(x), bits);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long pairs = (n + 1) / 2;
  const long long want2 = (pairs + 255) / 256;
  const unsigned blocks2 = (unsigned)(want2 < 8 * 148 ? want2 : 8 * 148);
  if (dtype)
    cast_kernel<<<blocks2, 256, 0, s>>>(n, reinterpret_cast<const __nv_bfloat16*>(x), scales, q);
  else
    cast_kernel<<<blocks2, 256, 0, s>>>(n, reinterpret_cast<const float*>(x), scales, q);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dequant_factor_kernel<<<1, 1, 0, s>>>(scales);
  return cudaGetLastError();
}

}  // namespace mgt
