// Tensor-core GEMM for sm_100a: TMA -> shared-memory ring -> tcgen05.mma (one issuing thread)
// -> fp32 accumulators in tensor memory -> epilogue warps (tcgen05.ld) -> global memory.
//
// This one kernel serves every contraction of the layer:
//   forward  QKV / fc1 (column-parallel): A = activations (K-major), B = packed weight rows
//            (K-major); out-proj / fc2 (row-parallel): the K loop runs over the tp shards
//            (K groups), so the shard partials are summed in the tensor-memory accumulator
//            -- the on-device equivalent of the AllReduce after RowParallelLinear described
//            on the trdm.cn page, section 2.1.
//   backward dgrad: B = weight read N-major (no transpose copy); for row-parallel layers the
//            N dimension is grouped by shard. wgrad: A = dY^T and B = X, both read MN-major
//            along the token dimension; fp32 output written straight into the packed layout.
//
// CTA: 320 threads. warp 0 = TMA producer (one lane), warp 1 = TMEM owner + MMA issuer (one
// lane), warps 2..9 = epilogue: warp w reads TMEM lanes 32*(w%4)..+31, and the two warps of
// each lane quarter split the tile's columns, so the epilogue keeps pace with the MMAs. Persistent: grid =
// min(#tiles, #SMs); tiles are taken round-robin. Accumulators are double-buffered in TMEM so
// the epilogue of tile i overlaps the main loop of tile i+1.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "mgt_device.cuh"

namespace mgt {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes = one 128B-swizzle row
constexpr int kThreads = 320;  // 2 producer/MMA warps + 8 epilogue warps
constexpr int kEpiWarps = 8;
constexpr int kChunkBytes = 64 * BK * 2;  // one [64 x 64] bf16 box = 8 KB

template <int BN>
struct Cfg {
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
};

struct TileCoord {
  int ng, mb, nb;
};

// Tile order within a group. The CTAs of one wave run consecutive tiles, and the operand that
// the fast index sweeps is read again by every wave, so the fast index is the one whose
// operand is smaller (it then stays in L2): M fastest (the wave shares B tiles and sweeps A)
// unless A is the larger operand (M > N, the wide weight gradients), then N fastest.
__device__ __forceinline__ TileCoord tile_coord(int tile, int num_m, int num_n, int n_fast) {
  TileCoord t;
  const int per_group = num_m * num_n;
  t.ng = tile / per_group;
  const int r = tile - t.ng * per_group;
  if (n_fast) {
    t.mb = r / num_n;
    t.nb = r - t.mb * num_n;
  } else {
    t.nb = r / num_m;
    t.mb = r - t.nb * num_m;
  }
  return t;
}

// ---------------------------------------------------------------------------- epilogue
// Every loop over the 32 accumulator values is unrolled with compile-time indices (ragged chunks
// are predicated, not shortened), so v stays in registers instead of local memory.
template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& a, int row, int col,
                                               int count, float (&v)[32]) {
  const long long off = (long long)(col / a.out_ng) * a.out_gs + (long long)row * a.ldc +
                        (col % a.out_ng);
  if constexpr (EPI == kEpiStoreF32) {
    float* o = reinterpret_cast<float*>(a.out) + off;
    if (count == 32) {
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(o + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < count) o[i] = v[i];
    }
    return;
  } else if constexpr (EPI == kEpiDSwiglu) {
    // The chunk lies inside one group ng (tiles never cross groups).
    const int ng = col / a.Ng, n = col - ng * a.Ng;
    const long long zo = (long long)row * a.ld_aux + 2LL * ng * a.Ng + n;
    const long long oo = (long long)row * a.ldc + 2LL * ng * a.Ng + n;
    const __nv_bfloat16* zg = reinterpret_cast<const __nv_bfloat16*>(a.aux) + zo;
    __nv_bfloat16* og = reinterpret_cast<__nv_bfloat16*>(a.out) + oo;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i < count) {
        float sl, ds;
        silu_and_grad_bf16out(__bfloat162float(zg[i]), sl, ds);
        og[i] = __float2bfloat16_rn(v[i] * __bfloat162float(zg[a.Ng + i]) * ds);
        og[a.Ng + i] = __float2bfloat16_rn(v[i] * sl);
      }
    }
    return;
  } else {
    // bias / residual / aux come in the activation dtype (bf16)
    const __nv_bfloat16* bias = reinterpret_cast<const __nv_bfloat16*>(a.bias);
    if (EPI == kEpiBf16 || EPI == kEpiGelu) {
      if (bias) {
        if (count == 32) {
          const uint4* bp = reinterpret_cast<const uint4*>(bias + col);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 w = __ldg(bp + q);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              v[q * 8 + 2 * j] += bf16_lo(ww[j]);
              v[q * 8 + 2 * j + 1] += bf16_hi(ww[j]);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < count) v[i] += __bfloat162float(bias[col + i]);
        }
      }
    }
    if (EPI == kEpiBf16 && a.res) {
      const __nv_bfloat16* r =
          reinterpret_cast<const __nv_bfloat16*>(a.res) + (long long)row * a.ldr + col;
      if (count == 32) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 w = *reinterpret_cast<const uint4*>(r + q * 8);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            v[q * 8 + 2 * j] += bf16_lo(ww[j]);
            v[q * 8 + 2 * j + 1] += bf16_hi(ww[j]);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i < count) v[i] += __bfloat162float(r[i]);
      }
    }
    if (EPI == kEpiDGelu) {  // aux holds u, stored by the forward epilogue: du = dA GeLU'(u)
      const __nv_bfloat16* g =
          reinterpret_cast<const __nv_bfloat16*>(a.aux) + (long long)row * a.ld_aux + col;
      if (count == 32) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 w = *reinterpret_cast<const uint4*>(g + q * 8);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            v[q * 8 + 2 * j] *= gelu_grad_bf16out(bf16_lo(ww[j]), a.gelu_tanh);
            v[q * 8 + 2 * j + 1] *= gelu_grad_bf16out(bf16_hi(ww[j]), a.gelu_tanh);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i < count) v[i] *= gelu_grad_bf16out(__bfloat162float(g[i]), a.gelu_tanh);
      }
    }
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + off;
    if (EPI == kEpiGelu) {  // out = GeLU(u), out2 = u for the backward
      __nv_bfloat16* o2 = reinterpret_cast<__nv_bfloat16*>(a.out2) + off;
      if (count == 32) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float ga[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) ga[j] = gelu_bf16out(v[q * 8 + j], a.gelu_tanh);
          uint4 wd, wa;
          wd.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
          wd.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
          wd.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
          wd.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
          *reinterpret_cast<uint4*>(o2 + q * 8) = wd;
          wa.x = pack_bf16x2(ga[0], ga[1]);
          wa.y = pack_bf16x2(ga[2], ga[3]);
          wa.z = pack_bf16x2(ga[4], ga[5]);
          wa.w = pack_bf16x2(ga[6], ga[7]);
          *reinterpret_cast<uint4*>(o + q * 8) = wa;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i < count) {
            o2[i] = __float2bfloat16_rn(v[i]);
            o[i] = __float2bfloat16_rn(gelu_bf16out(v[i], a.gelu_tanh));
          }
        }
      }
      return;
    }
    if (count == 32) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
        w.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
        w.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
        w.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
        *reinterpret_cast<uint4*>(o + q * 8) = w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < count) o[i] = __float2bfloat16_rn(v[i]);
    }
  }
}

// The per-element source of a bf16 epilogue chunk (32 columns from col of row `row`): the
// residual (kEpiBf16 with a residual) or u (kEpiDGelu); zeros for a row past M. Loaded ahead
// of the accumulator so that its latency overlaps the TMEM read (and the previous chunk).
template <int EPI>
__device__ __forceinline__ bool epi_has_src(const GemmArgs& a) {
  return (EPI == kEpiBf16 && a.res) || EPI == kEpiDGelu;
}
template <int EPI>
__device__ __forceinline__ void epi_load_src(const GemmArgs& a, int row, int col, bool row_ok,
                                             uint4 (&r4)[4]) {
  const __nv_bfloat16* src =
      EPI == kEpiDGelu
          ? reinterpret_cast<const __nv_bfloat16*>(a.aux) + (long long)row * a.ld_aux + col
          : reinterpret_cast<const __nv_bfloat16*>(a.res) + (long long)row * a.ldr + col;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    r4[q] = row_ok ? *reinterpret_cast<const uint4*>(src + q * 8) : make_uint4(0, 0, 0, 0);
}

// Values of one whole 32-column chunk of a bf16 epilogue, packed as bf16 pairs for a staged
// (TMA) store: w holds out, w2 out2 (kEpiGelu only); r4 is the chunk's source as loaded by
// epi_load_src (read when epi_has_src). Rows at or past M (row_ok false) read no residual or
// aux; the store clips them.
template <int EPI>
__device__ __forceinline__ void epi_values_bf16(const GemmArgs& a, int row, int col, bool row_ok,
                                                float (&v)[32], const uint4 (&r4)[4],
                                                uint32_t (&w)[16], uint32_t (&w2)[16]) {
  const __nv_bfloat16* bias = reinterpret_cast<const __nv_bfloat16*>(a.bias);
  if ((EPI == kEpiBf16 || EPI == kEpiGelu) && bias) {
    const uint4* bp = reinterpret_cast<const uint4*>(bias + col);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u4 = __ldg(bp + q);
      const uint32_t ww[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[q * 8 + 2 * j] += bf16_lo(ww[j]);
        v[q * 8 + 2 * j + 1] += bf16_hi(ww[j]);
      }
    }
  }
  if (epi_has_src<EPI>(a)) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t ww[4] = {r4[q].x, r4[q].y, r4[q].z, r4[q].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (EPI == kEpiDGelu) {  // aux holds u, stored by the forward epilogue
          v[q * 8 + 2 * j] *= gelu_grad_bf16out(bf16_lo(ww[j]), a.gelu_tanh);
          v[q * 8 + 2 * j + 1] *= gelu_grad_bf16out(bf16_hi(ww[j]), a.gelu_tanh);
        } else {
          v[q * 8 + 2 * j] += bf16_lo(ww[j]);
          v[q * 8 + 2 * j + 1] += bf16_hi(ww[j]);
        }
      }
    }
  }
  if constexpr (EPI == kEpiDSwiglu) {  // w: d gate, w2: d up (aux = [g | u] of this group)
    const int ng = col / a.Ng, n = col - ng * a.Ng;
    const __nv_bfloat16* zg = reinterpret_cast<const __nv_bfloat16*>(a.aux) +
                              (long long)row * a.ld_aux + 2LL * ng * a.Ng + n;
    uint4 g4[4], u4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      g4[q] = row_ok ? *reinterpret_cast<const uint4*>(zg + q * 8) : make_uint4(0, 0, 0, 0);
      u4[q] = row_ok ? *reinterpret_cast<const uint4*>(zg + a.Ng + q * 8)
                     : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t gg[4] = {g4[q].x, g4[q].y, g4[q].z, g4[q].w};
      const uint32_t uu[4] = {u4[q].x, u4[q].y, u4[q].z, u4[q].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float s0, s1, d0, d1;
        silu_and_grad_bf16out(bf16_lo(gg[j]), s0, d0);
        silu_and_grad_bf16out(bf16_hi(gg[j]), s1, d1);
        const float a0 = v[q * 8 + 2 * j], a1 = v[q * 8 + 2 * j + 1];
        w[q * 4 + j] = pack_bf16x2(a0 * bf16_lo(uu[j]) * d0, a1 * bf16_hi(uu[j]) * d1);
        w2[q * 4 + j] = pack_bf16x2(a0 * s0, a1 * s1);
      }
    }
    return;
  }
  if constexpr (EPI == kEpiGelu) {  // w: GeLU(u), w2: u
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      w[i] = pack_bf16x2(gelu_bf16out(v[2 * i], a.gelu_tanh),
                         gelu_bf16out(v[2 * i + 1], a.gelu_tanh));
      w2[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  }
}

// SwiGLU forward, element by element (ragged chunks): gate and up accumulators of output
// columns ng*Ng + n0 .. + count-1.
__device__ __forceinline__ void swiglu_chunk_elem(const GemmArgs& a, int row, int ng, int n0,
                                                  int count, const float (&vg)[32],
                                                  const float (&vu)[32]) {
  const __nv_bfloat16* bias = reinterpret_cast<const __nv_bfloat16*>(a.bias);
  const long long brow = 2LL * ng * a.Ng + n0;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + (long long)row * a.ldc +
                     (long long)ng * a.Ng + n0;
  __nv_bfloat16* z = reinterpret_cast<__nv_bfloat16*>(a.out2) + (long long)row * a.ldc2 + brow;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (i < count) {
      float g = vg[i], u = vu[i];
      if (bias) {
        g += __bfloat162float(bias[brow + i]);
        u += __bfloat162float(bias[brow + a.Ng + i]);
      }
      float sl, ds;
      silu_and_grad_bf16out(g, sl, ds);
      o[i] = __float2bfloat16_rn(sl * u);
      z[i] = __float2bfloat16_rn(g);
      z[a.Ng + i] = __float2bfloat16_rn(u);
    }
  }
}

// SwiGLU forward for a whole chunk, packed for staged stores: w = silu(g)*u, w2 = g, w3 = u.
__device__ __forceinline__ void swiglu_values(const GemmArgs& a, int ng, int n0, float (&vg)[32],
                                              float (&vu)[32], uint32_t (&w)[16],
                                              uint32_t (&w2)[16], uint32_t (&w3)[16]) {
  const __nv_bfloat16* bias = reinterpret_cast<const __nv_bfloat16*>(a.bias);
  if (bias) {
    const long long brow = 2LL * ng * a.Ng + n0;
    const uint4* bg = reinterpret_cast<const uint4*>(bias + brow);
    const uint4* bu = reinterpret_cast<const uint4*>(bias + brow + a.Ng);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 g4 = __ldg(bg + q), u4 = __ldg(bu + q);
      const uint32_t gg[4] = {g4.x, g4.y, g4.z, g4.w}, uu[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        vg[q * 8 + 2 * j] += bf16_lo(gg[j]);
        vg[q * 8 + 2 * j + 1] += bf16_hi(gg[j]);
        vu[q * 8 + 2 * j] += bf16_lo(uu[j]);
        vu[q * 8 + 2 * j + 1] += bf16_hi(uu[j]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float s0, s1, d0, d1;
    silu_and_grad_bf16out(vg[2 * i], s0, d0);
    silu_and_grad_bf16out(vg[2 * i + 1], s1, d1);
    w[i] = pack_bf16x2(s0 * vu[2 * i], s1 * vu[2 * i + 1]);
    w2[i] = pack_bf16x2(vg[2 * i], vg[2 * i + 1]);
    w3[i] = pack_bf16x2(vu[2 * i], vu[2 * i + 1]);
  }
}

// ---------------------------------------------------------------------------- kernel
template <int BN, bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB, const GemmArgs args, int num_m,
                   int num_n) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  // 128B-swizzled tiles need 1024-byte alignment in the shared window itself.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kt_per_group = (args.Kg + BK - 1) / BK;
  const int k_iters = args.KG * kt_per_group;
  const int num_tiles = args.NG * num_m * num_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (k_iters > 0 && warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    SeqCursor cur{0, 0};
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const TileCoord tc = tile_coord(tile, num_m, num_n, args.n_fast);
      // token coordinates go through the sequence-parallel row map where set: M of a
      // K-major A once per tile, the K of an MN-major operand through the cursor
      const int ma = (!A_MN && args.a_sp) ? seq_row(args, tc.mb * BM) : tc.mb * BM;
      for (int kg = 0; kg < args.KG && ok; ++kg) {
        for (int kt = 0; kt < kt_per_group; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, args.err, kErrTimeoutProducer, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          uint8_t* a_dst = sA + stage * C::A_BYTES;
          uint8_t* b_dst = sB + stage * C::B_BYTES;
          const int kk = ((A_MN && args.a_sp) || (B_MN && args.b_sp)) ? cur.row(args, kt * BK)
                                                                       : kt * BK;
          const int ka = args.a_sp ? kk : kt * BK;
          const int kb = args.b_sp ? kk : kt * BK;
          if constexpr (!A_MN) {
            tma_load_3d(&tmA, &full[stage], a_dst, kt * BK, kg, ma);
          } else {
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              tma_load_3d(&tmA, &full[stage], a_dst + c * kChunkBytes, tc.mb * BM + c * 64,
                          ka, 0);
          }
          if constexpr (!B_MN) {
            tma_load_3d(&tmB, &full[stage], b_dst, kt * BK, tc.nb * BN, kg);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_3d(&tmB, &full[stage], b_dst + c * kChunkBytes, tc.nb * BN + c * 64,
                          kb, tc.ng);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
    {
      // Let every load this thread issued land before the CTA can exit (after a timeout too).
      // The slots issued most recently are the STAGES before the cursor; wait (bounded) for
      // their phase. Slots never issued report their previous phase as complete.
      for (int i = 1; i <= C::STAGES; ++i) {
        int s = stage - i;
        uint32_t ph = phase;
        if (s < 0) {
          s += C::STAGES;
          ph ^= 1;
        }
        mbar_wait(&full[s], ph, args.err, kErrTimeoutDrain, nullptr);
      }
    }
  } else if (k_iters > 0 && warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1, args.err, kErrTimeoutMma, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int it = 0; it < k_iters; ++it) {
        if (!mbar_wait(&full[stage], phase, args.err, kErrTimeoutMma, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
        const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          // K-major: advance 16 elements (32 bytes) inside the 128-byte swizzle row.
          // MN-major: advance 16 rows of 128 bytes; 64-wide MN chunks are kChunkBytes apart.
          const uint64_t ad = A_MN ? smem_desc_sw128(a_addr + k * 2048, kChunkBytes, 1024)
                                   : smem_desc_sw128(a_addr + k * 32, 16, 1024);
          const uint64_t bd = B_MN ? smem_desc_sw128(b_addr + k * 2048, kChunkBytes, 1024)
                                   : smem_desc_sw128(b_addr + k * 32, 16, 1024);
          tc_mma_f16(d_tmem, ad, bd, idesc, (it > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&empty[stage]);  // frees the slot once these MMAs have read it
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      tc_commit(&tfull[acc]);  // accumulator ready once all MMAs above complete
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    // Make sure no MMA is still writing tensor memory when the CTA frees it.
    tc_commit(drain);
    mbar_wait(drain, 0, args.err, kErrTimeoutDrain, nullptr);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp & 3;  // TMEM lane quarter this warp may access
    const int c_begin = ((warp - 2) >> 2) * (BN / 64);  // this warp's half of the columns
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const TileCoord tc = tile_coord(tile, num_m, num_n, args.n_fast);
      const int row = tc.mb * BM + ew * 32 + lane;
      if (k_iters > 0) {
        const bool ok = mbar_wait(&tfull[acc], acc_phase, args.err, kErrTimeoutEpilogue,
                                  abort_flag);
        // Lanes leave the polling loop independently; tcgen05.ld is .sync.aligned and needs
        // the whole warp converged, and the exit decision must be warp-uniform.
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
      }
#pragma unroll 1
      for (int c = c_begin; c < c_begin + BN / 64; ++c) {
        float v[32];
        if (k_iters > 0) {
          tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + acc * BN + c * 32,
                             v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        const int n0 = tc.nb * BN + c * 32;
        if (row < args.M && n0 < args.Ng) {
          const int count = min(32, args.Ng - n0);
          epilogue_chunk<EPI>(args, args.out_sp ? seq_row(args, row) : row,
                              tc.ng * args.Ng + n0, count, v);
        }
      }
      if (k_iters > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------- CTA-pair kernel
// Same contract as gemm_tc_kernel, but a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256): CTA r of the pair loads rows
// [m0 + 128 r, +128) of A and the half [n0 + 128 r, +128) of B into its own shared memory, and
// the pair's leader issues one MMA that reads both CTAs' halves and writes each CTA's 128
// accumulator rows into that CTA's tensor memory. Each CTA moves 32 KB per 64-deep k-step
// instead of 48 KB for the same MMA work per SM, which is what keeps the shared-memory port
// below its limit at full tensor throughput.
//
// Synchronisation: both CTAs' TMA loads complete on the leader's `full` barrier (the leader
// posts the expected bytes of both); the leader's tcgen05.commit multicasts to `empty` and
// `tfull` in both CTAs; both CTAs' epilogue warps arrive on the leader's `tempty` (count 8).
// A cluster barrier after initialisation and another before exit bracket all cross-CTA
// traffic; every wait in between is bounded.
// Six 32 KB stages; the SwiGLU forward keeps five to make room for its three staged outputs,
// and the fp32 store, which stages nothing, takes seven.
constexpr int pair_stages(int epi) {
  return epi == kEpiSwiglu ? 5 : (epi == kEpiStoreF32 ? 7 : 6);
}
constexpr int stage_out_bytes(int epi) {
  return epi == kEpiSwiglu ? 6144 : (epi == kEpiStoreF32 ? 0 : 4096);
}
constexpr int kPairAB = BM * BK * 2;            // 16 KB: this CTA's A rows or B half
constexpr int kPairStageBytes = 2 * kPairAB;    // 32 KB per CTA per stage
// Output staging per epilogue warp: up to three 32 x 32 bf16 chunks (64-byte rows, 2 KB apart:
// out, then out2 / the second GLU half); none for fp32 outputs, which are stored from registers.
// stages | barriers (padded to 1 KB) | output staging | 1 KB alignment slack
constexpr int pair_smem(int epi) {
  return pair_stages(epi) * kPairStageBytes + 1024 + kEpiWarps * stage_out_bytes(epi) + 1024;
}
static_assert(pair_smem(kEpiStoreF32) <= 232448, "shared memory per CTA");
static_assert(pair_smem(kEpiSwiglu) <= 232448, "shared memory per CTA");

template <bool A_MN, bool B_MN, int EPI, bool F8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC,
                    const __grid_constant__ CUtensorMap tmC2, const GemmArgs args, int num_m2,
                    int num_n, int BN, int staged) {
  // tmC (tmC2: out2 of kEpiGelu): output viewed as {out_ng, M, groups}; for bf16 outputs each
  // epilogue warp stages a 32 x 32 chunk in a swizzled shared buffer (64-byte rows) and stores
  // it with one TMA bulk tensor store (full lines, coalesced; rows past M are clipped); fp32
  // chunks are stored from registers in whole 32-byte sectors. A chunk that straddles N is
  // written element by element instead, and so is every chunk when `staged` is 0 (the host
  // found a column offset that is not a multiple of 16 bytes, which a TMA store cannot start
  // at and the 8-byte fp32 stores assume).
  // BN: the pair's N tile, a multiple of 32 up to 256 (256 when B is MN-major); each CTA
  // loads BN/2 rows of B. Accumulator buffers stay 256 columns apart in TMEM.
  constexpr int STAGES = pair_stages(EPI);
  constexpr int kStageOut = stage_out_bytes(EPI);
  constexpr bool kGlu = EPI == kEpiSwiglu;
  // K elements per stage: one 128-byte swizzle row per operand row (64 bf16 or 128 e4m3);
  // either way a stage holds the same bytes and takes four MMAs of 32 bytes of K each.
  constexpr int KE = F8 ? 128 : BK;
  static_assert(!F8 || (!A_MN && !B_MN && !kGlu), "FP8 operands are K-major");
  const uint32_t b_bytes = (uint32_t)(BN / 2) * BK * 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kPairAB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * kPairStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* stage_out = smem + STAGES * kPairStageBytes + 1024;  // 1024-aligned

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int kt_per_group = (args.Kg + KE - 1) / KE;
  const int k_iters = args.KG * kt_per_group;
  const int num_tiles = args.NG * num_m2 * num_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);  // epilogue warps of both CTAs of the pair
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (staged) {
      tma_prefetch_desc(&tmC);
      if (EPI == kEpiGelu || kGlu) tma_prefetch_desc(&tmC2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrive or load
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dependency_wait();  // the operands are the previous kernel's results

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    SeqCursor cur{0, 0};
    for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
      const TileCoord tc = tile_coord(tile, num_m2, num_n, args.n_fast);
      const int m0 = tc.mb * 256 + rank * 128;
      const int n0 = tc.nb * BN + rank * (BN / 2);
      // token coordinates go through the sequence-parallel row map where set: M of a
      // K-major A once per tile, the K of an MN-major operand through the cursor
      const int am0 = (!A_MN && args.a_sp) ? seq_row(args, m0) : m0;
      for (int kg = 0; kg < args.KG && ok; ++kg) {
        for (int kt = 0; kt < kt_per_group; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, args.err, kErrTimeoutProducer, abort_flag)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (kPairAB + b_bytes));
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          uint8_t* a_dst = sA + stage * kPairAB;
          uint8_t* b_dst = sB + stage * kPairAB;
          const int kk = ((A_MN && args.a_sp) || (B_MN && args.b_sp)) ? cur.row(args, kt * BK)
                                                                       : kt * BK;
          const int ka = args.a_sp ? kk : kt * BK;
          const int kb = args.b_sp ? kk : kt * BK;
          if constexpr (!A_MN) {
            tma_load_3d_pair(&tmA, fb, a_dst, kt * KE, kg, am0);
          } else {
            tma_load_3d_pair(&tmA, fb, a_dst, m0, ka, 0);
            tma_load_3d_pair(&tmA, fb, a_dst + kChunkBytes, m0 + 64, ka, 0);
          }
          if constexpr (kGlu) {
            // GLU tile: this CTA's half of B is the gate (rank 0) or up (rank 1) block of
            // group ng, rows nb*BN/2 ..; the map views B as {K, Ng, 2*NG}.
            tma_load_3d_pair(&tmB, fb, b_dst, kt * BK, tc.nb * (BN / 2), 2 * tc.ng + rank);
          } else if constexpr (!B_MN) {
            tma_load_3d_pair(&tmB, fb, b_dst, kt * KE, n0, kg);
          } else {
            tma_load_3d_pair(&tmB, fb, b_dst, n0, kb, tc.ng);
            tma_load_3d_pair(&tmB, fb, b_dst + kChunkBytes, n0 + 64, kb, tc.ng);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
    // Loads of this CTA complete on the leader's barrier, so only the leader can see them
    // land; the peer relies on the end-of-kernel cluster barrier, which the leader reaches
    // only after its MMA issuer consumed (or gave up on) every stage.
    if (leader) {
      for (int i = 1; i <= STAGES; ++i) {
        int s = stage - i;
        uint32_t ph = phase;
        if (s < 0) {
          s += STAGES;
          ph ^= 1;
        }
        mbar_wait(&full[s], ph, args.err, kErrTimeoutDrain, nullptr);
      }
    }
  } else if (leader && warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    const uint32_t idesc = F8 ? idesc_e4m3_f32(256, BN) : idesc_bf16_f32(256, BN, A_MN, B_MN);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1, args.err, kErrTimeoutMma, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * 256;
      for (int it = 0; it < k_iters; ++it) {
        if (!mbar_wait(&full[stage], phase, args.err, kErrTimeoutMma, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + stage * kPairAB);
        const uint32_t b_addr = smem_u32(sB + stage * kPairAB);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t ad = A_MN ? smem_desc_sw128(a_addr + k * 2048, kChunkBytes, 1024)
                                   : smem_desc_sw128(a_addr + k * 32, 16, 1024);
          const uint64_t bd = B_MN ? smem_desc_sw128(b_addr + k * 2048, kChunkBytes, 1024)
                                   : smem_desc_sw128(b_addr + k * 32, 16, 1024);
          if constexpr (F8)
            tc_mma_f8_pair(d_tmem, ad, bd, idesc, (it > 0 || k > 0) ? 1u : 0u);
          else
            tc_mma_f16_pair(d_tmem, ad, bd, idesc, (it > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit_pair_mc(&empty[stage], 0x3);  // frees the slot in both CTAs
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      tc_commit_pair_mc(&tfull[acc], 0x3);  // both CTAs' accumulator rows are ready
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    tc_commit_pair(drain);
    mbar_wait(drain, 0, args.err, kErrTimeoutDrain, nullptr);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int ew = warp & 3;
    // 32-column chunks, split over 2 warp sets; a GLU tile yields BN/64 output chunks, each
    // from one gate chunk and the up chunk BN/2 columns further on.
    const int nch = kGlu ? BN / 64 : BN / 32, half = (nch + 1) / 2;
    const int c_begin = ((warp - 2) >> 2) ? half : 0;
    const int c_end = ((warp - 2) >> 2) ? nch : half;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    // FP8: dequantisation factor of the product (operand scales, device scalars)
    const float dq = F8 ? __ldg(args.a_scale) * __ldg(args.b_scale) : 1.f;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs) {
      const TileCoord tc = tile_coord(tile, num_m2, num_n, args.n_fast);
      const int row = tc.mb * 256 + rank * 128 + ew * 32 + lane;
      // bf16 epilogues with a residual or u: each staged chunk's source is loaded one chunk
      // ahead, the first one before the accumulator is ready
      constexpr bool kSrcEpi = !kGlu && (EPI == kEpiBf16 || EPI == kEpiDGelu);
      const int src_row0 = tc.mb * 256 + rank * 128 + ew * 32;
      const int src_orow = args.out_sp ? seq_row(args, row) : row;
      auto src_chunk = [&](int c) {  // chunk c is stored staged and reads a source
        const int n0 = tc.nb * BN + c * 32;
        return epi_has_src<EPI>(args) && staged && n0 + 32 <= args.Ng && src_row0 < args.M;
      };
      uint4 src_next[4] = {};
      if constexpr (kSrcEpi)
        if (c_begin < c_end && src_chunk(c_begin))
          epi_load_src<EPI>(args, src_orow, tc.ng * args.Ng + tc.nb * BN + c_begin * 32,
                            row < args.M, src_next);
      const bool ok = mbar_wait(&tfull[acc], acc_phase, args.err, kErrTimeoutEpilogue,
                                abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      if constexpr (kGlu) {
#pragma unroll 1
        for (int c = c_begin; c < c_end; ++c) {
          float vg[32], vu[32];
          const uint32_t t0 = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + acc * 256;
          tmem_ld_32x32b_x32(t0 + c * 32, vg);
          tmem_ld_32x32b_x32(t0 + BN / 2 + c * 32, vu);
          const int n0 = tc.nb * (BN / 2) + c * 32;
          const int row0 = tc.mb * 256 + rank * 128 + ew * 32;
          if (n0 < args.Ng && (n0 + 32 > args.Ng || !staged)) {
            if (row < args.M)
              swiglu_chunk_elem(args, row, tc.ng, n0, min(32, args.Ng - n0), vg, vu);
          } else if (n0 < args.Ng && row0 < args.M) {  // warp-uniform
            uint8_t* buf = stage_out + (warp - 2) * kStageOut;
            uint32_t w[16], w2[16], w3[16];
            swiglu_values(args, tc.ng, n0, vg, vu, w, w2, w3);
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
            const int sw = (lane >> 1) & 3;  // 64-byte swizzle, as below
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int o = lane * 64 + ((j ^ sw) << 4);
              *reinterpret_cast<uint4*>(buf + o) =
                  make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
              *reinterpret_cast<uint4*>(buf + 2048 + o) =
                  make_uint4(w2[4 * j], w2[4 * j + 1], w2[4 * j + 2], w2[4 * j + 3]);
              *reinterpret_cast<uint4*>(buf + 4096 + o) =
                  make_uint4(w3[4 * j], w3[4 * j + 1], w3[4 * j + 2], w3[4 * j + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmC, buf, tc.ng * args.Ng + n0, row0, 0);
              tma_store_3d(&tmC2, buf + 2048, n0, row0, 2 * tc.ng);
              tma_store_3d(&tmC2, buf + 4096, n0, row0, 2 * tc.ng + 1);
              bulk_commit();
            }
          }
        }
      } else {
#pragma unroll 1
      for (int c = c_begin; c < c_end; ++c) {
        if constexpr (EPI == kEpiStoreF32) {
          // fp32 chunk written straight from registers: two 16-lane loads in the 16x256b
          // layout, so each group of four threads stores 32 consecutive bytes of one row
          // (whole sectors) and nothing passes through shared memory, whose port the
          // operand traffic of the next tile's mainloop needs.
          const int n0 = tc.nb * BN + c * 32;
          const int row0 = tc.mb * 256 + rank * 128 + ew * 32;
          if (staged && n0 + 32 <= args.Ng && row0 < args.M) {
            const int col = tc.ng * args.Ng + n0;
            float* o = reinterpret_cast<float*>(args.out) +
                       (long long)(col / args.out_ng) * args.out_gs + (col % args.out_ng) +
                       2 * (lane & 3);
            uint32_t r16[2][16];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
              tmem_ld_16x256b_x4_nw(tmem_base + (static_cast<uint32_t>(ew * 32 + hh * 16) << 16) +
                                        acc * 256 + c * 32,
                                    r16[hh]);
            tmem_ld_wait();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              reg_fence(r16[hh]);
#pragma unroll
              for (int e = 0; e < 2; ++e) {  // rows t/4 and t/4 + 8 of this 16-lane half
                const int rr = row0 + hh * 16 + e * 8 + (lane >> 2);
                if (rr < args.M) {
                  float* orow = o + (long long)(args.out_sp ? seq_row(args, rr) : rr) * args.ldc;
#pragma unroll
                  for (int k = 0; k < 4; ++k)
                    *reinterpret_cast<float2*>(orow + 8 * k) =
                        make_float2(__uint_as_float(r16[hh][4 * k + 2 * e]) * dq,
                                    __uint_as_float(r16[hh][4 * k + 2 * e + 1]) * dq);
                }
              }
            }
            continue;
          }
        }
        uint4 src_cur[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) src_cur[q] = src_next[q];
        if constexpr (kSrcEpi)
          if (c + 1 < c_end && src_chunk(c + 1))
            epi_load_src<EPI>(args, src_orow, tc.ng * args.Ng + tc.nb * BN + (c + 1) * 32,
                              row < args.M, src_next);
        float v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + acc * 256 + c * 32,
                           v);
        if constexpr (F8) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= dq;
        }
        const int n0 = tc.nb * BN + c * 32;
        const int row0 = tc.mb * 256 + rank * 128 + ew * 32;
        const int col = tc.ng * args.Ng + n0;
        // output (and residual) rows in the sequence-parallel layout where set; the 32 rows of
        // a warp stay contiguous there (the shard length is a multiple of 128)
        const int orow = args.out_sp ? seq_row(args, row) : row;
        const int orow0 = args.out_sp ? seq_row(args, row0) : row0;
        // Whole chunks go through TMA; a chunk straddling N is written element by element
        // (the bulk store clips the inner dimension only at 16-byte granularity).
        if (n0 < args.Ng && (n0 + 32 > args.Ng || !staged)) {
          if (row < args.M) epilogue_chunk<EPI>(args, orow, col, min(32, args.Ng - n0), v);
        } else if (n0 < args.Ng && row0 < args.M) {  // warp-uniform
          // (bf16 outputs only: whole fp32 chunks were stored from registers above)
          if constexpr (EPI != kEpiStoreF32) {
            uint8_t* buf = stage_out + (warp - 2) * kStageOut;
            uint32_t w[16], w2[16];
            epi_values_bf16<EPI>(args, orow, col, row < args.M, v, src_cur, w, w2);
            constexpr bool two = EPI == kEpiGelu || EPI == kEpiDSwiglu;
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
            // 64-byte rows, 64-byte swizzle: 16-byte unit j of row r sits at unit
            // j ^ ((r >> 1) & 3), so the 32 lanes' stores fill whole 128-byte wavefronts.
            const int sw = (lane >> 1) & 3;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ sw) << 4)) =
                  make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
              if (two)
                *reinterpret_cast<uint4*>(buf + 2048 + lane * 64 + ((j ^ sw) << 4)) =
                    make_uint4(w2[4 * j], w2[4 * j + 1], w2[4 * j + 2], w2[4 * j + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if constexpr (EPI == kEpiDSwiglu) {  // tmC views dz as {Ng, M, 2*NG}
                tma_store_3d(&tmC, buf, n0, orow0, 2 * tc.ng);
                tma_store_3d(&tmC, buf + 2048, n0, orow0, 2 * tc.ng + 1);
              } else {
                tma_store_3d(&tmC, buf, col % args.out_ng, orow0, col / args.out_ng);
                if (EPI == kEpiGelu)
                  tma_store_3d(&tmC2, buf + 2048, col % args.out_ng, orow0, col / args.out_ng);
              }
              bulk_commit();
            }
          }
        }
      }
      }  // kGlu
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + acc * 8);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  if (warp >= 2 && lane == 0) bulk_wait0();  // staged stores have finished reading smem
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its barriers or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

// 3-D bf16 tensor map with 128-byte swizzle; strides in elements (converted to bytes here).
bool make_tensor_map_bf16_3d(CUtensorMap* m, const void* base, const uint64_t dims[3],
                             const uint64_t strides[2], const uint32_t box[3]) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t gs[2] = {strides[0] * 2, strides[1] * 2};
  cuuint32_t bd[3] = {box[0], box[1], box[2]};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gd, gs, bd,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tensor_map_i32_3d(CUtensorMap* m, const void* base, const uint64_t dims[3],
                            const uint64_t strides[2], const uint32_t box[3]) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t gs[2] = {strides[0] * 4, strides[1] * 4};
  cuuint32_t bd[3] = {box[0], box[1], box[2]};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_INT32, 3, const_cast<void*>(base), gd, gs, bd, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

bool make_map(CUtensorMap* m, const void* base, const uint64_t dims[3], const uint64_t strides[2],
              const uint32_t box[3]) {
  return make_tensor_map_bf16_3d(m, base, dims, strides, box);
}

template <int BN, bool A_MN, bool B_MN, int EPI>
cudaError_t launch_inst(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a,
                        int num_sms, cudaStream_t stream) {
  using C = Cfg<BN>;
  auto kern = gemm_tc_kernel<BN, A_MN, B_MN, EPI>;
  static bool attr_done = false;  // per instantiation
  if (!attr_done) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int num_m = (a.M + BM - 1) / BM;
  const int num_n = (a.Ng + BN - 1) / BN;
  const int tiles = a.NG * num_m * num_n;
  const int grid = tiles < num_sms ? tiles : num_sms;
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(ta, tb, a, num_m, num_n);
  return cudaGetLastError();
}

template <int BN, bool A_MN, bool B_MN>
cudaError_t launch_epi(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a,
                       int num_sms, cudaStream_t s) {
  switch (a.epi) {
    case kEpiStoreF32: return launch_inst<BN, A_MN, B_MN, kEpiStoreF32>(ta, tb, a, num_sms, s);
    case kEpiBf16: return launch_inst<BN, A_MN, B_MN, kEpiBf16>(ta, tb, a, num_sms, s);
    case kEpiGelu: return launch_inst<BN, A_MN, B_MN, kEpiGelu>(ta, tb, a, num_sms, s);
    case kEpiDGelu: return launch_inst<BN, A_MN, B_MN, kEpiDGelu>(ta, tb, a, num_sms, s);
    case kEpiDSwiglu:
      if constexpr (!A_MN && B_MN)
        return launch_inst<BN, A_MN, B_MN, kEpiDSwiglu>(ta, tb, a, num_sms, s);
      break;
  }
  return cudaErrorInvalidValue;
}

// Output tensor map for the staged epilogue store: {out_ng, M, groups}, box 32 x 32; fp32 with
// 128-byte swizzle (128-byte rows), bf16 with 64-byte swizzle (64-byte rows).
bool make_out_map(CUtensorMap* m, const GemmArgs& a, void* base, bool f32) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const long long esz = f32 ? 4 : 2;
  const long long ncols = (long long)a.Ng * a.NG;
  const long long groups = (ncols + a.out_ng - 1) / a.out_ng;
  cuuint64_t gd[3] = {(cuuint64_t)(ncols < a.out_ng ? ncols : a.out_ng), (cuuint64_t)a.M,
                      (cuuint64_t)groups};
  cuuint64_t gs[2] = {(cuuint64_t)(a.ldc * esz),
                      (cuuint64_t)((groups > 1 ? a.out_gs : a.ldc * a.M) * esz)};
  cuuint32_t bd[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base,
            gd, gs, bd, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 view {Ng, M, 2*NG} of a [M][NG][2][Ng] buffer with row stride ld (elements): group
// 2*ng is the gate half of group ng, 2*ng + 1 its up half. Box 32 x 32, 64-byte swizzle.
bool make_glu_map(CUtensorMap* m, const GemmArgs& a, void* base, long long ld) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3] = {(cuuint64_t)a.Ng, (cuuint64_t)a.M, 2 * (cuuint64_t)a.NG};
  cuuint64_t gs[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)a.Ng * 2};
  cuuint32_t bd[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, gd, gs, bd, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool A_MN, bool B_MN, int EPI, bool F8 = false>
cudaError_t launch_pair_inst(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a,
                             int num_sms, int bn, cudaStream_t stream) {
  auto kern = gemm_tc2_kernel<A_MN, B_MN, EPI, F8>;
  constexpr int smem_bytes = pair_smem(EPI);
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  CUtensorMap tc, tc2;
  std::memset(&tc, 0, sizeof(tc));
  std::memset(&tc2, 0, sizeof(tc2));
  // A staged store covers output columns col .. col+31, col = ng*Ng + n0 with n0 a multiple of
  // 32, at inner coordinate col % out_ng. It needs col to be a multiple of 16 bytes' worth of
  // elements (true for one group, else Ng must be) and must not run across an out_ng boundary
  // (true if one out_ng block holds every column, else out_ng must be a multiple of 32).
  // Tensor-map encoding also needs 16-byte aligned bases and strides.
  // The SwiGLU epilogues store [gate | up] halves through a view {Ng, M, 2*NG} of their
  // buffer (row stride ldc2 / ldc, group stride Ng), at inner coordinate n0: they need Ng to
  // be a multiple of 32 (whole chunks inside a group) and the SwiGLU forward also stores a at
  // column ng*Ng + n0 of out.
  const int vec = EPI == kEpiStoreF32 ? 4 : 8;
  int staged;
  if (EPI == kEpiSwiglu || EPI == kEpiDSwiglu) {
    staged = a.Ng % 32 == 0 ? 1 : 0;
    if (staged && !make_glu_map(&(EPI == kEpiSwiglu ? tc2 : tc), a,
                                EPI == kEpiSwiglu ? a.out2 : a.out,
                                EPI == kEpiSwiglu ? a.ldc2 : a.ldc))
      staged = 0;
    if (staged && EPI == kEpiSwiglu && !make_out_map(&tc, a, a.out, false)) staged = 0;
  } else {
    const bool cols_ok = (a.NG == 1 || a.Ng % vec == 0) &&
                         ((long long)a.out_ng >= (long long)a.Ng * a.NG || a.out_ng % 32 == 0);
    staged = cols_ok ? 1 : 0;
    if (staged && !make_out_map(&tc, a, a.out, EPI == kEpiStoreF32)) staged = 0;
    if (staged && EPI == kEpiGelu && !make_out_map(&tc2, a, a.out2, false)) staged = 0;
  }
  const int num_m2 = (a.M + 255) / 256;
  const int tile_cols = EPI == kEpiSwiglu ? bn / 2 : bn;  // outputs per tile and group
  const int num_n = (a.Ng + tile_cols - 1) / tile_cols;
  const int tiles = a.NG * num_m2 * num_n;
  const int pairs = tiles < num_sms / 2 ? tiles : num_sms / 2;
  return launch_kernel(!a.plain_launch, kern, dim3(2 * pairs), dim3(kThreads), smem_bytes,
                       stream, ta, tb, tc, tc2, a, num_m2, num_n, bn, staged);
}

template <bool A_MN, bool B_MN>
cudaError_t launch_pair_epi(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a,
                            int num_sms, int bn, cudaStream_t s) {
  switch (a.epi) {
    case kEpiStoreF32:
      return launch_pair_inst<A_MN, B_MN, kEpiStoreF32>(ta, tb, a, num_sms, bn, s);
    case kEpiBf16: return launch_pair_inst<A_MN, B_MN, kEpiBf16>(ta, tb, a, num_sms, bn, s);
    case kEpiGelu: return launch_pair_inst<A_MN, B_MN, kEpiGelu>(ta, tb, a, num_sms, bn, s);
    case kEpiDGelu: return launch_pair_inst<A_MN, B_MN, kEpiDGelu>(ta, tb, a, num_sms, bn, s);
    case kEpiSwiglu:
      if constexpr (!A_MN && !B_MN)
        return launch_pair_inst<A_MN, B_MN, kEpiSwiglu>(ta, tb, a, num_sms, bn, s);
      break;
    case kEpiDSwiglu:
      if constexpr (!A_MN && B_MN)
        return launch_pair_inst<A_MN, B_MN, kEpiDSwiglu>(ta, tb, a, num_sms, bn, s);
      break;
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a,
                        int num_sms, int bn, cudaStream_t s) {
  if (!a.a_mn && !a.b_mn) return launch_pair_epi<false, false>(ta, tb, a, num_sms, bn, s);
  if (!a.a_mn && a.b_mn) return launch_pair_epi<false, true>(ta, tb, a, num_sms, bn, s);
  if (a.a_mn && !a.b_mn) return launch_pair_epi<true, false>(ta, tb, a, num_sms, bn, s);
  return launch_pair_epi<true, true>(ta, tb, a, num_sms, bn, s);
}

// N tile of the pair kernel: the width (multiple of 32, <= 256) that minimises the number of
// tile rounds over the pairs times the tile width (+ a fixed per-tile cost), so the last round
// is as full as possible. MN-major B loads 64-wide chunks per CTA half, so it keeps 256.
int pick_pair_bn(const GemmArgs& a, int num_sms) {
  if (a.b_mn) return 256;
  const bool glu = a.epi == kEpiSwiglu;  // a GLU tile covers bn/2 outputs (gate + up halves)
  const int pairs = num_sms / 2;
  const long long m2 = (a.M + 255) / 256;
  int best = 256;
  long long best_cost = -1;
  for (int bn = 256; bn >= (glu ? 64 : 128); bn -= (glu ? 64 : 32)) {
    const int cols = glu ? bn / 2 : bn;
    const long long tiles = (long long)a.NG * m2 * ((a.Ng + cols - 1) / cols);
    const long long rounds = (tiles + pairs - 1) / pairs;
    const long long cost = rounds * (bn + 48);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a,
                      int num_sms, cudaStream_t s) {
  if (!a.a_mn && !a.b_mn) return launch_epi<BN, false, false>(ta, tb, a, num_sms, s);
  if (!a.a_mn && a.b_mn) return launch_epi<BN, false, true>(ta, tb, a, num_sms, s);
  if (a.a_mn && !a.b_mn) return launch_epi<BN, true, false>(ta, tb, a, num_sms, s);
  return launch_epi<BN, true, true>(ta, tb, a, num_sms, s);
}

}  // namespace

// FP8 GEMM: C = (A B^T) * (*a_scale) * (*b_scale) with e4m3 A [M][K] and B [N][K] (K-major,
// strides lda / ldb bytes-as-elements), on the CTA-pair kernel with 128-element K stages.
cudaError_t launch_gemm_fp8(const GemmArgs& a, int num_sms, cudaStream_t stream) {
  if (a.M <= 0 || a.Ng <= 0 || a.Kg <= 0 || a.NG != 1 || a.KG != 1 || a.a_mn || a.b_mn ||
      !a.a_scale || !a.b_scale || num_sms < 2 ||
      (a.epi != kEpiStoreF32 && a.epi != kEpiBf16))
    return cudaErrorInvalidValue;
  auto fn = get_encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  const int bn = pick_pair_bn(a, num_sms);
  auto map_u8 = [&](CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t ld, uint32_t box_rows) {
    cuuint64_t gd[3] = {inner, 1, rows};
    cuuint64_t gs[2] = {ld, ld};
    cuuint32_t bd[3] = {128, 1, box_rows};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), gd, gs, bd, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
  };
  // A viewed as {K, 1, M}: coordinates (k, 0, m) like a bf16 K-major A with one K group;
  // B as {K, N, 1}: coordinates (k, n, 0).
  CUtensorMap ta, tb;
  if (!map_u8(&ta, a.A, a.Kg, a.M, a.lda, BM)) return cudaErrorInvalidValue;
  {
    cuuint64_t gd[3] = {(cuuint64_t)a.Kg, (cuuint64_t)a.Ng, 1};
    cuuint64_t gs[2] = {(cuuint64_t)a.ldb, (cuuint64_t)a.ldb * a.Ng};
    cuuint32_t bd[3] = {128, (cuuint32_t)(bn / 2), 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (fn(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(a.B), gd, gs, bd, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (a.epi == kEpiStoreF32)
    return launch_pair_inst<false, false, kEpiStoreF32, true>(ta, tb, a, num_sms, bn, stream);
  return launch_pair_inst<false, false, kEpiBf16, true>(ta, tb, a, num_sms, bn, stream);
}

cudaError_t launch_gemm_tc(const GemmArgs& a, int num_sms, cudaStream_t stream) {
  // Shape rules of the tensor maps (checked by the callers too).
  if (a.M <= 0 || a.Ng <= 0 || a.NG <= 0 || a.Kg <= 0 || a.KG <= 0) return cudaErrorInvalidValue;
  const bool glu = a.epi == kEpiSwiglu;
  if ((a.a_mn && a.KG != 1) || (a.b_mn && a.KG != 1) || (!a.b_mn && a.NG != 1 && !glu))
    return cudaErrorInvalidValue;
  if (glu && (a.a_mn || a.b_mn || a.KG != 1 || num_sms < 2)) return cudaErrorInvalidValue;
  if (a.epi == kEpiDSwiglu && (a.a_mn || !a.b_mn)) return cudaErrorInvalidValue;
  // Wide tiles run on CTA pairs (cta_group::2, 256 x BN per pair); narrow N on one CTA. GLU
  // tiles (gate and up halves from the two CTAs) exist only on pairs.
  const bool pair = (a.Ng > 128 || glu) && num_sms >= 2;
  const int BN = (a.Ng <= 128) ? 128 : 256;
  const int pair_bn = pair ? pick_pair_bn(a, num_sms) : BN;
  const int b_rows = pair ? pair_bn / 2 : BN;  // B rows per CTA per k-step
  CUtensorMap ta, tb;
  {
    uint64_t dims[3], str[2];
    uint32_t box[3];
    if (!a.a_mn) {
      dims[0] = a.Kg; dims[1] = a.KG; dims[2] = a.M;
      str[0] = a.KG > 1 ? (uint64_t)a.Kg : (uint64_t)a.lda;
      str[1] = a.lda;
      box[0] = BK; box[1] = 1; box[2] = BM;
    } else {
      dims[0] = a.M; dims[1] = a.Kg; dims[2] = 1;
      str[0] = a.lda; str[1] = a.lda;
      box[0] = 64; box[1] = BK; box[2] = 1;
    }
    if (!make_map(&ta, a.A, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[3], str[2];
    uint32_t box[3];
    if (glu) {  // B rows [NG][2][Ng] (gate block, up block per group) viewed as {K, Ng, 2*NG}
      dims[0] = a.Kg; dims[1] = a.Ng; dims[2] = 2 * (uint64_t)a.NG;
      str[0] = a.ldb;
      str[1] = (uint64_t)a.Ng * a.ldb;
      box[0] = BK; box[1] = b_rows; box[2] = 1;
    } else if (!a.b_mn) {
      dims[0] = a.Kg; dims[1] = a.Ng; dims[2] = a.KG;
      str[0] = a.ldb;
      str[1] = a.KG > 1 ? (uint64_t)a.b_kgs : (uint64_t)a.ldb;
      box[0] = BK; box[1] = b_rows; box[2] = 1;
    } else {
      dims[0] = a.Ng; dims[1] = a.Kg; dims[2] = a.NG;
      str[0] = a.ldb;
      str[1] = a.NG > 1 ? (uint64_t)a.b_ngs : (uint64_t)a.ldb;
      box[0] = 64; box[1] = BK; box[2] = 1;
    }
    if (!make_map(&tb, a.B, dims, str, box)) return cudaErrorInvalidValue;
  }
  GemmArgs ka = a;
  ka.n_fast = (long long)a.M > (long long)a.Ng * a.NG ? 1 : 0;
  if (pair) return launch_pair(ta, tb, ka, num_sms, pair_bn, stream);
  if (BN == 128) return launch_bn<128>(ta, tb, ka, num_sms, stream);
  return launch_bn<256>(ta, tb, ka, num_sms, stream);
}

}  // namespace mgt
