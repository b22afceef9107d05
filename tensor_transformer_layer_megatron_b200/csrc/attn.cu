// Causal multi-head attention, forward and backward, on the packed qkv of the column-parallel
// QKV projection: qkv [T][p][3][H/p][d]. Each logical shard owns whole heads, so every head's
// softmax is local (the trdm.cn page, section 2.1: column-split Q/K/V let each shard compute its
// heads without communication). Softmax arithmetic is fp32 (section 3.2,
// attention_softmax_in_fp32). Scale 1/sqrt(d); key j visible to query i iff j <= i.
//
// bf16 path: the forward runs on tcgen05 (attn_tc.cu). The backward here is FlashAttention-
// style tiling on mma.sync m16n8k16 with ldmatrix from swizzled shared memory and cp.async
// double buffering; it recomputes the probabilities from the saved log-sum-exp (the page's
// section 4.1 recompute), keeps dK/dV in registers per key block, and accumulates dQ with
// fp32 atomics into a workspace buffer that a last pass scales and converts.
// fp32 path: plain per-row kernels (tiny shapes only).
#include "mgt_device.cuh"

namespace mgt {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

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

// ============================================================================ bf16 helpers
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Shared-memory tile [rows][D] bf16 with 16-byte chunks XOR-swizzled by row: conflict-free
// ldmatrix for 8 consecutive rows at one logical chunk.
template <int D>
__device__ __forceinline__ uint32_t tile_addr(uint32_t base, int r, int chunk) {
  return base + r * (D * 2) + ((chunk ^ (r & 7)) << 4);
}

// Copy `rows` rows of D bf16 (global row stride ld elements, first row r0 of `nvalid`) into a
// swizzled tile; rows >= nvalid are zero-filled.
template <int D, int NT>
__device__ __forceinline__ void load_tile(uint32_t sbase, const __nv_bfloat16* g, long long ld,
                                          int r0, int rows, int nvalid) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  for (int i = threadIdx.x; i < rows * CPR; i += NT) {
    const int r = i / CPR, c = i % CPR;
    const int gr = r0 + r;
    const bool ok = gr < nvalid;
    const __nv_bfloat16* src = g + (long long)(ok ? gr : 0) * ld + c * 8;
    cp_async16(tile_addr<D>(sbase, r, c), src, ok);
  }
}

// ============================================================================ bf16 backward
// D[b][n][q] = sum_c dO[q, n*d + c] * O[q, n*d + c]; one warp per (token, head).
template <int D>
__global__ void attn_bwd_pre_kernel(AttnArgs a) {
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long total = (long long)a.b * a.s * a.H;
  if (w >= total) return;
  const int n = (int)(w % a.H);
  const long long tok = w / a.H;
  const int b = (int)(tok / a.s), q = (int)(tok % a.s);
  constexpr int E = D / 32;  // 2 or 4 elements per lane
  const __nv_bfloat16* o = reinterpret_cast<const __nv_bfloat16*>(a.o) + tok * a.H * D + n * D;
  const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(a.dO) + tok * a.H * D + n * D;
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const uint32_t ov = *reinterpret_cast<const uint32_t*>(o + lane * E + e);
    const uint32_t dv = *reinterpret_cast<const uint32_t*>(dO + lane * E + e);
    s += bf16_lo(ov) * bf16_lo(dv) + bf16_hi(ov) * bf16_hi(dv);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) a.Dsum[((long long)b * a.H + n) * a.s + q] = s;
}

// Key block of 64 per CTA (16 keys per warp), query blocks of 32 streamed through.
template <int D>
__global__ void __launch_bounds__(128) attn_bwd_bf16_kernel(AttnArgs a, float scale_log2,
                                                            float scale) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sK = smem_u32(smem);
  const uint32_t sV = sK + 64 * D * 2;
  const uint32_t sQ0 = sV + 64 * D * 2;          // [2][32][D]
  const uint32_t sdO0 = sQ0 + 2 * 32 * D * 2;    // [2][32][D]
  const uint32_t sdS = sdO0 + 2 * 32 * D * 2;    // [64 keys][32 queries] bf16
  float* sL = reinterpret_cast<float*>(smem + 4 * 64 * D * 2 + 64 * 32 * 2);  // [2][32]
  float* sDv = sL + 64;                                                     // [2][32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const int S = a.s, H = a.H, hp = H / a.p;
  const int kb = blockIdx.x;
  const int bh = blockIdx.y, b = bh / H, n = bh % H, t = n / hp, jh = n % hp;
  const long long ld = 3LL * H * D;
  const long long head_off = (long long)b * S * ld + (long long)t * 3 * hp * D + (long long)jh * D;
  const __nv_bfloat16* qg = reinterpret_cast<const __nv_bfloat16*>(a.qkv) + head_off;
  const __nv_bfloat16* kg = qg + (long long)hp * D;
  const __nv_bfloat16* vg = qg + 2LL * hp * D;
  const long long ldo = (long long)H * D;
  const __nv_bfloat16* dOg = reinterpret_cast<const __nv_bfloat16*>(a.dO) + (long long)b * S * ldo +
                             (long long)n * D;
  const float* lse_g = a.lse + ((long long)b * H + n) * S;
  const float* D_g = a.Dsum + ((long long)b * H + n) * S;

  const int q_first = (kb * 64) / 32;  // first query block that sees any key of this block
  const int nq = (S + 31) / 32;

  load_tile<D, 128>(sK, kg, ld, kb * 64, 64, S);
  load_tile<D, 128>(sV, vg, ld, kb * 64, 64, S);
  cp_async_commit();
  auto load_q = [&](int qi, int buf) {
    load_tile<D, 128>(sQ0 + buf * 32 * D * 2, qg, ld, qi * 32, 32, S);
    load_tile<D, 128>(sdO0 + buf * 32 * D * 2, dOg, ldo, qi * 32, 32, S);
    if (threadIdx.x < 32) {
      const int q = qi * 32 + threadIdx.x;
      sL[buf * 32 + threadIdx.x] = q < S ? lse_g[q] * kLog2e : 0.f;
      sDv[buf * 32 + threadIdx.x] = q < S ? D_g[q] : 0.f;
    }
  };
  if (q_first < nq) load_q(q_first, 0);
  cp_async_commit();

  float dv[D / 8][4], dk[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dv[i][e] = dk[i][e] = 0.f;

  for (int qi = q_first; qi < nq; ++qi) {
    const int buf = (qi - q_first) & 1;
    if (qi + 1 < nq) {
      load_q(qi + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sQ = sQ0 + buf * 32 * D * 2, sdO = sdO0 + buf * 32 * D * 2;
    const float* L = sL + buf * 32;
    const float* Dq = sDv + buf * 32;

    // S^T = K Q^T (16 keys x 32 queries per warp) and dP^T = V dO^T
    float st[4][4], dpt[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[i][e] = dpt[i][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int mi = lane >> 3, r = lane & 7;
      uint32_t k0, k1, k2, k3, v0, v1, v2, v3;
      ldsm_x4(tile_addr<D>(sK, warp * 16 + (mi & 1) * 8 + r, ks * 2 + (mi >> 1)), k0, k1, k2, k3);
      ldsm_x4(tile_addr<D>(sV, warp * 16 + (mi & 1) * 8 + r, ks * 2 + (mi >> 1)), v0, v1, v2, v3);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tile_addr<D>(sQ, np * 16 + (mi >> 1) * 8 + r, ks * 2 + (mi & 1)), b0, b1, b2, b3);
        mma16816(st[2 * np], k0, k1, k2, k3, b0, b1);
        mma16816(st[2 * np + 1], k0, k1, k2, k3, b2, b3);
        ldsm_x4(tile_addr<D>(sdO, np * 16 + (mi >> 1) * 8 + r, ks * 2 + (mi & 1)), b0, b1, b2, b3);
        mma16816(dpt[2 * np], v0, v1, v2, v3, b0, b1);
        mma16816(dpt[2 * np + 1], v0, v1, v2, v3, b2, b3);
      }
    }
    // P^T and dS^T = P^T * (dP^T - D)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kb * 64 + warp * 16 + g + (e >= 2 ? 8 : 0);
        const int ql = nt * 8 + 2 * q4 + (e & 1);
        const int query = qi * 32 + ql;
        float p = exp2f(st[nt][e] * scale_log2 - L[ql]);
        if (key > query || query >= S) p = 0.f;
        st[nt][e] = p;
        dpt[nt][e] = p * (dpt[nt][e] - Dq[ql]);
      }
    }
    // dV += P^T dO ; dK += dS^T Q  (k = queries, two k-steps of 16)
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const uint32_t pa0 = pack_bf16x2(st[2 * kk][0], st[2 * kk][1]);
      const uint32_t pa1 = pack_bf16x2(st[2 * kk][2], st[2 * kk][3]);
      const uint32_t pa2 = pack_bf16x2(st[2 * kk + 1][0], st[2 * kk + 1][1]);
      const uint32_t pa3 = pack_bf16x2(st[2 * kk + 1][2], st[2 * kk + 1][3]);
      const uint32_t sa0 = pack_bf16x2(dpt[2 * kk][0], dpt[2 * kk][1]);
      const uint32_t sa1 = pack_bf16x2(dpt[2 * kk][2], dpt[2 * kk][3]);
      const uint32_t sa2 = pack_bf16x2(dpt[2 * kk + 1][0], dpt[2 * kk + 1][1]);
      const uint32_t sa3 = pack_bf16x2(dpt[2 * kk + 1][2], dpt[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        const int mi = lane >> 3, r = lane & 7;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(tile_addr<D>(sdO, kk * 16 + (mi & 1) * 8 + r, dp * 2 + (mi >> 1)), b0, b1, b2, b3);
        mma16816(dv[2 * dp], pa0, pa1, pa2, pa3, b0, b1);
        mma16816(dv[2 * dp + 1], pa0, pa1, pa2, pa3, b2, b3);
        ldsm_x4_t(tile_addr<D>(sQ, kk * 16 + (mi & 1) * 8 + r, dp * 2 + (mi >> 1)), b0, b1, b2, b3);
        mma16816(dk[2 * dp], sa0, sa1, sa2, sa3, b0, b1);
        mma16816(dk[2 * dp + 1], sa0, sa1, sa2, sa3, b2, b3);
      }
    }
    // dS^T -> shared [64 keys][32 queries], 64-byte rows, chunk swizzle c ^ ((row >> 1) & 3)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = warp * 16 + g + hh * 8;
        const int col = nt * 8 + 2 * q4;
        const uint32_t addr = sdS + row * 64 + (((col >> 3) ^ ((row >> 1) & 3)) << 4) + (col & 7) * 2;
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr),
                     "r"(pack_bf16x2(dpt[nt][2 * hh], dpt[nt][2 * hh + 1])));
      }
    }
    __syncthreads();
    // dQ (32 queries x D) += dS K: warp w takes query rows (w&1)*16.., columns half (w>>1)
    {
      float dq[D / 16][4];
#pragma unroll
      for (int i = 0; i < D / 16; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
      const int m0 = (warp & 1) * 16;
      const int nbase = (warp >> 1) * (D / 16);  // in 8-column tiles
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {  // 64 keys
        const int mi = lane >> 3, r = lane & 7;
        const int krow = ks * 16 + (mi >> 1) * 8 + r;
        const int mchunk = (m0 >> 3) + (mi & 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(sdS + krow * 64 + ((mchunk ^ ((krow >> 1) & 3)) << 4), a0, a1, a2, a3);
#pragma unroll
        for (int np = 0; np < D / 32; ++np) {
          uint32_t b0, b1, b2, b3;
          const int dchunk = (nbase >> 0) + np * 2;  // 8-col tile index == 16-byte chunk index
          ldsm_x4_t(tile_addr<D>(sK, ks * 16 + (mi & 1) * 8 + r, dchunk + (mi >> 1)), b0, b1, b2, b3);
          mma16816(dq[2 * np], a0, a1, a2, a3, b0, b1);
          mma16816(dq[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      float* dqa = a.dq_acc + (long long)b * S * ldo + (long long)n * D;
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int query = qi * 32 + m0 + g + hh * 8;
          if (query < S) {
            float* p = dqa + (long long)query * ldo + (nbase + i) * 8 + 2 * q4;
            atomicAdd(p, dq[i][2 * hh]);
            atomicAdd(p + 1, dq[i][2 * hh + 1]);
          }
        }
      }
    }
    __syncthreads();  // sdS and this Q/dO buffer are free again
  }

  // write dK (scaled) and dV for this warp's 16 keys
  __nv_bfloat16* dg = reinterpret_cast<__nv_bfloat16*>(a.dqkv) + head_off;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int key = kb * 64 + warp * 16 + g + hh * 8;
    if (key < S) {
      __nv_bfloat16* dkr = dg + (long long)key * ld + (long long)hp * D;
      __nv_bfloat16* dvr = dg + (long long)key * ld + 2LL * hp * D;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        *reinterpret_cast<uint32_t*>(dkr + i * 8 + 2 * q4) =
            pack_bf16x2(dk[i][2 * hh] * scale, dk[i][2 * hh + 1] * scale);
        *reinterpret_cast<uint32_t*>(dvr + i * 8 + 2 * q4) =
            pack_bf16x2(dv[i][2 * hh], dv[i][2 * hh + 1]);
      }
    }
  }
}

// dq slots of dqkv = bf16(dq_acc * scale)
__global__ void attn_dq_convert_kernel(AttnArgs a, float scale) {
  const long long total = (long long)a.b * a.s * a.H * a.d;
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= total) return;
  const int hd = a.H * a.d;
  const long long tok = i / hd;
  const int c = (int)(i % hd);
  const int n = c / a.d, e = c % a.d, hp = a.H / a.p, t = n / hp, jh = n % hp;
  const float4 v = *reinterpret_cast<const float4*>(a.dq_acc + i);
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.dqkv) + tok * 3LL * hd +
                       (long long)t * 3 * hp * a.d + (long long)jh * a.d + e;
  uint2 w;
  w.x = pack_bf16x2(v.x * scale, v.y * scale);
  w.y = pack_bf16x2(v.z * scale, v.w * scale);
  *reinterpret_cast<uint2*>(dst) = w;
}

template <int D>
constexpr int bwd_smem() { return 4 * 64 * D * 2 + 64 * 32 * 2 + 4 * 32 * 4; }

template <int D>
cudaError_t bwd_bf16(const AttnArgs& a, cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_bf16_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bwd_smem<D>());
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const long long T = (long long)a.b * a.s;
  cudaError_t e = cudaMemsetAsync(a.dq_acc, 0, sizeof(float) * T * a.H * D, s);
  if (e != cudaSuccess) return e;
  const long long warps = T * a.H;
  attn_bwd_pre_kernel<D><<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 grid((a.s + 63) / 64, a.b * a.H);
  const float scale = 1.f / sqrtf((float)D);
  attn_bwd_bf16_kernel<D><<<grid, 128, bwd_smem<D>(), s>>>(a, kLog2e * scale, scale);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long n4 = T * a.H * D / 4;
  attn_dq_convert_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(a, scale);
  return cudaGetLastError();
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
  if (a.d == 64) return bwd_bf16<64>(a, s);
  if (a.d == 128) return bwd_bf16<128>(a, s);
  return cudaErrorInvalidValue;
}

int attn_bwd_kernel_count(int dtype) { return dtype ? 3 : 1; }

}  // namespace mgt
