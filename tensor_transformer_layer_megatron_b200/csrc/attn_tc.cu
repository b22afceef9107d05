// Causal attention on the fifth-generation tensor cores (tcgen05 + TMEM + TMA): the forward,
// and the backward with the probabilities recomputed from the saved log-sum-exp (below).
//
// The heads are local to their tensor-parallel shard (the column split of W_q/W_k/W_v on the
// trdm.cn page, section 2.1, keeps whole heads on a shard), so the softmax never needs another
// shard's data. Softmax arithmetic is fp32 (section 3.2, attention_softmax_in_fp32); scale
// 1/sqrt(d); key j visible to query i iff j <= i.
//
// Forward: one CTA per pair of consecutive 128-query tiles of one head, longest pairs first.
// Per tile and key block of 128 (double-buffered K/V tiles from TMA):
//   S = Q K^T            tcgen05.mma M=128 N=128, fp32 into the tile's S buffer in TMEM
//   softmax warps        one thread per query row reads all 128 of its scores with tcgen05.ld,
//                        so the row max and sum need no exchange between threads;
//                        P = exp2(S*scale*log2e - m) is packed to bf16 and written back into the
//                        first 64 columns of the same S buffer
//   O += P V             tcgen05.mma M=128 N=d with A = P read from TMEM and V read N-major
//                        straight from its TMA tile
// One tile's softmax runs while the tensor pipe works on the other tile's products, and P
// reaches the MMA in two halves of 64 keys so that PV starts before the softmax ends. The
// running max is updated lazily: O and the row sum are rescaled only when a row's max grows by
// more than 2^8 (P stays <= 256 otherwise, exact in fp32 and safe in bf16). Finally O / l is
// staged in bf16 in the tile's Q buffer and written by bulk tensor stores, and
// lse = (m + log2 l) * ln 2.
//
// Forward warps: 0-3 softmax and output of query tile 0, 4-7 of tile 1 (warp w owns TMEM lanes
// 32 (w % 4) .., i.e. query rows); warp 8 TMA producer; warp 9 TMEM owner and MMA issuer.
// Every wait is bounded.
#include "mgt_device.cuh"

namespace mgt {
namespace {

constexpr float kLog2eF = 1.4426950408889634f;
constexpr float kLn2F = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct FwdLayout {
  static constexpr int CH = D / 64;              // 64-wide (128-byte) swizzle chunks per row
  static constexpr int TILE = 128 * D * 2;       // one 128-row Q, K or V tile
  static constexpr int Q_OFF = 0;                // 2 tiles: query blocks q0 and q0 + 1
  static constexpr int K_OFF = 2 * TILE;         // 2 stages
  static constexpr int V_OFF = K_OFF + 2 * TILE; // 2 stages
  static constexpr int BAR_OFF = V_OFF + 2 * TILE;
  static constexpr int BYTES = BAR_OFF + 256 + 1024;
  // TMEM per query tile: one S buffer (P packed into its first 64 columns) and one O
  static constexpr int TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O0 = 256, TMEM_O1 = 256 + D;
};

// Forward CTA: warps 0-3 softmax of query tile 0, warps 4-7 of tile 1 (warp w: TMEM lane
// quarter w % 4), warp 8 TMA, warp 9 MMA.
constexpr int kAttnFwdThreads = 320;
// Backward CTAs: warps 0-7 do the elementwise work on TMEM rows (warp w: TMEM lane quarter w%4,
// column half w/4), warp 8 is the TMA producer, warp 9 owns TMEM and issues MMAs.
constexpr int kBwdThreads = 320;

template <int D>
__global__ void __launch_bounds__(kAttnFwdThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm,
                       const __grid_constant__ CUtensorMap tm_o, const AttnArgs a,
                       float scale_log2) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2] stages
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* k_empty = bars + 5;   // [2]: released once every S of that block has read K
  uint64_t* v_empty = bars + 7;   // [2]: released once every PV of that block has read V
  uint64_t* s_full = bars + 9;    // [2] per tile: S of the tile's current block is in TMEM
  // [2 tiles][2 halves]: P of keys 0-63 / 64-127 of the tile's current block is in TMEM
  uint64_t* p_half = bars + 11;
  uint64_t* drain = bars + 15;    // every MMA done (one-shot: the output waits on it)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.s, H = a.H, hp = H / a.p;
  const int nqb = (S + 127) / 128, npair = (nqb + 1) / 2;
  // Heads vary fastest in the launch order and pairs of query blocks run from the longest
  // rows down (longest-processing-time order). Tile u of the pair is query block q0 + u.
  const int q0 = 2 * (npair - 1 - (int)blockIdx.y);
  const bool two = q0 + 1 < nqb;   // the pair has a second tile
  const int last = two ? q0 + 1 : q0;  // last key block any tile of the pair needs
  const int bh = blockIdx.x, b = bh / H, n = bh % H, t = n / hp, jh = n % hp;
  const int col_q = t * 3 * hp * D + jh * D, col_k = col_q + hp * D, col_v = col_q + 2 * hp * D;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_half[2 * i], 4);
      mbar_init(&p_half[2 * i + 1], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();  // qkv is the previous kernel's result

  if (warp == 8) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      mbar_arrive_expect_tx(q_full, (two ? 2 : 1) * L::TILE);
      for (int u = 0; u < (two ? 2 : 1); ++u)
#pragma unroll
        for (int c = 0; c < L::CH; ++c)
          tma_load_3d(&tm, q_full, smem + L::Q_OFF + u * L::TILE + c * 16384, col_q + c * 64,
                      (q0 + u) * 128, b);
      int issued_k = 0, issued_v = 0;
      for (int kb = 0; kb <= last; ++kb) {
        const int st = kb & 1;
        if (!mbar_wait(&k_empty[st], ((kb >> 1) & 1) ^ 1, a.err, kErrTimeoutAttn, abort_flag))
          break;
        mbar_arrive_expect_tx(&k_full[st], L::TILE);
#pragma unroll
        for (int c = 0; c < L::CH; ++c)
          tma_load_3d(&tm, &k_full[st], smem + L::K_OFF + st * L::TILE + c * 16384,
                      col_k + c * 64, kb * 128, b);
        issued_k = kb + 1;
        if (!mbar_wait(&v_empty[st], ((kb >> 1) & 1) ^ 1, a.err, kErrTimeoutAttn, abort_flag))
          break;
        mbar_arrive_expect_tx(&v_full[st], L::TILE);
#pragma unroll
        for (int c = 0; c < L::CH; ++c)
          tma_load_3d(&tm, &v_full[st], smem + L::V_OFF + st * L::TILE + c * 16384,
                      col_v + c * 64, kb * 128, b);
        issued_v = kb + 1;
      }
      // every issued load lands before the CTA can exit
      mbar_wait(q_full, 0, a.err, kErrTimeoutDrain, nullptr);
      for (int kb = issued_k - 2 < 0 ? 0 : issued_k - 2; kb < issued_k; ++kb)
        mbar_wait(&k_full[kb & 1], (kb >> 1) & 1, a.err, kErrTimeoutDrain, nullptr);
      for (int kb = issued_v - 2 < 0 ? 0 : issued_v - 2; kb < issued_v; ++kb)
        mbar_wait(&v_full[kb & 1], (kb >> 1) & 1, a.err, kErrTimeoutDrain, nullptr);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // Order per key block kb: S0(kb), S1(kb) | PV0(kb), S0(kb+1), PV1(kb), S1(kb+1) | ...
      // so that one tile's softmax overlaps the other tile's products. A tile's S(kb+1)
      // overwrites the P that its PV(kb) reads, and is issued after it (tcgen05.mma
      // operations of one thread execute in issue order); the commit of S(kb+1) therefore
      // also covers PV(kb), so the softmax may rescale O once it has seen S(kb+1).
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      bool ok = mbar_wait(q_full, 0, a.err, kErrTimeoutAttn, abort_flag);
      auto issue_s = [&](int u, int kb) -> bool {  // S_u = Q_u K_kb^T
        const int st = kb & 1;
        if (!mbar_wait(&k_full[st], (kb >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::Q_OFF + u * L::TILE);
        const uint32_t k_addr = smem_u32(smem + L::K_OFF + st * L::TILE);
        const uint32_t d = tmem + (u ? L::TMEM_S1 : L::TMEM_S0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc_mma_f16(d, smem_desc_sw128(q_addr + off, 16, 1024),
                     smem_desc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[u]);
        return true;
      };
      auto issue_pv = [&](int u, int kb) -> bool {  // O_u += P_u V_kb, keys 0-63 first
        if (!mbar_wait(&v_full[kb & 1], (kb >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag))
          return false;
        const uint32_t v_addr = smem_u32(smem + L::V_OFF + (kb & 1) * L::TILE);
        const uint32_t p_tmem = tmem + (u ? L::TMEM_S1 : L::TMEM_S0);
        const uint32_t o_tmem = tmem + (u ? L::TMEM_O1 : L::TMEM_O0);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!mbar_wait(&p_half[2 * u + hf], kb & 1, a.err, kErrTimeoutAttn, abort_flag))
            return false;
          tc_fence_after();
#pragma unroll
          for (int kk = hf * 4; kk < hf * 4 + 4; ++kk)  // 16 keys (8 packed P columns) each
            tc_mma_f16_tmem_a(o_tmem, p_tmem + kk * 8,
                              smem_desc_sw128(v_addr + kk * 2048, 16384, 1024), idesc_o,
                              (kb > 0 || kk > 0) ? 1u : 0u);
        }
        return true;
      };
      if (ok) ok = issue_s(0, 0);
      if (ok && two) ok = issue_s(1, 0);
      if (ok) tc_commit(&k_empty[0]);  // every S of block 0 is issued
      for (int kb = 0; kb <= last && ok; ++kb) {
        const bool a_on = kb <= q0, a_next = kb + 1 <= q0;  // tile 0 needs blocks 0..q0
        const bool b_next = two && kb + 1 <= last;          // tile 1 needs blocks 0..q0+1
        if (a_on && !(ok = issue_pv(0, kb))) break;
        if (a_next && !(ok = issue_s(0, kb + 1))) break;
        if (two && !(ok = issue_pv(1, kb))) break;
        tc_commit(&v_empty[kb & 1]);  // every PV reading V of block kb is issued
        if (b_next && !(ok = issue_s(1, kb + 1))) break;
        if (a_next || b_next) tc_commit(&k_empty[(kb + 1) & 1]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, a.err, kErrTimeoutDrain, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax + output
    const int u = warp >> 2;                 // query tile of this warp group
    const int qb = q0 + u;
    const int r = (warp & 3) * 32 + lane;    // query row within the tile = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_col = u ? L::TMEM_S1 : L::TMEM_S0;
    const uint32_t o_col = u ? L::TMEM_O1 : L::TMEM_O0;
    const int nkv = (u == 0 || two) ? qb + 1 : 0;  // no blocks for a missing second tile
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int kb = 0; kb < nkv; ++kb) {
      ok = mbar_wait(&s_full[u], kb & 1, a.err, kErrTimeoutAttn, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // The whole row of scores in registers (one TMEM read), the row maximum, then
      // P = 2^(S*scale*log2e - m) on pairs of scores, packed to bf16 and written over the
      // first 64 columns of the row's own scores.
      const bool diag = kb == qb;  // keys after this query are masked
      float sv[128];
      {
        uint32_t raw[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32_nw(lane_base + s_col + c * 32, raw[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          reg_fence(raw[c]);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(raw[c][i]);
        }
      }
      if (diag) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > r) sv[i] = -INFINITY;
      }
      // row max of the raw scores (the scale is positive): eight chains, then a tree
      float m8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) m8[k] = fmax3(sv[k], sv[8 + k], sv[16 + k]);
#pragma unroll
      for (int i = 24; i < 128; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = fmax3(m8[k], sv[i + k], sv[i + 8 + k]);
      const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                             fmaxf(m8[6], m8[7])) * scale_log2;
      const bool need = mx > m_run + kRescaleThreshold;
      const float alpha = need ? ex2_approx(m_run - mx) : 1.f;
      if (need) m_run = mx;
      // exponent arguments on pairs of scores (paired fp32 FMA), 2^x on the special-function
      // unit, row sums in four paired accumulators; P of keys 0-63 is handed to the MMA before
      // keys 64-127 are computed, so the first half of this block's PV overlaps the second
      const uint64_t c2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_run, -m_run);
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float pw[32];
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          float pa, pb;
          f2_unpack(f2_fma(f2_pack(sv[c * 64 + i], sv[c * 64 + i + 1]), c2, nm2), pa, pb);
          pa = ex2_approx(pa);
          pb = ex2_approx(pb);
          acc2[(i >> 1) & 3] = f2_add(acc2[(i >> 1) & 3], f2_pack(pa, pb));
          pw[i >> 1] = __uint_as_float(pack_bf16x2(pa, pb));
        }
        tmem_st_32x32b_x32(lane_base + s_col + c * 32, pw);  // includes the store wait
        // O holds the sum up to block kb-1 (its PV completed before this S was committed); it
        // is rescaled before this block's first PV, which waits for the first half of P
        if (c == 0 && kb > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int oc = 0; oc < D / 32; ++oc) {
            float o[32];
            const uint32_t ta = lane_base + o_col + oc * 32;
            tmem_ld_32x32b_x32(ta, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st_32x32b_x32(ta, o);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_half[2 * u + c]);
      }
      float rs[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) f2_unpack(acc2[k], rs[2 * k], rs[2 * k + 1]);
      l_run = l_run * alpha +
              (((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7])));
    }
    if (nkv > 0) {
      // drain is committed once, after the last MMA (a one-shot barrier: no phase aliasing)
      if (ok) ok = mbar_wait(drain, 0, a.err, kErrTimeoutAttn, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      // O / l in bf16 into this tile's Q buffer (every MMA has completed, so Q is no longer
      // read), laid out as the 128-byte-swizzled boxes the tensor map describes: 16-byte piece
      // j of row r's 64-column chunk at r * 128 + (j ^ (r % 8)) * 16. A bulk tensor store per
      // chunk then writes whole rows; rows past the sequence end are clipped by the map.
      uint8_t* stage = smem + L::Q_OFF + u * L::TILE;
      const int qrow = qb * 128 + r;
      if (ok) {
        tc_fence_after();
        const float inv = 1.f / l_run;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld_32x32b_x32(lane_base + o_col + c * 32, o);
          uint8_t* rowp = stage + (c >> 1) * 16384 + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16x2(o[q * 8 + 0] * inv, o[q * 8 + 1] * inv);
            w.y = pack_bf16x2(o[q * 8 + 2] * inv, o[q * 8 + 3] * inv);
            w.z = pack_bf16x2(o[q * 8 + 4] * inv, o[q * 8 + 5] * inv);
            w.w = pack_bf16x2(o[q * 8 + 6] * inv, o[q * 8 + 7] * inv);
            const int j = (c & 1) * 4 + q;
            *reinterpret_cast<uint4*>(rowp + ((j ^ (r & 7)) << 4)) = w;
          }
        }
        fence_proxy_async_smem();
        if (qrow < S) a.lse[((long long)b * H + n) * S + qrow] = (m_run + log2f(l_run)) * kLn2F;
      }
      // the tile's four warps always meet here (also after an error), then one thread stores
      asm volatile("bar.sync %0, 128;" ::"r"(1 + u) : "memory");
      if ((warp & 3) == 0 && lane == 0 && ok && !*abort_flag) {
#pragma unroll
        for (int c = 0; c < L::CH; ++c)
          tma_store_3d(&tm_o, stage + c * 16384, n * D + c * 64, qb * 128, b);
        bulk_commit();
        bulk_wait0();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================================ backward
// Head dimension 128 (bf16) runs the single key-stationary kernel further below
// (attn_bwd_fused_tc_kernel: S and dP once per tile pair, dQ accumulated in 32-bit fixed point
// through bulk tensor reduce-adds) between a pre-pass and a conversion. Head dimension 64 uses
// two kernels, both on tcgen05 with the probabilities recomputed from the saved log-sum-exp:
//   dK/dV kernel, one CTA per 128-key block (key-stationary), looping over query blocks in
//     64-query sub-blocks with double-buffered TMEM: S^T = K Q^T and dP^T = V dO^T; one
//     thread per key row forms P^T = exp2(S^T*scale*log2e - lse*log2e) and
//     dS^T = P^T * (dP^T - D) (D = rowsum(dO*O)) and writes both back into TMEM as packed
//     bf16; then dV += P^T dO and dK += dS^T Q run with the A operand read from TMEM and dO, Q
//     read N-major from their TMA tiles. The next sub-block's S^T, dP^T are computed while the
//     softmax warps work on this one.
//   dQ kernel, one CTA per 128-query block (query-stationary), looping over key blocks:
//     S = Q K^T, dP = dO V^T, dS = P * (dP - D) per query row, dQ += dS K.
// dQ therefore needs no atomics and is written once, in bf16, scaled by 1/sqrt(d); the cost is
// recomputing S and dP in the second kernel. TMEM: S 0-127, dP 128-255, accumulators above.
template <int D>
struct BwdLayout {
  static constexpr int CH = D / 64;
  static constexpr int TILE = 128 * D * 2;
  // dK/dV kernel: K, V resident; Q and dO double-buffered; per-query stats double-buffered.
  static constexpr int A_K = 0, A_V = TILE, A_Q = 2 * TILE, A_DO = 4 * TILE;
  static constexpr int A_STAT = 6 * TILE;  // float lse2[2][128], dsum[2][128]
  static constexpr int A_BAR = A_STAT + 4 * 128 * 4;
  static constexpr int A_BYTES = A_BAR + 256 + 1024;
  // dQ kernel: Q, dO resident; K and V double-buffered.
  static constexpr int B_Q = 0, B_DO = TILE, B_K = 2 * TILE, B_V = 4 * TILE;
  static constexpr int B_BAR = 6 * TILE;
  static constexpr int B_RED = B_BAR + 256;  // float [2 halves][128 rows]: partial rowsum(dO*O)
  static constexpr int B_BYTES = B_RED + 1024 + 1024;
  // dK/dV kernel: each 128-query block runs as two 64-query sub-blocks; sub-block g uses
  // buffer x = g & 1 with S^T in columns x*128 .. +63 and dP^T in x*128 + 64 .. +63; the dV
  // and dK accumulators follow.
  static constexpr int T_SUB = 128, T_ACC0 = 256, T_ACC1 = 256 + D;
  // dQ kernel: two S buffers so the next block's S overlaps this block's dS computation.
  static constexpr int Q_S0 = 0, Q_S1 = 128, Q_DP = 256, Q_DQ = 384;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                            const __grid_constant__ CUtensorMap tm_do, const AttnArgs a,
                            float scale_log2, float scale) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::A_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;   // [2]: Q and dO of one query block
  uint64_t* q_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;   // [2]: S^T, dP^T of a sub-block in buffer x
  uint64_t* p_full = bars + 7;   // [2]: P^T, dS^T of a sub-block written back
  uint64_t* drain = bars + 11;   // every MMA done (the output reads dV, dK after it)
  uint64_t* stat_bar = bars + 12;  // [2]: per-query stats of a block staged by the 8 warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* lse_s = reinterpret_cast<float*>(smem + L::A_STAT);  // [2][128], log2 units
  float* dsum_s = lse_s + 256;                                 // [2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.s, H = a.H, hp = H / a.p;
  // Key block; kb = 0 sees the most query blocks. Heads vary fastest in the launch order, so
  // the longest tiles of every head go first.
  const int kb = blockIdx.y;
  const int bh = blockIdx.x, b = bh / H, n = bh % H, t = n / hp, jh = n % hp;
  const int col_q = t * 3 * hp * D + jh * D, col_k = col_q + hp * D, col_v = col_q + 2 * hp * D;
  const int nq = (S + 127) / 128;
  const int niter = nq - kb;  // query blocks qi = kb .. nq-1 see keys of this block

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);
    }
    mbar_init(drain, 1);
    mbar_init(&stat_bar[0], 256);
    mbar_init(&stat_bar[1], 256);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
#pragma unroll
      for (int c = 0; c < L::CH; ++c) {
        tma_load_3d(&tm_qkv, kv_full, smem + L::A_K + c * 16384, col_k + c * 64, kb * 128, b);
        tma_load_3d(&tm_qkv, kv_full, smem + L::A_V + c * 16384, col_v + c * 64, kb * 128, b);
      }
      int issued = 0;
      for (int it = 0; it < niter; ++it) {
        const int st = it & 1, qi = kb + it;
        if (!mbar_wait(&q_empty[st], ((it >> 1) & 1) ^ 1, a.err, kErrTimeoutAttn, abort_flag))
          break;
        mbar_arrive_expect_tx(&q_full[st], 2 * L::TILE);
#pragma unroll
        for (int c = 0; c < L::CH; ++c) {
          tma_load_3d(&tm_qkv, &q_full[st], smem + L::A_Q + st * L::TILE + c * 16384,
                      col_q + c * 64, qi * 128, b);
          tma_load_3d(&tm_do, &q_full[st], smem + L::A_DO + st * L::TILE + c * 16384,
                      n * D + c * 64, qi * 128, b);
        }
        issued = it + 1;
      }
      mbar_wait(kv_full, 0, a.err, kErrTimeoutDrain, nullptr);
      for (int it = issued - 2 < 0 ? 0 : issued - 2; it < issued; ++it)
        mbar_wait(&q_full[it & 1], (it >> 1) & 1, a.err, kErrTimeoutDrain, nullptr);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // Sub-block g (query block it = g/2, half j = g%2) in TMEM buffer x = g%2:
      //   S^T = K Q_j^T and dP^T = V dO_j^T (M=128 keys, N=64 queries), then, once the
      //   softmax warps have written P^T and dS^T back, dV += P^T dO_j and dK += dS^T Q_j
      //   (K=64 queries, A from TMEM). S^T, dP^T of g+1 are issued before waiting for the
      //   softmax of g, so the tensor pipe and the softmax warps overlap.
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);
      const uint32_t k_addr = smem_u32(smem + L::A_K), v_addr = smem_u32(smem + L::A_V);
      const int G = 2 * niter;
      auto issue_sd = [&](int g) -> bool {
        const int it = g >> 1, j = g & 1, st = it & 1;
        const uint32_t x = (g & 1) * L::T_SUB;
        if (j == 0 && !mbar_wait(&q_full[st], (it >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::A_Q + st * L::TILE) + j * 8192;
        const uint32_t do_addr = smem_u32(smem + L::A_DO + st * L::TILE) + j * 8192;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc_mma_f16(tmem + x, smem_desc_sw128(k_addr + off, 16, 1024),
                     smem_desc_sw128(q_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc_mma_f16(tmem + x + 64, smem_desc_sw128(v_addr + off, 16, 1024),
                     smem_desc_sw128(do_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[g & 1]);
        return true;
      };
      bool ok = mbar_wait(kv_full, 0, a.err, kErrTimeoutAttn, abort_flag);
      if (ok && G > 0) ok = issue_sd(0);
      for (int g = 0; g < G && ok; ++g) {
        // Buffer (g+1)&1 was last read (P^T, dS^T as A operands) by the dV/dK MMAs of g-1,
        // issued earlier by this thread: MMAs of one thread execute in issue order, so those
        // reads precede the S^T, dP^T writes of g+1 and no wait is needed. (The softmax
        // warps' own reads of that buffer finished before they signalled p_full of g-1.)
        if (g + 1 < G && !issue_sd(g + 1)) break;
        if (!mbar_wait(&p_full[g & 1], (g >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag)) break;
        tc_fence_after();
        const int it = g >> 1, j = g & 1, st = it & 1;
        const uint32_t x = (g & 1) * L::T_SUB;
        const uint32_t q_addr = smem_u32(smem + L::A_Q + st * L::TILE) + j * 8192;
        const uint32_t do_addr = smem_u32(smem + L::A_DO + st * L::TILE) + j * 8192;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 64 queries, 16 per MMA
          const uint32_t acc = (g > 0 || kk > 0) ? 1u : 0u;
          // packed P^T / dS^T: queries 0-31 in columns 0-15, queries 32-63 in 32-47
          const uint32_t pc = kk * 8 + (kk >= 2 ? 16 : 0);
          tc_mma_f16_tmem_a(tmem + L::T_ACC0, tmem + x + pc,
                            smem_desc_sw128(do_addr + kk * 2048, 16384, 1024), idesc_acc, acc);
          tc_mma_f16_tmem_a(tmem + L::T_ACC1, tmem + x + 64 + pc,
                            smem_desc_sw128(q_addr + kk * 2048, 16384, 1024), idesc_acc, acc);
        }
        if (j == 1) tc_commit(&q_empty[st]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, a.err, kErrTimeoutDrain, nullptr);
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T and the output
    // warp w: TMEM lane quarter w%4 (key rows), 32-query half w/4 of each 64-query sub-block
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // key row within the block = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float* lse_g = a.lse + ((long long)b * H + n) * S;
    const float* dsum_g = a.Dsum + ((long long)b * H + n) * S;
    bool ok = true;
    // Per-query stats of the next block are fetched one block ahead (registers); warps of
    // half 0 stage lse, half 1 stage D, each for query r of the block.
    const float* stat_g = hf ? dsum_g : lse_g;
    float* stat_s = hf ? dsum_s : lse_s;
    auto fetch = [&](int qi) -> float {
      const int q = qi * 128 + r;  // padded queries get lse = +inf, hence P = 0
      if (hf == 0) return q < S ? stat_g[q] * kLog2eF : INFINITY;
      return q < S ? stat_g[q] : 0.f;
    };
    float nv = niter > 0 ? fetch(kb) : 0.f;
    for (int g = 0; g < 2 * niter; ++g) {
      const int it = g >> 1, j = g & 1, st = it & 1, qi = kb + it;
      if (j == 0) {
        stat_s[st * 128 + r] = nv;
        if (it + 1 < niter) nv = fetch(qi + 1);
        mbar_arrive(&stat_bar[st]);
        ok = mbar_wait(&stat_bar[st], (it >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
      }
      ok = mbar_wait(&s_full[g & 1], (g >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t x = (g & 1) * L::T_SUB;
      const int q0 = j * 64 + hf * 32;  // first query (within the block) of this warp's columns
      const float* ls = lse_s + st * 128 + q0;
      const float* ds_ = dsum_s + st * 128 + q0;
      uint32_t sr[32], dr[32];
      tmem_ld_32x32b_x32_nw(lane_base + x + hf * 32, sr);
      tmem_ld_32x32b_x32_nw(lane_base + x + 64 + hf * 32, dr);
      tmem_ld_wait();
      reg_fence(sr);
      reg_fence(dr);
      if (qi == kb) {  // diagonal block: queries before this key see nothing of it
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (q0 + i < r) sr[i] = __float_as_uint(-INFINITY);
      }
      uint32_t pw[16], dw[16];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(ls + i);
        const float4 d4 = *reinterpret_cast<const float4*>(ds_ + i);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
        float p4[4], q4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          p4[e] = ex2_approx(fmaf(__uint_as_float(sr[i + e]), scale_log2, -lv[e]));
          q4[e] = p4[e] * (__uint_as_float(dr[i + e]) - dv[e]);
        }
        pw[i >> 1] = pack_bf16x2(p4[0], p4[1]);
        pw[(i >> 1) + 1] = pack_bf16x2(p4[2], p4[3]);
        dw[i >> 1] = pack_bf16x2(q4[0], q4[1]);
        dw[(i >> 1) + 1] = pack_bf16x2(q4[2], q4[3]);
      }
      // Packed into the first half of the 32 columns this warp itself read, so the other
      // warp of the quarter (reading its own 32 columns) is never overwritten.
      tmem_st_32x32b_x16(lane_base + x + hf * 32, pw);
      tmem_st_32x32b_x16(lane_base + x + 64 + hf * 32, dw);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[g & 1]);
    }
    if (ok && niter > 0) {
      // drain is committed once, after the last MMA (a one-shot barrier: no phase aliasing)
      ok = mbar_wait(drain, 0, a.err, kErrTimeoutAttn, abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const int key = kb * 128 + r;
        const long long ld = 3LL * H * D;
        __nv_bfloat16* dk = reinterpret_cast<__nv_bfloat16*>(a.dqkv) + ((long long)b * S + key) * ld +
                            (long long)t * 3 * hp * D + (long long)jh * D + (long long)hp * D;
        __nv_bfloat16* dv = dk + (long long)hp * D;
#pragma unroll 1
        for (int c = hf * (D / 64); c < (hf + 1) * (D / 64); ++c) {  // this half of d
          float v[32], kk[32];
          tmem_ld_32x32b_x32(lane_base + L::T_ACC0 + c * 32, v);
          tmem_ld_32x32b_x32(lane_base + L::T_ACC1 + c * 32, kk);
          if (key < S) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 wv, wk;
              wv.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
              wv.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
              wv.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
              wv.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
              wk.x = pack_bf16x2(kk[q * 8 + 0] * scale, kk[q * 8 + 1] * scale);
              wk.y = pack_bf16x2(kk[q * 8 + 2] * scale, kk[q * 8 + 3] * scale);
              wk.z = pack_bf16x2(kk[q * 8 + 4] * scale, kk[q * 8 + 5] * scale);
              wk.w = pack_bf16x2(kk[q * 8 + 6] * scale, kk[q * 8 + 7] * scale);
              *reinterpret_cast<uint4*>(dv + c * 32 + q * 8) = wv;
              *reinterpret_cast<uint4*>(dk + c * 32 + q * 8) = wk;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                          const __grid_constant__ CUtensorMap tm_do, const AttnArgs a,
                          float scale_log2, float scale) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::B_BAR);
  uint64_t* q_full = bars + 0;    // Q and dO of this query block
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* drain = bars + 8;
  uint64_t* dsum_bar = bars + 9;  // [4 quarters]: the two halves of D = rowsum(dO*O)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.s, H = a.H, hp = H / a.p;
  const int nqb = (S + 127) / 128;
  const int qb = nqb - 1 - blockIdx.y;  // longest rows first, heads fastest (as above)
  const int bh = blockIdx.x, b = bh / H, n = bh % H, t = n / hp, jh = n % hp;
  const int col_q = t * 3 * hp * D + jh * D, col_k = col_q + hp * D, col_v = col_q + 2 * hp * D;
  const int nkv = qb + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);
    mbar_init(drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&dsum_bar[i], 64);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * L::TILE);
#pragma unroll
      for (int c = 0; c < L::CH; ++c) {
        tma_load_3d(&tm_qkv, q_full, smem + L::B_Q + c * 16384, col_q + c * 64, qb * 128, b);
        tma_load_3d(&tm_do, q_full, smem + L::B_DO + c * 16384, n * D + c * 64, qb * 128, b);
      }
      int issued = 0;
      for (int kb = 0; kb < nkv; ++kb) {
        const int st = kb & 1;
        if (!mbar_wait(&kv_empty[st], ((kb >> 1) & 1) ^ 1, a.err, kErrTimeoutAttn, abort_flag))
          break;
        mbar_arrive_expect_tx(&kv_full[st], 2 * L::TILE);
#pragma unroll
        for (int c = 0; c < L::CH; ++c) {
          tma_load_3d(&tm_qkv, &kv_full[st], smem + L::B_K + st * L::TILE + c * 16384,
                      col_k + c * 64, kb * 128, b);
          tma_load_3d(&tm_qkv, &kv_full[st], smem + L::B_V + st * L::TILE + c * 16384,
                      col_v + c * 64, kb * 128, b);
        }
        issued = kb + 1;
      }
      mbar_wait(q_full, 0, a.err, kErrTimeoutDrain, nullptr);
      for (int kb = issued - 2 < 0 ? 0 : issued - 2; kb < issued; ++kb)
        mbar_wait(&kv_full[kb & 1], (kb >> 1) & 1, a.err, kErrTimeoutDrain, nullptr);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(smem + L::B_Q), do_addr = smem_u32(smem + L::B_DO);
      // S_kb -> S buffer kb&1; dP_kb -> the single dP buffer; dQ += dS_kb K_kb with dS_kb in
      // S buffer kb&1. S_{kb+1} is issued before waiting for this block's dS, so it overlaps
      // the softmax warps; dP_{kb+1} waits until they have read dP_kb.
      auto issue_s = [&](int kb) {
        const uint32_t k_addr = smem_u32(smem + L::B_K + (kb & 1) * L::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc_mma_f16(tmem + ((kb & 1) ? L::Q_S1 : L::Q_S0),
                     smem_desc_sw128(q_addr + off, 16, 1024),
                     smem_desc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_dp = [&](int kb) {
        const uint32_t v_addr = smem_u32(smem + L::B_V + (kb & 1) * L::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc_mma_f16(tmem + L::Q_DP, smem_desc_sw128(do_addr + off, 16, 1024),
                     smem_desc_sw128(v_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, a.err, kErrTimeoutAttn, abort_flag) &&
                mbar_wait(&kv_full[0], 0, a.err, kErrTimeoutAttn, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        tc_commit(s_full);
      }
      for (int kb = 0; kb < nkv && ok; ++kb) {
        const bool more = kb + 1 < nkv;
        if (more) {
          // S buffer (kb+1)&1 was last read (as dS) by the dQ MMAs of block kb-1, issued
          // earlier by this thread: MMAs execute in issue order, so no wait is needed.
          if (!mbar_wait(&kv_full[(kb + 1) & 1], ((kb + 1) >> 1) & 1, a.err, kErrTimeoutAttn,
                         abort_flag))
            break;
          tc_fence_after();
          issue_s(kb + 1);
        }
        if (!mbar_wait(p_full, kb & 1, a.err, kErrTimeoutAttn, abort_flag)) break;
        tc_fence_after();
        // The softmax warps are done with dP_kb: dP_{kb+1} goes first, so they can start on
        // the next block while the tensor pipe still works on dQ += dS_kb K_kb.
        if (more) {
          issue_dp(kb + 1);
          tc_commit(s_full);
        }
        const uint32_t k_addr = smem_u32(smem + L::B_K + (kb & 1) * L::TILE);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // 128 keys, 16 per MMA; dS sits in S buffer kb&1
          tc_mma_f16_tmem_a(tmem + L::Q_DQ,
                            tmem + ((kb & 1) ? L::Q_S1 : L::Q_S0) + kk * 8 + (kk >= 4 ? 32 : 0),
                            smem_desc_sw128(k_addr + kk * 2048, 16384, 1024), idesc_acc,
                            (kb > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&kv_empty[kb & 1]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, a.err, kErrTimeoutDrain, nullptr);
    }
  } else {
    // warp w: TMEM lane quarter w%4 (query rows), key-column half w/4 (64 keys)
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // query row within the block = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int q = qb * 128 + r;
    const float lse2 = q < S ? a.lse[((long long)b * H + n) * S + q] * kLog2eF : INFINITY;
    // D = rowsum(dO * O) of this query row, each warp of the quarter pair summing half of d
    // while the first tiles load; the dK/dV kernel, launched next, reads it from a.Dsum.
    float dpart = 0.f;
    if (q < S) {
      const long long off = ((long long)b * S + q) * H * D + (long long)n * D + hf * (D / 2);
      const __nv_bfloat16* orow = reinterpret_cast<const __nv_bfloat16*>(a.o) + off;
      const __nv_bfloat16* drow = reinterpret_cast<const __nv_bfloat16*>(a.dO) + off;
#pragma unroll
      for (int i = 0; i < D / 2; i += 8) {
        const uint4 ov = *reinterpret_cast<const uint4*>(orow + i);
        const uint4 dv = *reinterpret_cast<const uint4*>(drow + i);
        const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, dw4[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dpart += bf16_lo(ow[e]) * bf16_lo(dw4[e]) + bf16_hi(ow[e]) * bf16_hi(dw4[e]);
      }
    }
    float* dred = reinterpret_cast<float*>(smem + L::B_RED);  // [2][128]
    dred[hf * 128 + r] = dpart;
    mbar_arrive(&dsum_bar[quarter]);
    bool ok = mbar_wait(&dsum_bar[quarter], 0, a.err, kErrTimeoutAttn, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    const float dq_sum = ok ? dpart + dred[(hf ^ 1) * 128 + r] : 0.f;
    if (ok && hf == 0 && q < S) a.Dsum[((long long)b * H + n) * S + q] = dq_sum;
    for (int kb = 0; kb < nkv && ok; ++kb) {
      ok = mbar_wait(s_full, kb & 1, a.err, kErrTimeoutAttn, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_col = (kb & 1) ? L::Q_S1 : L::Q_S0;
      {
        const int c2 = hf * 2;  // this half's two 32-column chunks of S and dP
        uint32_t sr[2][32], dr[2][32];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          tmem_ld_32x32b_x32_nw(lane_base + s_col + (c2 + u) * 32, sr[u]);
          tmem_ld_32x32b_x32_nw(lane_base + L::Q_DP + (c2 + u) * 32, dr[u]);
        }
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          reg_fence(sr[u]);
          reg_fence(dr[u]);
          const int c = c2 + u;
          uint32_t dw[16];
          if (kb == qb) {  // diagonal block: keys after this query are masked
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i > r) sr[u][i] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float d2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float p = ex2_approx(fmaf(__uint_as_float(sr[u][i + e]), scale_log2, -lse2));
              d2[e] = p * (__uint_as_float(dr[u][i + e]) - dq_sum);
            }
            dw[i >> 1] = pack_bf16x2(d2[0], d2[1]);
          }
          // packed into the first half of this warp's own 64 columns (see the dK/dV kernel)
          tmem_st_32x32b_x16(lane_base + s_col + hf * 64 + u * 16, dw);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) {
      // drain is committed once, after the last MMA (a one-shot barrier: no phase aliasing)
      ok = mbar_wait(drain, 0, a.err, kErrTimeoutAttn, abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const long long ld = 3LL * H * D;
        __nv_bfloat16* dq = reinterpret_cast<__nv_bfloat16*>(a.dqkv) + ((long long)b * S + q) * ld +
                            (long long)t * 3 * hp * D + (long long)jh * D;
#pragma unroll 1
        for (int c = hf * (D / 64); c < (hf + 1) * (D / 64); ++c) {  // this half of d
          float v[32];
          tmem_ld_32x32b_x32(lane_base + L::Q_DQ + c * 32, v);
          if (q < S) {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              uint4 w;
              w.x = pack_bf16x2(v[qq * 8 + 0] * scale, v[qq * 8 + 1] * scale);
              w.y = pack_bf16x2(v[qq * 8 + 2] * scale, v[qq * 8 + 3] * scale);
              w.z = pack_bf16x2(v[qq * 8 + 4] * scale, v[qq * 8 + 5] * scale);
              w.w = pack_bf16x2(v[qq * 8 + 6] * scale, v[qq * 8 + 7] * scale);
              *reinterpret_cast<uint4*>(dq + c * 32 + qq * 8) = w;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================================ fused backward
// One key-stationary kernel for head_dim 128 that computes S^T and dP^T once per (key block,
// query sub-block) and produces all three gradients:
//   S^T = K Q^T, dP^T = V dO^T           (M = 128 keys, N = 64 queries, fp32 in TMEM)
//   P^T = exp2(S^T*scale*log2e - lse*log2e), dS^T = P^T * (dP^T - D)   (softmax warps)
//   dQ^T = K^T dS^T                       (M = d, N = 64 queries) into the dP^T columns
//   dK += dS^T Q, dV += P^T dO            (TMEM accumulators)
// P^T goes back into TMEM as packed bf16 (the A operand of dV). dS^T goes to shared memory
// in the 128-byte swizzled layout, where one buffer serves as the K-major A operand of dK
// (rows = keys) and as the MN-major B operand of dQ^T (queries contiguous). Four drain warps
// read each dQ^T tile from TMEM, convert it to fixed point and stage it 16 queries at a time
// as [query][d] boxes that bulk tensor reduce-adds add into the accumulator a.dq_fix [T][H][d].
// Five products per (key block, query block) instead of the seven of the two-kernel form.
// After the last sub-block dK and dV leave through bulk tensor stores staged in the K and V
// tile buffers. The kernel is bound by shared-memory bandwidth: the N = 64 products read a
// 4 KB A tile and a 2 KB B tile per 32 cycles of math.
//
// The accumulator is 32-bit fixed point, so the result is bit-reproducible: integer addition
// is associative, and the key blocks of a query block arrive in no fixed order. Every partial
// sum of dQ is bounded: |dQ[q,d]| <= max|K| * sum_k |dS[q,k]| and
// sum_k |dS[q,k]| <= sum_k P[q,k] (|dP[q,k]| + |D[q]|) <= 2 |dO_q| max_k |V_k|
// (Cauchy-Schwarz for dP = dO.V; |D| = |dO.O| with O a convex combination of the V rows; the
// probabilities of a row sum to 1). With B = 2 max|K| max|dO_q| max|V_k| over the head, values
// are scaled by 2^e with B * 2^e < 2^29 and rounded to integers: four times headroom below the
// int32 limit for rounding, and a resolution of B * 2^-29 per addend.
//
// Warps 0-7: softmax (lane quarter w%4 = 32 key rows, query half w/4 of each sub-block);
// warp 8: TMA producer; warp 9: TMEM owner and MMA issuer; warps 10-13: dQ drain (lane
// quarter w%4 = 32 of the d rows of dQ^T). Every wait is bounded.
// Power of two e with B * 2^e < 2^29 for B = 2 max|K| max|dO row| max|V row| over a head's
// 32-token chunk bounds ([nchunk][3]: max |K|, max |V row|^2, max |dO row|^2). Every CTA of a head and
// nothing else computes it, from the same values, so all agree.
__device__ __forceinline__ int dq_fixed_exponent(const float* bound, int nchunk) {
  float km = 0.f, v2 = 0.f, g2 = 0.f;
  for (int c = 0; c < nchunk; ++c) {
    km = fmaxf(km, bound[3 * c]);
    v2 = fmaxf(v2, bound[3 * c + 1]);
    g2 = fmaxf(g2, bound[3 * c + 2]);
  }
  const float B = 2.f * km * sqrtf(v2) * sqrtf(g2);
  if (!(B > 0.f)) return 100;        // all-zero gradients: any scale is exact
  if (!(B < INFINITY)) return -100;  // non-finite inputs: the result is undefined anyway
  int ex;
  frexpf(B, &ex);                    // B < 2^ex
  const int e = 29 - ex;
  return e > 100 ? 100 : (e < -100 ? -100 : e);
}

template <int D>
struct FusedBwdLayout {
  static constexpr int CH = D / 64;
  static constexpr int TILE = 128 * D * 2;
  static constexpr int K_OFF = 0, V_OFF = TILE, Q_OFF = 2 * TILE, DO_OFF = 4 * TILE;  // Q, dO x2
  static constexpr int DS_OFF = 6 * TILE;           // dS^T [128 keys][64 queries] bf16
  static constexpr int STG_OFF = DS_OFF + 16384;    // dQ staging: 4 warps x [16 q][32 d] int32
  static constexpr int STAT_OFF = STG_OFF + 8192;   // [2 stages][-lse*log2e | -D][128 queries]
  static constexpr int BAR_OFF = STAT_OFF + 2048;
  static constexpr int BYTES = BAR_OFF + 256 + 1024;
  // TMEM buffer x (sub-block parity) at x*128: S^T in +0..63 (P^T packed into its first
  // halves), dP^T in +64..127 (then dQ^T); dV and dK accumulators above.
  static constexpr int T_SUB = 128, T_DV = 256, T_DK = 256 + D;
};
constexpr int kFusedBwdThreads = 448;

template <int D>
__global__ void __launch_bounds__(kFusedBwdThreads, 1)
    attn_bwd_fused_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                             const __grid_constant__ CUtensorMap tm_do,
                             const __grid_constant__ CUtensorMap tm_dq,
                             const __grid_constant__ CUtensorMap tm_dqkv, const AttnArgs a,
                             float scale_log2, float scale) {
  using L = FusedBwdLayout<D>;
  static_assert(D == 128, "dQ^T tiles use M = head_dim = 128");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;     // [2]: Q and dO of one query block
  uint64_t* q_empty = bars + 3;    // [2]
  uint64_t* s_full = bars + 5;     // [2]: S^T, dP^T of a sub-block in buffer x
  uint64_t* p_full = bars + 7;     // [2]: P^T in TMEM and dS^T in shared memory
  uint64_t* ds_empty = bars + 9;   // dK and dQ^T of the previous sub-block have read dS^T
  uint64_t* dq_full = bars + 10;   // [2]: dQ^T of a sub-block is in buffer x
  uint64_t* dq_empty = bars + 12;  // [2]: the drain warps have read it
  uint64_t* drain = bars + 14;     // every MMA done (the output reads dV, dK after it)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* ds_buf = smem + L::DS_OFF;
  float* stat_s = reinterpret_cast<float*>(smem + L::STAT_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.s, H = a.H, hp = H / a.p;
  // Key block; kb = 0 sees the most query blocks. Heads vary fastest in the launch order, so
  // the longest tiles of every head go first.
  const int kb = blockIdx.y;
  const int bh = blockIdx.x, b = bh / H, n = bh % H, t = n / hp, jh = n % hp;
  const int col_q = t * 3 * hp * D + jh * D, col_k = col_q + hp * D, col_v = col_q + 2 * hp * D;
  const int nq = (S + 127) / 128;
  const int niter = nq - kb;  // query blocks qi = kb .. nq-1 see keys of this block
  const int G = 2 * niter;    // 64-query sub-blocks

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);
      mbar_init(&dq_full[i], 1);
      mbar_init(&dq_empty[i], 4);
    }
    mbar_init(ds_empty, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
    tma_prefetch_desc(&tm_dqkv);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();  // the pre-pass's statistics and zeroed accumulator

  if (warp == 8) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
#pragma unroll
      for (int c = 0; c < L::CH; ++c) {
        tma_load_3d(&tm_qkv, kv_full, smem + L::K_OFF + c * 16384, col_k + c * 64, kb * 128, b);
        tma_load_3d(&tm_qkv, kv_full, smem + L::V_OFF + c * 16384, col_v + c * 64, kb * 128, b);
      }
      int issued = 0;
      for (int it = 0; it < niter; ++it) {
        const int st = it & 1, qi = kb + it;
        if (!mbar_wait(&q_empty[st], ((it >> 1) & 1) ^ 1, a.err, kErrTimeoutAttn, abort_flag))
          break;
        mbar_arrive_expect_tx(&q_full[st], 2 * L::TILE + 1024);
#pragma unroll
        for (int c = 0; c < L::CH; ++c) {
          tma_load_3d(&tm_qkv, &q_full[st], smem + L::Q_OFF + st * L::TILE + c * 16384,
                      col_q + c * 64, qi * 128, b);
          tma_load_3d(&tm_do, &q_full[st], smem + L::DO_OFF + st * L::TILE + c * 16384,
                      n * D + c * 64, qi * 128, b);
        }
        // the block's -lse*log2(e) and -D rows (padded past the sequence by the pre-pass)
        const float* srow = a.dq_stat + (long long)bh * 2 * (nq * 128) + qi * 128;
        bulk_load_1d(stat_s + st * 256, srow, 512, &q_full[st]);
        bulk_load_1d(stat_s + st * 256 + 128, srow + nq * 128, 512, &q_full[st]);
        issued = it + 1;
      }
      mbar_wait(kv_full, 0, a.err, kErrTimeoutDrain, nullptr);
      for (int it = issued - 2 < 0 ? 0 : issued - 2; it < issued; ++it)
        mbar_wait(&q_full[it & 1], (it >> 1) & 1, a.err, kErrTimeoutDrain, nullptr);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // Per sub-block g (query block it = g/2, half j = g%2, TMEM buffer x = g%2):
      //   S^T(g+1), dP^T(g+1) are issued before waiting for the softmax of g, so the tensor
      //   pipe computes them (and then dQ^T, dK, dV of g) while the softmax warps work.
      //   dP^T(g+1) overwrites dQ^T(g-1) in the same buffer: it waits until the drain warps
      //   have read that tile. S^T(g+1) overwrites P^T(g-1), read by dV(g-1) which was issued
      //   earlier by this thread (tcgen05.mma operations of one thread execute in order).
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, 64, true, true);
      const uint32_t k_addr = smem_u32(smem + L::K_OFF), v_addr = smem_u32(smem + L::V_OFF);
      const uint32_t ds_addr = smem_u32(ds_buf);
      auto issue_sd = [&](int g) -> bool {
        const int it = g >> 1, j = g & 1, st = it & 1;
        const uint32_t x = (g & 1) * L::T_SUB;
        if (j == 0 && !mbar_wait(&q_full[st], (it >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::Q_OFF + st * L::TILE) + j * 8192;
        const uint32_t do_addr = smem_u32(smem + L::DO_OFF + st * L::TILE) + j * 8192;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc_mma_f16(tmem + x, smem_desc_sw128(k_addr + off, 16, 1024),
                     smem_desc_sw128(q_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        if (g >= 2 && !mbar_wait(&dq_empty[g & 1], ((g - 2) >> 1) & 1, a.err, kErrTimeoutAttn,
                                 abort_flag))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc_mma_f16(tmem + x + 64, smem_desc_sw128(v_addr + off, 16, 1024),
                     smem_desc_sw128(do_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[g & 1]);
        return true;
      };
      bool ok = mbar_wait(kv_full, 0, a.err, kErrTimeoutAttn, abort_flag);
      if (ok && G > 0) ok = issue_sd(0);
      for (int g = 0; g < G && ok; ++g) {
        if (g + 1 < G && !(ok = issue_sd(g + 1))) break;
        if (!(ok = mbar_wait(&p_full[g & 1], (g >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag)))
          break;
        tc_fence_after();
        const int it = g >> 1, j = g & 1, st = it & 1;
        const uint32_t x = (g & 1) * L::T_SUB;
        const uint32_t q_addr = smem_u32(smem + L::Q_OFF + st * L::TILE) + j * 8192;
        const uint32_t do_addr = smem_u32(smem + L::DO_OFF + st * L::TILE) + j * 8192;
        // dQ^T(g) = K^T dS^T (128 keys, 16 per MMA): A = K read d-major from its tile, B = dS^T
        // read query-major; the result replaces dP^T(g), which the softmax has consumed.
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_f16(tmem + x + 64, smem_desc_sw128(k_addr + kk * 2048, 16384, 1024),
                     smem_desc_sw128(ds_addr + kk * 2048, 16384, 1024), idesc_dq,
                     kk > 0 ? 1u : 0u);
        tc_commit(&dq_full[g & 1]);
        // dK += dS^T Q (64 queries, 16 per MMA): A = dS^T read key-major from shared memory
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_f16(tmem + L::T_DK, smem_desc_sw128(ds_addr + kk * 32, 16, 1024),
                     smem_desc_sw128(q_addr + kk * 2048, 16384, 1024), idesc_acc,
                     (g > 0 || kk > 0) ? 1u : 0u);
        tc_commit(ds_empty);
        // dV += P^T dO: packed P^T, queries 0-31 in columns 0-15, 32-63 in 32-47
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t pc = kk * 8 + (kk >= 2 ? 16 : 0);
          tc_mma_f16_tmem_a(tmem + L::T_DV, tmem + x + pc,
                            smem_desc_sw128(do_addr + kk * 2048, 16384, 1024), idesc_acc,
                            (g > 0 || kk > 0) ? 1u : 0u);
        }
        if (j == 1) tc_commit(&q_empty[st]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, a.err, kErrTimeoutDrain, nullptr);
    }
  } else if (warp >= 10) {
    // ------------------------------------------------------------ dQ drain
    // Thread = row dd of dQ^T (one of the head dimensions); the 64 columns are the queries of
    // the sub-block. Each warp converts its 32 rows to fixed point, stages them 16 queries at
    // a time as a [query][d] box in shared memory and hands the box to one bulk tensor
    // reduce-add (integer add in L2), so the additions cost the warp no per-element
    // instructions.
    const int quarter = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int32_t* stg = reinterpret_cast<int32_t*>(smem + L::STG_OFF) + (warp - 10) * 512;
    // this head's fixed-point scale (the same computation in every CTA of the head)
    const int e = dq_fixed_exponent(a.dq_bound + (long long)bh * nq * 4 * 3, nq * 4);
    if (kb == 0 && quarter == 0 && lane == 0) a.dq_exp[bh] = e;
    const float fscale = exp2f((float)e);
    bool issued = false;
    for (int g = 0; g < G; ++g) {
      const bool ok = mbar_wait(&dq_full[g & 1], (g >> 1) & 1, a.err, kErrTimeoutAttn,
                                abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t x = (g & 1) * L::T_SUB;
      uint32_t v[2][32];
      tmem_ld_32x32b_x32_nw(lane_base + x + 64, v[0]);
      tmem_ld_32x32b_x32_nw(lane_base + x + 96, v[1]);
      tmem_ld_wait();
      reg_fence(v[0]);
      reg_fence(v[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dq_empty[g & 1]);
      const int q0 = (kb + (g >> 1)) * 128 + (g & 1) * 64;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {  // four boxes of 16 queries
        if (q0 + hh * 16 >= S) break;  // rows past the sequence are clipped; none left here
        if (lane == 0 && issued) bulk_wait_read0();  // the previous box has been read
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          stg[i * 32 + lane] = __float2int_rn(__uint_as_float(v[hh >> 1][(hh & 1) * 16 + i]) * fscale);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tm_dq, stg, n * D + quarter * 32, q0 + hh * 16, b);
          bulk_commit();
        }
        issued = true;
      }
    }
    if (lane == 0 && issued) bulk_wait0();  // every reduction has landed in global memory
  } else {
    // ------------------------------------------------------------ P^T, dS^T and the output
    // warp w: TMEM lane quarter w%4 (key rows), 32-query half w/4 of each 64-query sub-block
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // key row within the block = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    // per-query -lse*log2(e) and -D of the current query block (padded past the sequence
    // with -inf and 0, so P = 0 there), brought into shared memory with Q and dO
    // this thread's dS^T row in the swizzled buffer: 16-byte chunk c of the row sits at
    // chunk c ^ (r % 8)
    uint8_t* ds_row = ds_buf + r * 128;
    bool ok = true;
    for (int g = 0; g < G; ++g) {
      const int it = g >> 1, j = g & 1, st = it & 1, qi = kb + it;
      ok = mbar_wait(&s_full[g & 1], (g >> 1) & 1, a.err, kErrTimeoutAttn, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t x = (g & 1) * L::T_SUB;
      const int q0 = j * 64 + hf * 32;  // first query (within the block) of this warp's columns
      const float* ls = stat_s + st * 256 + q0;
      const float* ds_ = stat_s + st * 256 + 128 + q0;
      uint32_t sr[32], dr[32];
      tmem_ld_32x32b_x32_nw(lane_base + x + hf * 32, sr);
      tmem_ld_32x32b_x32_nw(lane_base + x + 64 + hf * 32, dr);
      tmem_ld_wait();
      reg_fence(sr);
      reg_fence(dr);
      if (qi == kb) {  // diagonal block: queries before this key see nothing of it
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (q0 + i < r) sr[i] = __float_as_uint(-INFINITY);
      }
      // P^T = 2^(S^T*scale*log2e - lse*log2e), dS^T = P^T (dP^T - D) on pairs of queries
      // (paired fp32 ops; 2^x on the special-function unit)
      uint32_t pw[16], dw[16];
      const uint64_t c2 = f2_pack(scale_log2, scale_log2);
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(ls + i);   // -lse * log2e
        const float4 d4 = *reinterpret_cast<const float4*>(ds_ + i);  // -D
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          float pa, pb;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[i + e]), __uint_as_float(sr[i + e + 1])),
                           c2, e ? f2_pack(l4.z, l4.w) : f2_pack(l4.x, l4.y)),
                    pa, pb);
          pa = ex2_approx(pa);
          pb = ex2_approx(pb);
          const uint64_t dpd = f2_add(
              f2_pack(__uint_as_float(dr[i + e]), __uint_as_float(dr[i + e + 1])),
              e ? f2_pack(d4.z, d4.w) : f2_pack(d4.x, d4.y));
          float qa, qb;
          f2_unpack(f2_mul(f2_pack(pa, pb), dpd), qa, qb);
          pw[(i + e) >> 1] = pack_bf16x2(pa, pb);
          dw[(i + e) >> 1] = pack_bf16x2(qa, qb);
        }
      }
      // P^T packed into the first half of the 32 columns this warp itself read, so the other
      // warp of the quarter (reading its own 32 columns) is never overwritten.
      tmem_st_32x32b_x16(lane_base + x + hf * 32, pw);
      // dS^T into shared memory once dK and dQ^T of the previous sub-block have read it
      if (g > 0) {
        ok = mbar_wait(ds_empty, (g - 1) & 1, a.err, kErrTimeoutAttn, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int chunk = (hf * 4 + c) ^ (r & 7);
        *reinterpret_cast<uint4*>(ds_row + chunk * 16) =
            make_uint4(dw[4 * c], dw[4 * c + 1], dw[4 * c + 2], dw[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[g & 1]);
    }
    if (niter > 0) {
      // drain is committed once, after the last MMA (a one-shot barrier: no phase aliasing)
      if (ok) ok = mbar_wait(drain, 0, a.err, kErrTimeoutAttn, abort_flag);
      // the eight warps meet at both barriers below on every path, and decide together
      uint32_t all_ok;
      asm volatile(
          "{ .reg .pred pi, po; setp.ne.u32 pi, %1, 0; bar.red.and.pred po, 1, 256, pi; "
          "selp.u32 %0, 1, 0, po; }"
          : "=r"(all_ok)
          : "r"((uint32_t)__all_sync(0xffffffffu, ok))
          : "memory");
      // dK (scaled) and dV in bf16 into the K and V tile buffers (every MMA has completed, so
      // they are no longer read), as the 128-byte-swizzled boxes of the dqkv tensor map:
      // 16-byte piece j of row r's 64-column chunk at r * 128 + (j ^ (r % 8)) * 16; rows past
      // the sequence are clipped by the map.
      uint8_t* stage_k = smem + L::K_OFF;
      uint8_t* stage_v = smem + L::V_OFF;
      if (all_ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c = hf * (D / 64); c < (hf + 1) * (D / 64); ++c) {  // this half of d
          float v[32], kk[32];
          tmem_ld_32x32b_x32(lane_base + L::T_DV + c * 32, v);
          tmem_ld_32x32b_x32(lane_base + L::T_DK + c * 32, kk);
          const int off = (c >> 1) * 16384 + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 wv, wk;
            wv.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
            wv.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
            wv.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
            wv.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
            wk.x = pack_bf16x2(kk[q * 8 + 0] * scale, kk[q * 8 + 1] * scale);
            wk.y = pack_bf16x2(kk[q * 8 + 2] * scale, kk[q * 8 + 3] * scale);
            wk.z = pack_bf16x2(kk[q * 8 + 4] * scale, kk[q * 8 + 5] * scale);
            wk.w = pack_bf16x2(kk[q * 8 + 6] * scale, kk[q * 8 + 7] * scale);
            const int jj = ((c & 1) * 4 + q) ^ (r & 7);
            *reinterpret_cast<uint4*>(stage_v + off + jj * 16) = wv;
            *reinterpret_cast<uint4*>(stage_k + off + jj * 16) = wk;
          }
        }
        fence_proxy_async_smem();
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");  // every row of both tiles is staged
      if (warp == 0 && lane == 0 && all_ok && !*abort_flag) {
        const int col_dk = t * 3 * hp * D + hp * D + jh * D, col_dv = col_dk + hp * D;
#pragma unroll
        for (int c = 0; c < L::CH; ++c) {
          tma_store_3d(&tm_dqkv, stage_k + c * 16384, col_dk + c * 64, kb * 128, b);
          tma_store_3d(&tm_dqkv, stage_v + c * 16384, col_dv + c * 64, kb * 128, b);
        }
        bulk_commit();
        bulk_wait0();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Per head and 32-token chunk c (grid b*H x ceil(s/128)*4, 8 warps x 4 tokens): D = rowsum(dO * O)
// into a.Dsum [b][H][s], the fixed-point dQ accumulator zeroed, the per-query statistics rows
// (-lse*log2e, -D, padded to whole 128-query blocks with -inf and 0) and the chunk's max |K|,
// max |V row|^2 and max |dO row|^2 into a.dq_bound. A lane holds 4 of the 128 dimensions; each
// warp issues the loads of its 4 tokens before using any, so that enough bytes are in flight.
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const AttnArgs a) {
  grid_dependency_wait();
  constexpr int D = 128;
  __shared__ float red[8][3];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x, c = blockIdx.y, nchunk = gridDim.y;
  const int H = a.H, hp = H / a.p, b = bh / H, n = bh % H, t = n / hp, jh = n % hp;
  const long long ld_qkv = 3LL * H * D, ld_o = (long long)H * D;
  const long long nqp = (long long)nchunk * 32;
  float* stat = a.dq_stat + (long long)bh * 2 * nqp;
  const __nv_bfloat16* o_ = reinterpret_cast<const __nv_bfloat16*>(a.o);
  const __nv_bfloat16* g_ = reinterpret_cast<const __nv_bfloat16*>(a.dO);
  const __nv_bfloat16* qkv_ = reinterpret_cast<const __nv_bfloat16*>(a.qkv);
  uint2 ov[4], gv[4], kv[4], vv[4];
  // lane i < 4 fetches token i's lse with the rows, so no load waits inside the loop below
  const int lpos = c * 32 + warp * 4 + lane;
  const float lse_l = (lane < 4 && lpos < a.s) ? a.lse[(long long)bh * a.s + lpos] : 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int pos = c * 32 + warp * 4 + i;
    if (pos < a.s) {
      const long long tok = (long long)b * a.s + pos;
      const long long oo = tok * ld_o + (long long)n * D + lane * 4;
      const long long ko = tok * ld_qkv + (long long)t * 3 * hp * D + (long long)(hp + jh) * D +
                           lane * 4;
      ov[i] = *reinterpret_cast<const uint2*>(o_ + oo);
      gv[i] = *reinterpret_cast<const uint2*>(g_ + oo);
      kv[i] = *reinterpret_cast<const uint2*>(qkv_ + ko);
      vv[i] = *reinterpret_cast<const uint2*>(qkv_ + ko + (long long)hp * D);
    }
  }
  float kmax = 0.f, v2max = 0.f, g2max = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int pos = c * 32 + warp * 4 + i;
    const float lse_i = __shfl_sync(0xffffffffu, lse_l, i);
    if (pos >= a.s) {  // warp-uniform: padding of the softmax statistics (P = 0 there)
      if (lane == 0) {
        stat[pos] = -INFINITY;
        stat[nqp + pos] = 0.f;
      }
      continue;
    }
    const long long tok = (long long)b * a.s + pos;
    const float o[4] = {bf16_lo(ov[i].x), bf16_hi(ov[i].x), bf16_lo(ov[i].y), bf16_hi(ov[i].y)};
    const float g[4] = {bf16_lo(gv[i].x), bf16_hi(gv[i].x), bf16_lo(gv[i].y), bf16_hi(gv[i].y)};
    const float k[4] = {bf16_lo(kv[i].x), bf16_hi(kv[i].x), bf16_lo(kv[i].y), bf16_hi(kv[i].y)};
    const float v[4] = {bf16_lo(vv[i].x), bf16_hi(vv[i].x), bf16_lo(vv[i].y), bf16_hi(vv[i].y)};
    float dsum = 0.f, g2 = 0.f, v2 = 0.f, km = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dsum = fmaf(o[e], g[e], dsum);
      g2 = fmaf(g[e], g[e], g2);
      v2 = fmaf(v[e], v[e], v2);
      km = fmaxf(km, fabsf(k[e]));
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
      dsum += __shfl_xor_sync(0xffffffffu, dsum, m);
      g2 += __shfl_xor_sync(0xffffffffu, g2, m);
      v2 += __shfl_xor_sync(0xffffffffu, v2, m);
      km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, m));
    }
    if (lane == 0) {
      a.Dsum[(long long)bh * a.s + pos] = dsum;
      stat[pos] = -lse_i * kLog2eF;
      stat[nqp + pos] = -dsum;
    }
    *reinterpret_cast<int4*>(a.dq_fix + tok * ld_o + (long long)n * D + lane * 4) =
        make_int4(0, 0, 0, 0);
    kmax = fmaxf(kmax, km);
    v2max = fmaxf(v2max, v2);
    g2max = fmaxf(g2max, g2);
  }
  if (lane == 0) {
    red[warp][0] = kmax;
    red[warp][1] = v2max;
    red[warp][2] = g2max;
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    float m = 0.f;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w][threadIdx.x]);
    a.dq_bound[((long long)bh * nchunk + c) * 3 + threadIdx.x] = m;
  }
}

// dQ = dq_fix * 2^-e / sqrt(d) in bf16 into the Q slots of dqkv [T][p][3][H/p][d]: 16 threads
// per (token, head), 8 elements each.
__global__ void attn_bwd_dq_convert_kernel(const AttnArgs a, float scale) {
  grid_dependency_wait();
  const long long rows = (long long)a.b * a.s * a.H;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = idx >> 4;
  const int part = (int)(idx & 15);
  if (row >= rows) return;
  const long long token = row / a.H;
  const int nh = (int)(row - token * a.H), hp = a.H / a.p, tt = nh / hp, jj = nh - tt * hp;
  const int bb = (int)(token / a.s);
  const float f = scale * exp2f((float)-a.dq_exp[(long long)bb * a.H + nh]);
  const int4* src = reinterpret_cast<const int4*>(a.dq_fix + row * 128 + part * 8);
  const int4 u = src[0], v = src[1];
  uint4 w;
  w.x = pack_bf16x2((float)u.x * f, (float)u.y * f);
  w.y = pack_bf16x2((float)u.z * f, (float)u.w * f);
  w.z = pack_bf16x2((float)v.x * f, (float)v.y * f);
  w.w = pack_bf16x2((float)v.z * f, (float)v.w * f);
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.dqkv) + token * 3LL * a.H * 128 +
                       (long long)tt * 3 * hp * 128 + (long long)jj * 128 + part * 8;
  *reinterpret_cast<uint4*>(dst) = w;
}

cudaError_t bwd_fused_tc(const AttnArgs& a, cudaStream_t s) {
  constexpr int D = 128;
  using L = FusedBwdLayout<D>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_fused_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap tm_qkv, tm_do;
  const uint64_t three_h = 3ull * a.H * D, hd = (uint64_t)a.H * D;
  const uint32_t box[3] = {64, 128, 1};
  {
    const uint64_t dims[3] = {three_h, (uint64_t)a.s, (uint64_t)a.b};
    const uint64_t strides[2] = {three_h, three_h * a.s};
    if (!make_tensor_map_bf16_3d(&tm_qkv, a.qkv, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {hd, (uint64_t)a.s, (uint64_t)a.b};
    const uint64_t strides[2] = {hd, hd * a.s};
    if (!make_tensor_map_bf16_3d(&tm_do, a.dO, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const float scale = 1.f / sqrtf((float)D);
  const long long threads = (long long)a.b * a.s * a.H * 16;  // 16 per (token, head)
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  cudaError_t e = launch_kernel(true, attn_bwd_prep_kernel,
                                dim3(a.b * a.H, (a.s + 127) / 128 * 4), dim3(256), 0, s, a);
  if (e != cudaSuccess) return e;
  CUtensorMap tm_dq;  // the fixed-point dQ accumulator as [b][s][H*d] int32, 32 x 16 boxes
  {
    const uint64_t dims[3] = {hd, (uint64_t)a.s, (uint64_t)a.b};
    const uint64_t strides[2] = {hd, hd * a.s};
    const uint32_t qbox[3] = {32, 16, 1};
    if (!make_tensor_map_i32_3d(&tm_dq, a.dq_fix, dims, strides, qbox))
      return cudaErrorInvalidValue;
  }
  CUtensorMap tm_dqkv;  // dK and dV written into dqkv, viewed as qkv is
  {
    const uint64_t dims[3] = {three_h, (uint64_t)a.s, (uint64_t)a.b};
    const uint64_t strides[2] = {three_h, three_h * a.s};
    if (!make_tensor_map_bf16_3d(&tm_dqkv, a.dqkv, dims, strides, box))
      return cudaErrorInvalidValue;
  }
  dim3 grid(a.b * a.H, (a.s + 127) / 128);
  e = launch_kernel(true, attn_bwd_fused_tc_kernel<D>, grid, dim3(kFusedBwdThreads), L::BYTES,
                    s, tm_qkv, tm_do, tm_dq, tm_dqkv, a, kLog2eF * scale, scale);
  if (e != cudaSuccess) return e;
  return launch_kernel(true, attn_bwd_dq_convert_kernel, dim3(blocks), dim3(256), 0, s, a,
                       scale);
}

template <int D>
cudaError_t bwd_tc(const AttnArgs& a, cudaStream_t s) {
  using L = BwdLayout<D>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::A_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, L::B_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap tm_qkv, tm_do;
  const uint64_t three_h = 3ull * a.H * D, hd = (uint64_t)a.H * D;
  const uint32_t box[3] = {64, 128, 1};
  {
    const uint64_t dims[3] = {three_h, (uint64_t)a.s, (uint64_t)a.b};
    const uint64_t strides[2] = {three_h, three_h * a.s};
    if (!make_tensor_map_bf16_3d(&tm_qkv, a.qkv, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {hd, (uint64_t)a.s, (uint64_t)a.b};
    const uint64_t strides[2] = {hd, hd * a.s};
    if (!make_tensor_map_bf16_3d(&tm_do, a.dO, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const float scale = 1.f / sqrtf((float)D);
  dim3 grid(a.b * a.H, (a.s + 127) / 128);
  // The dQ kernel goes first: it also forms D = rowsum(dO * O), which the dK/dV kernel reads.
  attn_bwd_dq_tc_kernel<D><<<grid, kBwdThreads, L::B_BYTES, s>>>(tm_qkv, tm_do, a,
                                                                  kLog2eF * scale, scale);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_dkdv_tc_kernel<D><<<grid, kBwdThreads, L::A_BYTES, s>>>(tm_qkv, tm_do, a,
                                                                    kLog2eF * scale, scale);
  return cudaGetLastError();
}

template <int D>
cudaError_t fwd_tc(const AttnArgs& a, cudaStream_t s) {
  using L = FwdLayout<D>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  // qkv viewed as [b][s][3h]; rows past s read as zeros, so tiles never cross sequences.
  CUtensorMap tm;
  const uint64_t three_h = 3ull * a.H * D;
  const uint64_t dims[3] = {three_h, (uint64_t)a.s, (uint64_t)a.b};
  const uint64_t strides[2] = {three_h, three_h * a.s};
  const uint32_t box[3] = {64, 128, 1};
  if (!make_tensor_map_bf16_3d(&tm, a.qkv, dims, strides, box)) return cudaErrorInvalidValue;
  // o viewed as [b][s][H*D], written in the same 64-column, 128-row boxes
  CUtensorMap tm_o;
  const uint64_t hd = (uint64_t)a.H * D;
  const uint64_t dims_o[3] = {hd, (uint64_t)a.s, (uint64_t)a.b};
  const uint64_t strides_o[2] = {hd, hd * a.s};
  if (!make_tensor_map_bf16_3d(&tm_o, a.o, dims_o, strides_o, box)) return cudaErrorInvalidValue;
  // one CTA per pair of 128-query blocks of one head
  dim3 grid(a.b * a.H, ((a.s + 127) / 128 + 1) / 2);
  return launch_kernel(true, attn_fwd_tc_kernel<D>, grid, dim3(kAttnFwdThreads), L::BYTES, s,
                       tm, tm_o, a, kLog2eF / sqrtf((float)D));
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const AttnArgs& a, cudaStream_t s) {
  if (a.d == 128 && a.dq_fix) return bwd_fused_tc(a, s);
  if (a.d == 64) return bwd_tc<64>(a, s);
  if (a.d == 128) return bwd_tc<128>(a, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_fwd_tc(const AttnArgs& a, cudaStream_t s) {
  if (a.d == 64) return fwd_tc<64>(a, s);
  if (a.d == 128) return fwd_tc<128>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace mgt
