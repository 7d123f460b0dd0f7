// backward_mom_tc.cuh -- chunkwise backward of the layer with SGD momentum on
// the sm_100a tensor cores (Variant 3 of Table 2 in the thelatestinai.com
// listing of "Test-Time Training with KV Binding Is Secretly Linear
// Attention": per-token learning rate, momentum in SGD; its Figure 4 trains
// with the parallel form, which needs this gradient).
//
// Forward (update, then read): M_t = beta M_{t-1} - sigma v_t k_t^T,
// W_t = W_{t-1} - eta_t M_t, o_t = W_t q_t.  Reverse mode, with G_t = dL/dW_t
// and H_t = dL/dM_t (dL/dW_T, dL/dM_T given):
//   G_t = G_{t+1} + do_t q_t^T              (G_T := dL/dW_T)
//   H_t = beta H_{t+1} - eta_t G_t          (beta H_T := dL/dM_T)
//   dv_t = -sigma H_t k_t,   dk_t = -sigma H_t^T v_t,
//   deta_t = -<G_t, M_t>,    dq_t = W_t^T do_t,
//   dL/dW_0 = G_0,           dL/dM_0 = beta H_0.
// dq is the momentum forward itself on (q, k, v) := (do, v, k) from W_0^T,
// M_0^T (chunked_tc_mom.cuh).  The rest regroups over chunks of C tokens
// (local i, j, n valid) exactly:
//
// Reverse kernel (chunks last to first; carried state G and X = beta H at
// the chunk's end), with e_i = sum_{r=i}^{n-1} beta^(r-i) eta_r and
// w_ij = sum_{r=i}^{j} beta^(r-i) eta_r = e_i - beta^(j+1-i) e_{j+1} (j >= i;
// no division, so no cancellation that grows like beta^-C):
//   dv_i = -sigma beta^(n-1-i) X k_i + sigma e_i G k_i
//          + sigma sum_{j>=i} w_ij (k_i . q_j) do_j
//   X   <- beta^n X - beta e_0 G - sum_j beta w_0j do_j q_j^T
//   G   <- G + sum_j do_j q_j^T
// and dk is the same kernel on (k, q, do) := (v, do, q) from the transposed
// states.  deta kernel (chunks first to last; carried state M and
// P = -G = sum of do q^T so far - dL/dW_0, G at the chunk's start):
//   <G_t, M_t> = beta^(i+1) (<G, M> - sum_{j<i} y_j) - sigma sum_{s<=i} beta^(i-s) z_s
//                + sigma sum_{s<=i} beta^(i-s) F_is,
//   y_j = do_j . (M q_j),  z_s = v_s . (G k_s),
//   F = Lstrict (Q K^T o dO V^T)   (Lstrict: ones strictly below the diagonal)
//   M <- beta^n M - sigma sum_s beta^(n-1-s) v_s k_s^T,  P <- P + sum_j do_j q_j^T.
// z reads G through two bf16 MMAs (bf16(x) + bf16(x - bf16(x)), which carries
// it to about 2^-17): deta is a d^2-term inner product that can cancel, and
// G holds dL/dW_T.  y reads M in bf16 alone (its rounding measured no larger
// than the rest at the test scales).
//
// One block per (b, h, 64 rows of the state) walks its chunks in order (no
// segment scan): every term above is linear in the rows of the states (and of
// dv, dk), so a block owns rows [r0, r0 + 64) of G, X (or M, P) and the
// matching 64 columns of the output, with its own copy of the scores; the
// deta blocks of one head add their partial sums into a zeroed deta.  Warp 0
// loads tiles with TMA, warp 1 owns TMEM and issues the MMAs, warps 2-5 (one
// TMEM lane each) run the epilogue, and the rest scale operand copies (and,
// in the reverse kernel, store the output rows).  Every wait is bounded
// (common.cuh); a thread whose wait runs out stops waiting but keeps
// arriving, so the block drains and exits.
#pragma once
#include "chunked_tc.cuh"
#include "common.cuh"

namespace ttt {

struct MomBwdParams {
  int BH, T, nchunks;
  const float* eta;    // [BH, T] or nullptr (reverse kernel)
  float eta_const, sigma, beta;
  const float* G_in;   // [BH, D, D] row-major: reverse: dL/dW_T (or its transpose), deta: dL/dW_0; or nullptr
  const float* X_in;   // reverse: dL/dM_T (or its transpose); deta: M_0; or nullptr (zero)
  float* G_out;        // reverse: dL/dW_0 or nullptr
  float* X_out;        // reverse: dL/dM_0 or nullptr
  float* deta;         // deta kernel: [BH, T]
  uint64_t limit_ns;
};

// x * s for both bf16 halves of `u`, in fp32 with one rounding.
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t u, float s) {
  const float2 f = unpack_bf16x2(u);
  return pack_bf16x2(f.x * s, f.y * s);
}

// fp32 row values (raw bits) split into bf16(x) and bf16(x - bf16(x)), written
// as row `row`, columns [col0, col0 + 32) of two 64-row K-major SW128 tiles.
__device__ __forceinline__ void store_row32_split(uint32_t hi, uint32_t lo, int row, int col0, uint32_t (&r)[32]) {
  store_row32_bf16(hi, 64 * 128, row, col0, r);
  to_residual(r);
  store_row32_bf16(lo, 64 * 128, row, col0, r);
}

// Store counterpart of tmem_ld_half32 (common.cuh): threads 0-15 write lanes
// 0-15 of the warp's quadrant at columns [c, c + 32), threads 16-31 the same
// lanes at [c + 32, c + 64).
__device__ __forceinline__ void tmem_st_half32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 32, {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// A block's share of the state rows (one M = 64 accumulator).
constexpr int kMomRows = 64;

template <int D>
struct MomRevCfg {
  static constexpr int C = 64, RS = kMomRows;
  static constexpr int TILE = C * D * 2;          // bf16 C x D
  static constexpr int SQ = RS * D * 2;           // bf16 RS x D
  static constexpr int NST = 3;
  static constexpr int STAGE = 3 * TILE;          // K, Q, dO roles
  // bf16 rows of X and of G stacked as one B operand of 128 rows per
  // 64-column block (X rows 0-63, G rows 64-127), so (2) is one N = 128 MMA
  static constexpr int OFF_XG = NST * STAGE;
  static constexpr int OFF_QW = OFF_XG + 2 * SQ;  // [2] diag(-beta w_0j) Q (chunk parity)
  static constexpr int OFF_P = OFF_QW + 2 * TILE; // C x C weights
  static constexpr int BIG = OFF_P + C * C * 2;
  static constexpr int NE = 3;                    // coefficient slots
  static constexpr int ES = C + 4;                // slot stride (floats): e_1 .. e_C 16-byte aligned
  static constexpr int NBAR = 3 * NST + 13;
  static_assert(NBAR % 2 == 0, "coefficient slots start 16-byte aligned");
  static constexpr int SMALL = NBAR * 8 + (NE * ES + (C + 1) + 4) * 4 + 16;
  static constexpr int SMEM = BIG + SMALL + 1024;
  static constexpr int TCOLS_USED = 2 * D + C + 3 * RS;  // G, X, scores, U1, U2, U3
  static constexpr int TCOLS = TCOLS_USED <= 256 ? 256 : 512;
  static constexpr int THREADS = 352;             // 11 warps
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(SMEM <= 232448, "shared memory");
};

template <int D>
struct MomDetaCfg {
  static constexpr int C = 64, RS = kMomRows;
  static constexpr int TILE = C * D * 2;
  static constexpr int NST = 2;
  // Q, then K with the chunk's bf16 rows of M stacked below it (one B
  // operand of 128 rows per 64-column block: K rows 0-63, M rows 64-127),
  // then V and dO
  static constexpr int OFF_SK = TILE, OFF_SV = 3 * TILE, OFF_SD = 4 * TILE;
  static constexpr int STAGE = 5 * TILE;
  static constexpr int SQ = RS * D * 2;
  static constexpr int OFF_GBF = NST * STAGE;     // bf16 rows of G and their residual
  static constexpr int OFF_GLO = OFF_GBF + SQ;
  static constexpr int OFF_KB = OFF_GLO + SQ;     // diag(-sigma beta^(n-1-s)) K
  static constexpr int OFF_A = OFF_KB + TILE;     // bf16(Q K^T o dO V^T), token-major
  static constexpr int OFF_L = OFF_A + C * C * 2; // strictly lower ones
  static constexpr int BIG = OFF_L + C * C * 2;
  static constexpr int NBAR = 2 * NST + 15;
  static constexpr int SMALL = NBAR * 8 + ((C + 1) + 6 * C + 10) * 4 + 16;
  static constexpr int SMEM = BIG + SMALL + 1024;
  static constexpr int TCOLS_USED = 2 * D + 3 * C + RS;  // M, P, S1, S2, F, Y / Z
  static constexpr int TCOLS = TCOLS_USED <= 256 ? 256 : 512;
  static constexpr int THREADS = 352;             // 11 warps
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(TCOLS_USED <= 512, "tensor memory");
  static_assert(SMEM <= 232448, "shared memory");
};

// Reverse kernel: tmK, tmQ, tmD are the K, Q and dO roles (dv: k, q, do;
// dk: v, do, q), tmO the output rows; block (bh, r0) owns state rows
// [r0, r0 + 64) and output columns [r0, r0 + 64) (dO_r: those columns of dO).
// Per chunk the MMA thread issues
//   (1) S  = K Q^T                            [TMEM, M=C, N=C]
//   (2) [U1 | U2] = K [Xbf ; Gbf]^T           [TMEM, M=C, N=128]
//   (3) G += dO_r^T Q,  (4) X += dO_r^T Qw    [TMEM, M=64, N=D]
//   (5) U3 += P dO_r                          P = bf16(sigma w o triu(S))
// after the epilogue has taken Xbf, Gbf and replaced X by beta^n X - beta e_0 G,
// and, before (5), set U3 to the rows' fp32 combination -sigma beta^(n-1-i) U1
// + sigma e_i U2; U3 is then the output row.  The epilogue takes the next
// chunk's Xbf, Gbf while (5) runs.
// The coefficients e and the copy Qw of a chunk are made while the previous
// chunk's MMAs run (three coefficient slots, two Qw buffers).
template <int D>
__global__ void __launch_bounds__(MomRevCfg<D>::THREADS, 1)
    mom_bwd_rev_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmO,
                       const MomBwdParams p) {
  using Cfg = MomRevCfg<D>;
  constexpr int C = Cfg::C, RS = Cfg::RS, NST = Cfg::NST, TILE = Cfg::TILE, STAGE = Cfg::STAGE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BIG);
  uint64_t* full = bars;                // [NST] tiles landed
  uint64_t* empty = bars + NST;         // [NST] output rows stored: stage free
  uint64_t* staged = bars + 2 * NST;    // [NST] output rows written into the stage's K slot
  // Barriers the coefficient warps fill run one per slot, so that none of
  // them can complete two phases ahead of a waiter.
  uint64_t* e_ready = bars + 3 * NST;   // [3] e of the chunks of slot c % 3 written
  uint64_t* qw_ready = e_ready + 3;     // [2] Qw of the chunks of parity c & 1 written
  uint64_t* ks_free = qw_ready + 2;     // [2] (2)-(4) of the chunks of parity c & 1 done: Qw buffer free
  uint64_t* wbf_ready = ks_free + 2;    // Xbf, Gbf written, X rewritten
  uint64_t* sc_full = wbf_ready + 1;    // (1) done
  uint64_t* sdone = wbf_ready + 2;      // (2)-(4) done
  uint64_t* p_ready = wbf_ready + 3;    // P written and U3 set
  uint64_t* o_full = wbf_ready + 4;     // (5) done
  uint64_t* drain = wbf_ready + 5;
  // [NE][ES]: slot x holds e_0 .. e_C (e_C = 0) from float 3, so that e_1 .. e_C are 16-byte aligned
  float* ebuf = reinterpret_cast<float*>(bars + Cfg::NBAR);
  float* bpow = ebuf + Cfg::NE * Cfg::ES;                     // [C + 1] beta^k
  float* xw = bpow + C + 1;                                   // [4] cross-warp carry of the e scan
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(xw + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.limit_ns;
  const int bh = blockIdx.x / (D / RS), r0 = (blockIdx.x % (D / RS)) * RS, rb = r0 / 64;
  const int nch = p.nchunks;
  // logical chunk c is chunk nch - 1 - c of the sequence, with n valid tokens
  auto phys = [&](int c) { return nch - 1 - c; };
  auto nvalid = [&](int c) { return min(C, p.T - phys(c) * C); };

  if (threadIdx.x <= C) {
    float b = 1.f;
    for (int k = 0; k < static_cast<int>(threadIdx.x); ++k) b *= p.beta;
    bpow[threadIdx.x] = b;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&staged[s], 128);
    }
    for (int x = 0; x < 3; ++x) mbar_init(&e_ready[x], 64);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&qw_ready[x], 128);
      mbar_init(&ks_free[x], 1);
    }
    mbar_init(wbf_ready, 128);
    mbar_init(sc_full, 1);
    mbar_init(sdone, 1);
    mbar_init(p_ready, 128);
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::TCOLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmD);
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t t_g = tmem, t_x = tmem + D, t_s = tmem + 2 * D;
  const uint32_t t_u1 = t_s + C, t_u2 = t_u1 + RS, t_u3 = t_u2 + RS;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      bool dead = false;
      for (int c = 0; c < nch; ++c) {
        const int s = c % NST, u = c / NST;
        if (u > 0 && !dead) dead = !mbar_wait(&empty[s], (u - 1) & 1, lim);
        mbar_arrive_expect_tx(&full[s], 3 * TILE);
        uint8_t* st = smem + s * STAGE;
        const int t0 = phys(c) * C;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_load_3d(&tmK, &full[s], st + kb * C * 128, kb * 64, t0, bh);
          tma_load_3d(&tmQ, &full[s], st + TILE + kb * C * 128, kb * 64, t0, bh);
          tma_load_3d(&tmD, &full[s], st + 2 * TILE + kb * C * 128, kb * 64, t0, bh);
        }
      }
      for (int j = max(0, nch - NST); j < nch; ++j) mbar_wait(&full[j % NST], (j / NST) & 1, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      bool dead = false;
      constexpr uint32_t ID_S = idesc_bf16_f32(C, C, false, false);
      constexpr uint32_t ID_U = idesc_bf16_f32(C, 2 * RS, false, false);
      constexpr uint32_t ID_ST = idesc_bf16_f32(RS, D, true, true);
      constexpr uint32_t ID_PU = idesc_bf16_f32(C, RS, false, true);
      const uint64_t d_xg = sdesc_sw128(sbase + Cfg::OFF_XG, 16, 1024);
      const uint64_t d_p = sdesc_sw128(sbase + Cfg::OFF_P, 16, 1024);
      for (int c = 0; c < nch; ++c) {
        const int s = c % NST, u = c / NST;
        const uint32_t st = sbase + s * STAGE;
        const uint64_t d_k = sdesc_sw128(st, 16, 1024), d_q = sdesc_sw128(st + TILE, 16, 1024);
        const uint64_t d_qm = sdesc_sw128(st + TILE, C * 128, 1024);
        const uint64_t d_dm = sdesc_sw128(st + 2 * TILE + rb * C * 128, C * 128, 1024);  // this block's dO columns
        const uint64_t d_qw = sdesc_sw128(sbase + Cfg::OFF_QW + (c & 1) * TILE, C * 128, 1024);  // MN-major
        if (!dead) dead = !mbar_wait(&full[s], u & 1, lim);
        tc_fence_after();
        // (1); the scores of chunk c-1 were read before p_ready(c-1), waited below
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_bf16_ss(t_s, d_k + k_step(C, kk), d_q + k_step(C, kk), ID_S, kk > 0);
        tc_commit(sc_full);
        if (!dead) dead = !mbar_wait(&qw_ready[c & 1], (c >> 1) & 1, lim);
        if (!dead) dead = !mbar_wait(wbf_ready, c & 1, lim);
        tc_fence_after();
        // (2) into U1 and U2 (adjacent columns); the epilogue read U1, U2 of chunk c-1 before wbf_ready(c)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(t_u1, d_k + k_step(C, kk), d_xg + k_step(2 * RS, kk), ID_U, kk > 0);
        // (3), (4)
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_g, d_dm + mn_step(kk), d_qm + mn_step(kk), ID_ST, 1);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_x, d_dm + mn_step(kk), d_qw + mn_step(kk), ID_ST, 1);
        tc_commit(sdone);
        tc_commit(&ks_free[c & 1]);
        if (!dead) dead = !mbar_wait(p_ready, c & 1, lim);
        tc_fence_after();
        // (5) onto U3, which the epilogue has set to the rows' combination of U1 and U2 (p_ready)
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_u3, d_p + k_step(C, kk), d_dm + mn_step(kk), ID_PU, 1);
        tc_commit(o_full);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, lim);
    }
  } else if (warp == 6) {
    // ------------------------------------------------ output store warp --
    if (lane == 0) {
      bool dead = false;
      for (int c = 0; c < nch; ++c) {
        const int s = c % NST;
        if (!dead) dead = !mbar_wait(&staged[s], (c / NST) & 1, lim);
        tma_store_3d(&tmO, smem + s * STAGE, r0, phys(c) * C, bh);
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(&empty[s]);
      }
      bulk_wait0();
    }
  } else if (warp >= 7) {
    // ------------------------------------------------ coefficient warps --
    // e_i of chunk c (warps 7-8, one token per thread: a shuffle scan within
    // each warp and one carry across), then Qw into the buffer of c's parity
    // (warps 7-10).  Both wait
    // only for (2)-(4) of chunk c - 2: slot c % 3 of e was last read by the
    // epilogue's P of chunk c - 3, which precedes its Xbf of chunk c - 2.
    const int tid = threadIdx.x - 224;  // 0..127; 0..63 (warps 7-8) also one token each
    const bool scan = tid < 64;
    bool dead = false;
    auto eta_of = [&](int c) {
      const int t = phys(c) * C + tid;
      return (tid < nvalid(c)) ? (p.eta ? __ldg(p.eta + static_cast<size_t>(bh) * p.T + t) : p.eta_const) : 0.f;
    };
    float eta_next = scan ? eta_of(0) : 0.f;
    for (int c = 0; c < nch; ++c) {
      const int s = c % NST;
      float* e = ebuf + (c % Cfg::NE) * Cfg::ES + 3;
      float v = eta_next;
      if (scan && c + 1 < nch) eta_next = eta_of(c + 1);
      if (c >= 2 && !dead) dead = !mbar_wait(&ks_free[c & 1], ((c >> 1) - 1) & 1, lim);
      // v_i = sum_{r=i}^{end of the warp's 32 tokens} beta^(r-i) eta_r
      if (scan) {
#pragma unroll
        for (int k = 1; k < 32; k <<= 1) {
          const float u = __shfl_down_sync(0xffffffffu, v, k);
          if (lane + k < 32) v = fmaf(bpow[k], u, v);
        }
        if (warp == 8 && lane == 0) xw[0] = v;  // e_32
        asm volatile("bar.sync 2, 64;" ::: "memory");
        if (warp == 7) v = fmaf(bpow[32 - lane], xw[0], v);
        e[tid] = v;
        if (tid == 0) e[C] = 0.f;
        asm volatile("bar.sync 2, 64;" ::: "memory");
        mbar_arrive(&e_ready[c % 3]);
      }
      asm volatile("bar.sync 3, 128;" ::: "memory");  // e of chunk c written
      if (!dead) dead = !mbar_wait(&full[s], (c / NST) & 1, lim);
      const uint8_t* qr = smem + s * STAGE + TILE;
      uint8_t* qw = smem + Cfg::OFF_QW + (c & 1) * TILE;
      const float e0 = e[0];
#pragma unroll 4
      for (int k = 0; k < D / 16; ++k) {
        const int idx = tid + 128 * k;
        const int r = idx / (D / 8), cc = idx % (D / 8);
        const uint32_t off = (cc >> 3) * C * 128 + sw128_off(r, cc & 7);
        const float cw = -p.beta * (e0 - bpow[r + 1] * e[r + 1]);
        const uint4 b = *reinterpret_cast<const uint4*>(qr + off);
        *reinterpret_cast<uint4*>(qw + off) =
            make_uint4(scale_bf16x2(b.x, cw), scale_bf16x2(b.y, cw), scale_bf16x2(b.z, cw), scale_bf16x2(b.w, cw));
      }
      fence_async_smem();
      mbar_arrive(&qw_ready[c & 1]);
    }
  } else {
    // --------------------------------------------------------- epilogue --
    const int g4 = warp & 3;  // TMEM lane quadrant of this warp
    const uint32_t lane_off = static_cast<uint32_t>(32 * g4) << 16;
    // M = 64 accumulators fill lanes 0-15 of each quadrant; the whole warp
    // reads them: row 16 g4 + lane % 16, column half lane / 16
    const int row64h = 16 * g4 + (lane & 15), half = lane >> 4;
    const size_t DD = static_cast<size_t>(D) * D, nst = static_cast<size_t>(p.BH) * DD;
    const size_t grow = bh * DD + static_cast<size_t>(r0 + row64h) * D;  // this thread's state row in global
    bool dead = false;
    // (b) of chunk c: Xbf, Gbf from the chunk-end states; X <- beta^n X - beta e_0 G
    auto take = [&](int c) {
      const int n = nvalid(c);
      const float* e = ebuf + (c % Cfg::NE) * Cfg::ES + 3;
      if (c >= 1 && !dead) dead = !mbar_wait(sdone, (c - 1) & 1, lim);
      if (!dead) dead = !mbar_wait(&e_ready[c % 3], (c / 3) & 1, lim);
      tc_fence_after();
      const float xs = bpow[n], gs = -p.beta * e[0];
#pragma unroll 1
      for (int cb = 0; cb < D; cb += 64) {
        const int col = cb + 32 * half;
        uint32_t g[32], x[32];
        if (c == 0) {
          const float* gi = p.G_in ? TTT_AT(p.G_in, grow + col, 32, nst) : nullptr;
          const float* xi = p.X_in ? TTT_AT(p.X_in, grow + col, 32, nst) : nullptr;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            g[j] = __float_as_uint(gi ? __ldg(gi + j) : 0.f);
            x[j] = __float_as_uint(xi ? __ldg(xi + j) : 0.f);
          }
          tmem_st_half32(t_g + lane_off + cb, g);  // G accumulator := dL/dW_T (rows)
        } else {
          tmem_ld_half32(t_g + lane_off + cb, g);
          tmem_ld_half32(t_x + lane_off + cb, x);
          tmem_ld_wait();
        }
        store_row32_bf16(sbase + Cfg::OFF_XG, 2 * RS * 128, row64h, col, x);
        store_row32_bf16(sbase + Cfg::OFF_XG, 2 * RS * 128, RS + row64h, col, g);
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = __float_as_uint(fmaf(xs, __uint_as_float(x[j]), gs * __uint_as_float(g[j])));
        tmem_st_half32(t_x + lane_off + cb, x);
      }
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(wbf_ready);
    };
    // Per chunk: P (the scores land early), U3 := -sigma beta^(n-1-i) U1 +
    // sigma e_i U2 once (2) is done, then (b) of the next chunk while (5) adds
    // P dO onto U3, then U3 out.
    take(0);
    for (int c = 0; c < nch; ++c) {
      const int s = c % NST, n = nvalid(c);
      const float* e = ebuf + (c % Cfg::NE) * Cfg::ES + 3;
      const int i = row64h;
      // (d) P_ij = sigma w_ij S_ij for j >= i, w_ij = e_i - beta^(j+1-i) e_{j+1}; the
      // power of beta runs along the row from the first unmasked column
      if (!dead) dead = !mbar_wait(sc_full, c & 1, lim);
      tc_fence_after();
      {
        uint32_t r[32];
        tmem_ld_half32(t_s + lane_off, r);
        tmem_ld_wait();
        const float ei = e[i];
        const int jlo = 32 * half;
        float pw = bpow[max(jlo, i) + 1 - i];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 e0 = *reinterpret_cast<const float4*>(e + jlo + 8 * q + 1);
          const float4 e1 = *reinterpret_cast<const float4*>(e + jlo + 8 * q + 5);
          const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
          float a[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const int j = jlo + 8 * q + h;
            a[h] = 0.f;
            if (j >= i) {
              a[h] = p.sigma * (ei - pw * ev[h]) * __uint_as_float(r[8 * q + h]);
              pw *= p.beta;
            }
          }
          st_shared_v4(sbase + Cfg::OFF_P + sw128_off(i, 4 * half + q), pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                       pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
        }
      }
      fence_async_smem();
      // (u) U1, U2 are complete with (2)-(4): their rows' combination goes into U3
      if (!dead) dead = !mbar_wait(sdone, c & 1, lim);
      tc_fence_after();
      {
        uint32_t u1[32], u2[32];
        tmem_ld_half32(t_u1 + lane_off, u1);
        tmem_ld_half32(t_u2 + lane_off, u2);
        tmem_ld_wait();
        const float a1 = (i < n) ? -p.sigma * bpow[max(n - 1 - i, 0)] : 0.f, a2 = p.sigma * e[i];
#pragma unroll
        for (int j = 0; j < 32; ++j) u1[j] = __float_as_uint(fmaf(a1, __uint_as_float(u1[j]), a2 * __uint_as_float(u2[j])));
        tmem_st_half32(t_u3 + lane_off, u1);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(p_ready);
      // (b) of the next chunk while (5) runs (U1, U2 of this chunk are read)
      if (c + 1 < nch) take(c + 1);
      // (f) U3 -> bf16 -> the stage's K slot (every MMA of the chunk is done), then the store warp
      if (!dead) dead = !mbar_wait(o_full, c & 1, lim);
      tc_fence_after();
      {
        uint32_t r[32];
        tmem_ld_half32(t_u3 + lane_off, r);
        tmem_ld_wait();
        store_row32_bf16(sbase + s * STAGE, C * 128, row64h, 32 * half, r);
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(&staged[s]);
    }
    // final states: G = dL/dW_0, X = beta H_0 = dL/dM_0 (this block's rows)
    if (!dead) dead = !mbar_wait(sdone, (nch - 1) & 1, lim);
    tc_fence_after();
#pragma unroll 1
    for (int cb = 0; cb < D; cb += 64) {
      const int col = cb + 32 * half;
      uint32_t g[32], x[32];
      tmem_ld_half32(t_g + lane_off + cb, g);
      tmem_ld_half32(t_x + lane_off + cb, x);
      tmem_ld_wait();
      if (p.G_out) {
        float4* d4 = reinterpret_cast<float4*>(TTT_AT(p.G_out, grow + col, 32, nst));
#pragma unroll
        for (int j = 0; j < 8; ++j)
          d4[j] = make_float4(__uint_as_float(g[4 * j]), __uint_as_float(g[4 * j + 1]), __uint_as_float(g[4 * j + 2]),
                              __uint_as_float(g[4 * j + 3]));
      }
      if (p.X_out) {
        float4* d4 = reinterpret_cast<float4*>(TTT_AT(p.X_out, grow + col, 32, nst));
#pragma unroll
        for (int j = 0; j < 8; ++j)
          d4[j] = make_float4(__uint_as_float(x[4 * j]), __uint_as_float(x[4 * j + 1]), __uint_as_float(x[4 * j + 2]),
                              __uint_as_float(x[4 * j + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::TCOLS);
}

// deta kernel: tmQ, tmK, tmV, tmD over q, k, v, do; G_in = dL/dW_0, X_in =
// M_0; block (bh, r0) owns rows [r0, r0 + 64) of M and P (V_r, dO_r: those
// columns of V and dO) and adds its partial deta.  Per chunk the MMA thread
// issues
//   (1) [S1 | Y] = Q [K ; Mbf]^T,  S2 = dO_r V_r^T   [TMEM, M=C, N=128 and 64]
//   (2') Z = K Gbf^T + K Glo^T                  (Y's columns, once y is read)
//   (4) M += V_r^T Kb,  P += dO_r^T Q           [TMEM, M=64, N=D]
//   (3) F  = Lstrict A,  A = bf16(S1 o S2)      [TMEM, M=C, N=C]
// after the epilogue has taken the bf16 copies of M and G = -P and replaced M
// by beta^n M.  The epilogue (warps 2-5) takes chunk c+1's states as soon as it
// has read z of chunk c and handed y, z over; warps 7-10 read F and finish the
// chunk's deta meanwhile.
template <int D>
__global__ void __launch_bounds__(MomDetaCfg<D>::THREADS, 1)
    mom_bwd_deta_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmD,
                        const MomBwdParams p) {
  using Cfg = MomDetaCfg<D>;
  constexpr int C = Cfg::C, RS = Cfg::RS, NST = Cfg::NST, TILE = Cfg::TILE, STAGE = Cfg::STAGE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BIG);
  uint64_t* full = bars;                 // [NST] tiles landed
  uint64_t* empty = bars + NST;          // [NST] stage free: (3) issued after (1)-(4), and the epilogue read V, dO
  uint64_t* mbf_ready = bars + 2 * NST;  // bf16 pairs written, M rewritten
  uint64_t* sc_full = mbf_ready + 1;
  // (mbf_ready + 2 unused: Y lands with S1, on sc_full)
  uint64_t* y_free = mbf_ready + 3;
  uint64_t* z_full = mbf_ready + 4;
  uint64_t* kb_ready = mbf_ready + 5;
  uint64_t* sdone = mbf_ready + 6;       // (2)-(4) done
  uint64_t* a_ready = mbf_ready + 7;
  uint64_t* f_full = mbf_ready + 8;
  uint64_t* drain = mbf_ready + 9;
  uint64_t* f_free = mbf_ready + 10;     // F read out of TMEM
  uint64_t* yz_ready = mbf_ready + 11;   // [2] y, z, <G, M> of the chunks of parity c & 1 handed over
  uint64_t* yz_free = mbf_ready + 13;    // [2] that slot read
  float* bpow = reinterpret_cast<float*>(bars + Cfg::NBAR);  // [C + 1] beta^k
  float* ybuf = bpow + C + 1;                                 // [2][C] y of the chunk (slot c & 1)
  float* zbuf = ybuf + 2 * C;                                 // [2][C] z
  float* ypre = zbuf + 2 * C;                                 // [C] prefix sums of y
  float* zpre = ypre + C;                                     // [C] beta-weighted prefix sums of z
  float* g0buf = zpre + C;                                    // [2] <G, M> at the chunk's start
  float* red = g0buf + 2;                                     // [8]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(red + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.limit_ns;
  const int bh = blockIdx.x / (D / RS), r0 = (blockIdx.x % (D / RS)) * RS, rb = r0 / 64;
  const int nch = p.nchunks;
  auto nvalid = [&](int c) { return min(C, p.T - c * C); };

  if (threadIdx.x <= C) {
    float b = 1.f;
    for (int k = 0; k < static_cast<int>(threadIdx.x); ++k) b *= p.beta;
    bpow[threadIdx.x] = b;
  }
  // Lstrict (K-major, one 64-column block): 1 where column < row
  for (int u = threadIdx.x; u < C * 8; u += blockDim.x) {
    const int r = u >> 3, c16 = u & 7;
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) w[h] = pack_bf16x2(8 * c16 + 2 * h < r ? 1.f : 0.f, 8 * c16 + 2 * h + 1 < r ? 1.f : 0.f);
    st_shared_v4(sbase + Cfg::OFF_L + sw128_off(r, c16), w[0], w[1], w[2], w[3]);
  }
  fence_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 129);
    }
    mbar_init(mbf_ready, 128);
    mbar_init(sc_full, 1);
    mbar_init(y_free, 128);
    mbar_init(z_full, 1);
    mbar_init(kb_ready, 1);
    mbar_init(sdone, 1);
    mbar_init(a_ready, 128);
    mbar_init(f_full, 1);
    mbar_init(drain, 1);
    mbar_init(f_free, 128);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&yz_ready[x], 128);
      mbar_init(&yz_free[x], 128);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::TCOLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmD);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // S1 and Y adjacent: (1) writes both
  const uint32_t t_m = tmem, t_p = tmem + D, t_s1 = tmem + 2 * D, t_yz = t_s1 + C, t_s2 = t_yz + RS, t_f = t_s2 + C;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      bool dead = false;
      for (int c = 0; c < nch; ++c) {
        const int s = c % NST, u = c / NST;
        if (u > 0 && !dead) dead = !mbar_wait(&empty[s], (u - 1) & 1, lim);
        mbar_arrive_expect_tx(&full[s], 4 * TILE);
        uint8_t* st = smem + s * STAGE;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_load_3d(&tmQ, &full[s], st + kb * C * 128, kb * 64, c * C, bh);
          tma_load_3d(&tmK, &full[s], st + Cfg::OFF_SK + kb * 2 * C * 128, kb * 64, c * C, bh);  // rows 0-63
          tma_load_3d(&tmV, &full[s], st + Cfg::OFF_SV + kb * C * 128, kb * 64, c * C, bh);
          tma_load_3d(&tmD, &full[s], st + Cfg::OFF_SD + kb * C * 128, kb * 64, c * C, bh);
        }
      }
      for (int j = max(0, nch - NST); j < nch; ++j) mbar_wait(&full[j % NST], (j / NST) & 1, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      bool dead = false;
      constexpr uint32_t ID_S = idesc_bf16_f32(C, C, false, false);
      constexpr uint32_t ID_SY = idesc_bf16_f32(C, C + RS, false, false);
      constexpr uint32_t ID_Y = idesc_bf16_f32(C, RS, false, false);
      constexpr uint32_t ID_ST = idesc_bf16_f32(RS, D, true, true);
      constexpr uint32_t ID_F = idesc_bf16_f32(C, C, false, true);
      const uint64_t d_gbf = sdesc_sw128(sbase + Cfg::OFF_GBF, 16, 1024);
      const uint64_t d_glo = sdesc_sw128(sbase + Cfg::OFF_GLO, 16, 1024);
      const uint64_t d_kbm = sdesc_sw128(sbase + Cfg::OFF_KB, C * 128, 1024);  // MN-major
      const uint64_t d_am = sdesc_sw128(sbase + Cfg::OFF_A, C * 128, 1024);    // MN-major
      const uint64_t d_l = sdesc_sw128(sbase + Cfg::OFF_L, 16, 1024);
      for (int c = 0; c < nch; ++c) {
        const int s = c % NST, u = c / NST;
        const uint32_t st = sbase + s * STAGE;
        const uint32_t vr = st + Cfg::OFF_SV + rb * C * 128, dr = st + Cfg::OFF_SD + rb * C * 128;  // this block's columns
        // K and [K ; Mbf]: 128-row blocks (k_step over 2C rows); K as an A operand reads rows 0-63
        const uint64_t d_q = sdesc_sw128(st, 16, 1024), d_k = sdesc_sw128(st + Cfg::OFF_SK, 16, 1024);
        const uint64_t d_vr = sdesc_sw128(vr, 16, 1024), d_dr = sdesc_sw128(dr, 16, 1024);
        const uint64_t d_qm = sdesc_sw128(st, C * 128, 1024);
        const uint64_t d_vrm = sdesc_sw128(vr, C * 128, 1024), d_drm = sdesc_sw128(dr, C * 128, 1024);
        if (!dead) dead = !mbar_wait(&full[s], u & 1, lim);
        // the epilogue has read S1, S2, Z of chunk c-1 before taking chunk c's bf16 pairs
        if (!dead) dead = !mbar_wait(mbf_ready, c & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(t_s1, d_q + k_step(C, kk), d_k + k_step(2 * C, kk), ID_SY, kk > 0);  // [S1 | Y]
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(t_s2, d_dr + k_step(C, kk), d_vr + k_step(C, kk), ID_S, kk > 0);
        tc_commit(sc_full);
        if (!dead) dead = !mbar_wait(y_free, c & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_bf16_ss(t_yz, d_k + k_step(2 * C, kk), d_gbf + k_step(RS, kk), ID_Y, kk > 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_bf16_ss(t_yz, d_k + k_step(2 * C, kk), d_glo + k_step(RS, kk), ID_Y, 1);
        tc_commit(z_full);
        if (!dead) dead = !mbar_wait(kb_ready, c & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
          mma_bf16_ss(t_m, d_vrm + mn_step(kk), d_kbm + mn_step(kk), ID_ST, 1);
          mma_bf16_ss(t_p, d_drm + mn_step(kk), d_qm + mn_step(kk), ID_ST, 1);
        }
        tc_commit(sdone);
        if (!dead) dead = !mbar_wait(a_ready, c & 1, lim);
        if (c >= 1 && !dead) dead = !mbar_wait(f_free, (c - 1) & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_f, d_l + k_step(C, kk), d_am + mn_step(kk), ID_F, kk > 0);
        tc_commit(f_full);
        tc_commit(&empty[s]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, lim);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------- K scaler --
    // Kb = diag(-sigma beta^(n-1-s)) K, once (4) of the previous chunk is done
    bool dead = false;
    for (int c = 0; c < nch; ++c) {
      const int s = c % NST, n = nvalid(c);
      if (!dead) dead = !mbar_wait(&full[s], (c / NST) & 1, lim);
      if (c >= 1 && !dead) dead = !mbar_wait(sdone, (c - 1) & 1, lim);
      const uint8_t* kt = smem + s * STAGE + Cfg::OFF_SK;
#pragma unroll 4
      for (int k = 0; k < D / 4; ++k) {
        const int idx = lane + 32 * k;
        const int r = idx / (D / 8), cc = idx % (D / 8);
        const uint32_t off = (cc >> 3) * C * 128 + sw128_off(r, cc & 7);  // Kb: 64-row blocks
        const uint32_t koff = (cc >> 3) * 2 * C * 128 + sw128_off(r, cc & 7);  // K: rows 0-63 of 128-row blocks
        const float cb = (r < n) ? -p.sigma * bpow[n - 1 - r] : 0.f;
        const uint4 a = *reinterpret_cast<const uint4*>(kt + koff);
        *reinterpret_cast<uint4*>(smem + Cfg::OFF_KB + off) =
            make_uint4(scale_bf16x2(a.x, cb), scale_bf16x2(a.y, cb), scale_bf16x2(a.z, cb), scale_bf16x2(a.w, cb));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(kb_ready);
    }
  } else if (warp >= 7) {
    // ------------------------------------------------ deta warps (7-10) --
    // Per chunk: rf_i = sum_{s<=i} beta^(i-s) F_is, the chunk's prefix sums
    // ypre_i = sum_{j<i} y_j and zpre_i = sum_{s<=i} beta^(i-s) z_s (two warps,
    // two tokens a lane, shuffle scans), then this block's part of deta.
    const int g4 = warp & 3;  // TMEM lane quadrant (warps 7-10 cover all four)
    const uint32_t lane_off = static_cast<uint32_t>(32 * g4) << 16;
    const int row64h = 16 * g4 + (lane & 15), half = lane >> 4;
    bool dead = false;
    for (int c = 0; c < nch; ++c) {
      const int n = nvalid(c);
      const float* ys = ybuf + (c & 1) * C;
      const float* zs = zbuf + (c & 1) * C;
      if (!dead) dead = !mbar_wait(&yz_ready[c & 1], (c >> 1) & 1, lim);
      if (!dead) dead = !mbar_wait(f_full, c & 1, lim);
      tc_fence_after();
      float rf = 0.f;
      {
        uint32_t r[32];
        tmem_ld_half32(t_f + lane_off, r);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int sc = 32 * half + jj;
          rf += (sc <= row64h) ? bpow[max(row64h - sc, 0)] * __uint_as_float(r[jj]) : 0.f;
        }
        rf += __shfl_xor_sync(0xffffffffu, rf, 16);
      }
      tc_fence_before();
      mbar_arrive(f_free);
      if (g4 < 2) {
        const float a0 = (g4 == 0 ? ys : zs)[2 * lane], a1 = (g4 == 0 ? ys : zs)[2 * lane + 1];
        // pair sum (y) or pair value beta a0 + a1 (z), then an inclusive scan over the lanes
        float pr = (g4 == 0) ? a0 + a1 : fmaf(p.beta, a0, a1);
#pragma unroll
        for (int k = 1; k < 32; k <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, pr, k);
          if (lane >= k) pr = fmaf(g4 == 0 ? 1.f : bpow[2 * k], u, pr);
        }
        const float prev = __shfl_up_sync(0xffffffffu, pr, 1);  // through token 2 lane - 1
        const float pv = lane > 0 ? prev : 0.f;
        if (g4 == 0) {
          ypre[2 * lane] = pv;
          ypre[2 * lane + 1] = pv + a0;
        } else {
          zpre[2 * lane] = fmaf(p.beta, pv, a0);
          zpre[2 * lane + 1] = pr;
        }
      }
      asm volatile("bar.sync 4, 128;" ::: "memory");
      if (half == 0 && row64h < n) {
        const int i = row64h;
        const float val = bpow[i + 1] * (g0buf[c & 1] - ypre[i]) - p.sigma * zpre[i] + p.sigma * rf;
        atomicAdd(TTT_AT(p.deta, static_cast<size_t>(bh) * p.T + c * C + i, 1, static_cast<size_t>(p.BH) * p.T), -val);
      }
      mbar_arrive(&yz_free[c & 1]);
      asm volatile("bar.sync 4, 128;" ::: "memory");  // ypre, zpre read before the next chunk's scans
    }
  } else {
    // ------------------------------------------------ epilogue (2-5) --
    const int g4 = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * g4) << 16;
    // M = 64 accumulators fill lanes 0-15 of each quadrant; the whole warp
    // reads them: row 16 g4 + lane % 16, column half lane / 16
    const int row64h = 16 * g4 + (lane & 15), half = lane >> 4;
    const size_t DD = static_cast<size_t>(D) * D, nst = static_cast<size_t>(p.BH) * DD;
    bool dead = false;
    // this thread's half (32 columns) of row row64h of Y or Z, dotted with the
    // same columns of this block's 64 columns of a token tile
    auto row_dot = [&](const uint8_t* tile, const uint32_t (&r)[32]) {
      float acc = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 x = *reinterpret_cast<const uint4*>(tile + sw128_off(row64h, 4 * half + q));
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          acc = fmaf(__uint_as_float(w[h] << 16), __uint_as_float(r[8 * q + 2 * h]), acc);
          acc = fmaf(__uint_as_float(w[h] & 0xffff0000u), __uint_as_float(r[8 * q + 2 * h + 1]), acc);
        }
      }
      return acc + __shfl_xor_sync(0xffffffffu, acc, 16);  // the row's other half
    };
    // (b) of chunk c: bf16 pairs of M and G = -P, this block's part of <G, M>
    // (returned), M <- beta^n M
    auto take_states = [&](int c) {
      if (c >= 1 && !dead) dead = !mbar_wait(sdone, (c - 1) & 1, lim);
      tc_fence_after();
      const float bn = bpow[nvalid(c)];
      float part = 0.f;
      // the whole warp: row row64h, columns [cb + 32 half, cb + 32 half + 32)
#pragma unroll 1
      for (int cb = 0; cb < D; cb += 64) {
        const int col = cb + 32 * half;
        uint32_t m[32], g[32];
        if (c == 0) {
          const size_t row = bh * DD + static_cast<size_t>(r0 + row64h) * D + col;
          const float* mi = p.X_in ? TTT_AT(p.X_in, row, 32, nst) : nullptr;
          const float* gi = TTT_AT(p.G_in, row, 32, nst);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            m[j] = __float_as_uint(mi ? __ldg(mi + j) : 0.f);
            g[j] = __float_as_uint(-__ldg(gi + j));  // P := -dL/dW_0
          }
          tmem_st_half32(t_p + lane_off + cb, g);
        } else {
          tmem_ld_half32(t_m + lane_off + cb, m);
          tmem_ld_half32(t_p + lane_off + cb, g);
          tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float gj = -__uint_as_float(g[j]);  // G = -P
          g[j] = __float_as_uint(gj);
          part = fmaf(gj, __uint_as_float(m[j]), part);
        }
        store_row32_bf16(sbase + (c % NST) * STAGE + Cfg::OFF_SK, 2 * C * 128, C + row64h, col, m);  // rows 64-127
        store_row32_split(sbase + Cfg::OFF_GBF, sbase + Cfg::OFF_GLO, row64h, col, g);
#pragma unroll
        for (int j = 0; j < 32; ++j) m[j] = __float_as_uint(bn * __uint_as_float(m[j]));
        tmem_st_half32(t_m + lane_off + cb, m);
      }
      tmem_st_wait();
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      // by chunk parity: the barrier of chunk c+1's call orders chunk c+2's writes after these reads
      float* rd = red + (c & 1) * 4;
      if (lane == 0) rd[warp - 2] = part;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const float g0 = rd[0] + rd[1] + rd[2] + rd[3];
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(mbf_ready);
      return g0;
    };
    float g0 = take_states(0);
    for (int c = 0; c < nch; ++c) {
      const int s = c % NST, n = nvalid(c);
      const uint8_t* st = smem + s * STAGE;
      // (d) A = bf16(S1 o S2), token-major (rows j, columns s)
      if (!dead) dead = !mbar_wait(sc_full, c & 1, lim);
      tc_fence_after();
      {
        uint32_t a[32], b[32];
        tmem_ld_half32(t_s1 + lane_off, a);
        tmem_ld_half32(t_s2 + lane_off, b);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int x = 8 * q + 2 * h;
            w[h] = pack_bf16x2(__uint_as_float(a[x]) * __uint_as_float(b[x]),
                               __uint_as_float(a[x + 1]) * __uint_as_float(b[x + 1]));
          }
          st_shared_v4(sbase + Cfg::OFF_A + sw128_off(row64h, 4 * half + q), w[0], w[1], w[2], w[3]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(a_ready);
      // (e) y_j = do_j . (M q_j) over this block's rows of M (Y landed with S1)
      float y, z;
      {
        uint32_t r[32];
        tmem_ld_half32(t_yz + lane_off, r);
        tmem_ld_wait();
        y = row_dot(st + Cfg::OFF_SD + rb * C * 128, r);
      }
      tc_fence_before();
      mbar_arrive(y_free);
      // (f) z_s = v_s . (G k_s)
      if (!dead) dead = !mbar_wait(z_full, c & 1, lim);
      tc_fence_after();
      {
        uint32_t r[32];
        tmem_ld_half32(t_yz + lane_off, r);
        tmem_ld_wait();
        z = row_dot(st + Cfg::OFF_SV + rb * C * 128, r);
      }
      tc_fence_before();
      mbar_arrive(&empty[s]);  // done with this stage's V and dO rows
      // hand y, z and <G, M> of chunk c to warps 7-10 (slot c & 1, free once
      // they are done with chunk c - 2), then take chunk c+1's states
      if (c >= 2 && !dead) dead = !mbar_wait(&yz_free[c & 1], ((c >> 1) - 1) & 1, lim);
      if (half == 0) {
        ybuf[(c & 1) * C + row64h] = y;
        zbuf[(c & 1) * C + row64h] = z;
      }
      if (threadIdx.x == 64) g0buf[c & 1] = g0;
      mbar_arrive(&yz_ready[c & 1]);
      const float g0_next = (c + 1 < nch) ? take_states(c + 1) : 0.f;
      g0 = g0_next;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::TCOLS);
}

// ------------------------------------------------------------ dL/dW_0 ----
// dL/dW_0 = dL/dW_T + sum_t do_t q_t^T: the recurrence of dL/dW does not
// involve the momentum.  Computed on its own, the deta kernel, which starts
// from it, need not wait for the reverse kernel that also carries it.
// Block (b, h, split) sums its share of the 64-token tiles into a TMEM
// accumulator, acc += do_tile^T q_tile (both operands MN-major, M = N = d),
// and writes the fp32 partial; mom_g0_sum_kernel adds the partials to
// dL/dW_T in a fixed order, so the result is the same bits on every run.
struct MomG0Params {
  int BH, T, nsplit, tiles_per_split;
  float* part;  // [nsplit][BH][d][d]
  uint64_t limit_ns;
};

template <int D>
struct MomG0Cfg {
  static constexpr int C = 64;
  static constexpr int TILE = C * D * 2;  // one bf16 64-token tile
  static constexpr int NST = 4;
  static constexpr int STAGE = 2 * TILE;  // do, then q
  static constexpr int SMEM = NST * STAGE + 256 + 1024;  // + barriers, alignment slack
  static constexpr int THREADS = 192;     // TMA, MMA, four readout warps
};

template <int D>
__global__ void __launch_bounds__(192, 1) mom_g0_kernel(const __grid_constant__ CUtensorMap tmD,
                                                        const __grid_constant__ CUtensorMap tmQ,
                                                        const MomG0Params p) {
  using Cfg = MomG0Cfg<D>;
  constexpr int C = Cfg::C, TILE = Cfg::TILE, NST = Cfg::NST, STAGE = Cfg::STAGE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NST * STAGE);  // [NST] tiles landed
  uint64_t* empty = full + NST;                                       // [NST] tiles consumed
  uint64_t* done = empty + NST;                                       // every MMA complete
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.limit_ns;
  const int bh = blockIdx.x / p.nsplit, split = blockIdx.x % p.nsplit;
  const int t_begin = split * p.tiles_per_split;
  const int n = max(0, min(p.tiles_per_split, (p.T + C - 1) / C - t_begin));

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, D);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmD);
    prefetch_tmap(&tmQ);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      bool dead = false;
      for (int i = 0; i < n; ++i) {
        const int s = i % NST;
        if (i >= NST && !dead) dead = !mbar_wait(&empty[s], ((i / NST) - 1) & 1, lim);
        mbar_arrive_expect_tx(&full[s], 2 * TILE);
        uint8_t* st = smem + s * STAGE;
        const int t0 = (t_begin + i) * C;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_load_3d(&tmD, &full[s], st + kb * C * 128, kb * 64, t0, bh);
          tma_load_3d(&tmQ, &full[s], st + TILE + kb * C * 128, kb * 64, t0, bh);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool dead = false;
      constexpr uint32_t ID = idesc_bf16_f32(D, D, true, true);
      for (int i = 0; i < n; ++i) {
        const int s = i % NST;
        if (!dead) dead = !mbar_wait(&full[s], (i / NST) & 1, lim);
        tc_fence_after();
        const uint32_t st = sbase + s * STAGE;
        const uint64_t da = sdesc_sw128(st, C * 128, 1024), db = sdesc_sw128(st + TILE, C * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          mma_bf16_ss(tacc, da + mn_step(kk), db + mn_step(kk), ID, (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(done);  // with no tile, arrives at once
    }
  } else {
    // readout: row d of the accumulator (an M = 64 accumulator fills lanes
    // 0-15 of each quadrant), written as this split's fp32 partial
    const int g4 = warp & 3;
    const bool ok = (D == 128) || lane < 16;
    const int row = (D == 128) ? 32 * g4 + lane : ok ? 16 * g4 + lane : 0;  // (lanes 16-31 idle at d = 64)
    bool dead = false;
    if (!dead) dead = !mbar_wait(done, 0, lim);
    tc_fence_after();
    const size_t DD = static_cast<size_t>(D) * D;
    float* dst = TTT_AT(p.part, (static_cast<size_t>(split) * p.BH + bh) * DD + static_cast<size_t>(row) * D, D,
                        static_cast<size_t>(p.nsplit) * p.BH * DD);
#pragma unroll
    for (int cb = 0; cb < D / 32; ++cb) {
      uint32_t r[32];
      tmem_ld32(tacc + (static_cast<uint32_t>(32 * g4) << 16) + cb * 32, r);
      tmem_ld_wait();
      if (ok) {
        float4* d4 = reinterpret_cast<float4*>(dst + cb * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          d4[j] = (n > 0) ? make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tacc, D);
}

// g0 = dL/dW_T (or zero) + the nsplit partials, in split order.
__global__ void mom_g0_sum_kernel(const float* GT, const float* part, int nsplit, long long n, float* g0) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float acc = GT ? GT[i] : 0.f;
    for (int s = 0; s < nsplit; ++s) acc += part[static_cast<long long>(s) * n + i];
    g0[i] = acc;
  }
}

}  // namespace ttt
