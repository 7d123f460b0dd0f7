// chunked_tc_mom.cuh -- chunk-parallel forward with SGD momentum on the sm_100a
// tensor cores (Variant 3 of Table 2 in the thelatestinai.com listing of
// "Test-Time Training with KV Binding Is Secretly Linear Attention": a single
// linear fast weight, per-token learning rate, momentum in SGD).
//
// The recurrence M_t = beta M_{t-1} - sigma v_t k_t^T, W_t = W_{t-1} - eta_t M_t,
// o_t = W_t q_t regroups exactly over a tile of C tokens (local i, j; n valid):
//   c_ij = sum_{r=j..i} eta_r beta^(r-j)                        (j <= i)
//   o_i  = W q_i - g_i M q_i + sigma sum_{j<=i} c_ij (q_i . k_j) v_j,  g_i = beta c_i0
//   W'   = W - g_{n-1} M + sigma sum_j c_{n-1,j} v_j k_j^T
//   M'   = beta^n M - sigma sum_j beta^(n-1-j) v_j k_j^T
// The coefficients come from the tile's suffix sums cl_j = c_{C-1,j} (a warp
// scan, no division): c_ij = cl_j - beta^(i+1-j) cl_{i+1}.  Unlike the
// factorisation beta^-j (P_i - P_{j-1}), whose cancellation grows like
// beta^-C, this one loses at most a factor ~1/(1-beta) for positive eta.
//
// Structure as in chunked_tc.cuh (one launch, segments, look-back), with the
// pair (W, M) as the carried state: a segment acts on it as the affine map
//   (W, M) -> (W - G M + dW, B M + dM),
// G = beta * (segment suffix coefficient at its first token), B = beta^L.
// Phase A walks the segment's tiles backwards so the suffix coefficients carry
// from tile to tile; the look-back composes the published maps.  Tiles are 64
// tokens (a 128-token request runs as two 64-token tiles: the same layer),
// which keeps the Q, K, V stages, the two scaled K tiles, Q~ = diag(-g) Q, P
// and (at d = 64) the bf16 copies of W and M within shared memory.
//
// Per phase-B tile the MMA thread issues
//   (1) Sc  = Q K^T                       [unscaled K]
//   (2) O   = Q Wbf^T + Q~ Mbf^T
//   (3) W  += V^T K1,  M += V^T K2        K1 = diag(sigma c_{n-1,.}) K, K2 = diag(-sigma beta^(n-1-.)) K
//                                         (one N = 2D MMA: W, M and K1, K2 are adjacent)
//   (4) O  += P V                         P = bf16(sigma c * Sc), masked
// after the epilogue has replaced W by W - g_{n-1} M and M by beta^n M in TMEM.
// At d = 128, (2) and (4) run transposed with M = d = 128:
//   (2) O^T  = Wbf Q^T + Mbf Q~^T          Wbf, Mbf: A operands in TMEM
//   (4) O^T += V^T P^T
// The bf16 copies of W and M then go from the state step into TMEM, not
// through shared memory, and the MMAs read only Q, Q~, V and P from shared
// memory (the 64-row form streams all of Wbf and Mbf, 64 KB, per tile for
// 64 output rows; the tensor core and the epilogue share that bandwidth).
// The epilogue reads O^T one output column per thread and writes it
// transposed into the staging tile.
#pragma once
#include "common.cuh"
#include "chunked_tc.cuh"

namespace ttt {

struct TcMomParams {
  int BH, T, nchunks, cps, nseg;
  const float* eta;
  float eta_const, sigma, beta;
  const float* S_in;   // [BH, dv, dk] or nullptr
  const float* M_in;   // [BH, dv, dk] or nullptr
  float* ws;           // [BH, nseg, 4, dv, dk]: dW, dM, then W, M inclusive (look-back) or at the start (prefix)
  float* wsc;          // [BH, nseg, 2]: G, B of each segment map
  unsigned* flags;     // [BH * nseg] flags, a tile counter, [BH] head counters
  int coop;            // 1: cooperative prefix (grid is one wave), 0: decoupled look-back
  float* S_out;
  float* M_out;
  uint64_t limit_ns;
  // Scratch bounds of the debug checks, from the sizes above (kept out of
  // the parameter struct, which stays at 120 bytes: at 136 the kernel
  // measured 10% slower).
  __device__ __forceinline__ size_t ws_floats_of(int D) const {
    return static_cast<size_t>(BH) * nseg * (4 * static_cast<size_t>(D) * D + 2);
  }
  __device__ __forceinline__ size_t flag_words_of() const { return static_cast<size_t>(BH) * nseg + 1 + BH; }
};

// D[tmem] (+)= A[tmem] * B[smem], kind::f16: A (M x K bf16) in tensor memory,
// row m at lane m, k pairs packed in 32-bit columns (K = 16: 8 columns).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns (thread i: lane base + i).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

template <int D>
struct TcMomCfg {
  static constexpr int C = 64;
  static constexpr int TILE = C * D * 2;         // bf16 C x D
  static constexpr int STAGE = 3 * TILE;         // Q, K, V
  static constexpr int NST = 2;
  static constexpr int SQ = D * D * 2;           // bf16 D x D
  static constexpr int OFF_WBF = NST * STAGE;
  static constexpr int OFF_MBF = OFF_WBF + SQ;
  static constexpr int OFF_K1 = OFF_MBF + SQ;
  static constexpr int OFF_K2 = OFF_K1 + TILE;
  static constexpr int OFF_QT = OFF_K2 + TILE;
  static constexpr int OFF_P = OFF_QT + TILE;
  static constexpr int BIG = OFF_P + C * C * 2;
  // Phase A streams only K and V, through NSA stages: the K/V slots of the
  // NST Q/K/V stages and two more in buffers that phase B needs only later
  // (the bf16 copies of W and M; Q~ and P for d = 64).
  static constexpr int NSA = NST + 2;
  static constexpr int KA2 = OFF_WBF;                      // K of phase-A stage NST (V at + TILE)
  static constexpr int KA3 = (D == 128) ? OFF_MBF : OFF_QT;  // K of phase-A stage NST + 1
  static_assert(KA2 + 2 * TILE <= KA3 && KA3 + 2 * TILE <= (D == 128 ? OFF_K1 : BIG), "phase-A stages");
  static constexpr int NBAR = 5 * NST + 16 + 2 * NSA + 4;
  static constexpr int SMALL = NBAR * 8 + (NST * (C + 1) + (C + 1) + 8 + 4 * C) * 4 + 32;
  static constexpr int SMEM = BIG + SMALL + 1024;
  // d = 128: O^T (M = d, C columns), bf16 copies of W and M as TMEM A
  // operands (D / 2 columns each); otherwise O with M = C (D columns)
  static constexpr bool TR = (D == 128);
  static constexpr int TCOLS_USED = TR ? 2 * D + 2 * C + D : C + 3 * D;  // W, M, O, scores (, Wbf, Mbf)
  static constexpr int TCOLS = TCOLS_USED <= 256 ? 256 : 512;
  static constexpr int MINB = 1;
  static constexpr int NSCW = 4;                 // K-scaling warps (7 and 8-10), 16 rows each
  static constexpr int THREADS = 32 * (7 + NSCW);
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(SMEM <= 232448, "shared memory");
};

template <int D>
__global__ void __launch_bounds__(TcMomCfg<D>::THREADS, TcMomCfg<D>::MINB)
    chunked_tc_mom_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                          const TcMomParams p) {
  using Cfg = TcMomCfg<D>;
  constexpr int C = Cfg::C, NST = Cfg::NST, TILE = Cfg::TILE, STAGE = Cfg::STAGE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BIG);
  // Phase-B stage s holds Q, K, V of tile it = s mod NST.  Its Q and K slots
  // are done once the readout (2) has run, its V slot only once O, staged
  // there, has been stored: two fill/free pairs, so the next tile's Q and K
  // can load while O is still leaving.
  uint64_t* full = bars;               // [NST] Q and K loaded
  uint64_t* empty = bars + NST;        // [NST] Q and K slots free
  uint64_t* staged = bars + 2 * NST;   // [NST] (indexed by phase-B tile % NST)
  uint64_t* fullV = bars + 3 * NST;    // [NST] V loaded
  uint64_t* emptyV = bars + 4 * NST;   // [NST] V slot free (O stored)
  uint64_t* kt_ready = bars + 5 * NST; // scaled K1/K2 (and the tile's cl) ready
  uint64_t* kt_free = kt_ready + 1;    // (3) of the previous tile done: K1/K2 buffers free
  uint64_t* sc_full = kt_ready + 2;
  uint64_t* sdone = kt_ready + 3;      // (2),(3) done / phase-A totals done
  uint64_t* wbf_ready = kt_ready + 4;  // Wbf, Mbf, Q~ written; W, M rewritten in TMEM
  uint64_t* p_ready = kt_ready + 5;
  uint64_t* o_full = kt_ready + 6;
  uint64_t* seg_ready = kt_ready + 7; // phase-A segment scalars G, B written
  uint64_t* drain = kt_ready + 8;
  uint64_t* cl_ready = kt_ready + 9;   // [NST] coefficients of phase-B tile `it` in cls[it % NST]
  uint64_t* cl_free = kt_ready + 11;   // [NST] the epilogue is done with cls[it % NST]
  uint64_t* o_free = kt_ready + 13;    // O of the previous tile read out of TMEM
  uint64_t* fullA = kt_ready + 14;     // [NSA] phase-A K/V stage loaded
  uint64_t* emptyA = fullA + Cfg::NSA; // [NSA] phase-A stage consumed
  // Phase A double-buffers K1/K2: tile g uses set g & 1, set 1 in the Q slots
  // of stages 0 and 1 (phase A loads no Q).
  uint64_t* ktA_ready = emptyA + Cfg::NSA;  // [2] set scaled
  uint64_t* ktA_free = ktA_ready + 2;       // [2] set consumed by its MMAs
  float* cls = reinterpret_cast<float*>(smem + Cfg::BIG + Cfg::NBAR * 8);  // [NST][C+1] tile suffix sums
  float* bp = cls + NST * (C + 1);                                          // beta^k, k = 0..C
  float* segsc = bp + (C + 1);                                              // [0] G, [1] B of this segment
  uint32_t* wpk = reinterpret_cast<uint32_t*>(segsc + 8);  // [2 tiles][K1, K2][C] bf16x2 row weights
  uint32_t* tmem_holder = wpk + 4 * C;
  int* sh_tile = reinterpret_cast<int*>(tmem_holder + 1);
  int* sh_lb = sh_tile + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&staged[s], 128);
      mbar_init(&fullV[s], 1);
      mbar_init(&emptyV[s], 1);
    }
    mbar_init(kt_ready, Cfg::NSCW);
    mbar_init(kt_free, 1);
    mbar_init(sc_full, 1);
    mbar_init(sdone, 1);
    mbar_init(wbf_ready, 128);
    mbar_init(p_ready, 128);
    mbar_init(o_full, 1);
    mbar_init(seg_ready, 1);
    mbar_init(drain, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&cl_ready[s], 1);
      mbar_init(&cl_free[s], 128);
    }
    mbar_init(o_free, 128);
    for (int k = 0; k < Cfg::NSA; ++k) {
      mbar_init(&fullA[k], 1);
      mbar_init(&emptyA[k], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ktA_ready[b], Cfg::NSCW);
      mbar_init(&ktA_free[b], 1);
    }
    fence_mbar_init();
    float b = 1.f;
    for (int k = 0; k <= C; ++k) {
      bp[k] = b;
      b *= p.beta;
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::TCOLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0)
    *sh_tile = p.flags ? static_cast<int>(atomicAdd(p.flags + p.BH * p.nseg, 1u)) : static_cast<int>(blockIdx.x);
  __syncthreads();
  const uint32_t tmem = *tmem_holder;
  const int tile = *sh_tile;
  const int seg = tile / p.BH, bh = tile % p.BH;
  const int chunk0 = seg * p.cps;
  const int nch = min(p.cps, p.nchunks - chunk0);
  const int nA = (p.nseg > 1 && seg < p.nseg - 1) ? nch : 0;
  const int nB = nch;
  const int NI = nA + nB;
  // tile of iteration g: phase A walks the segment backwards, phase B forwards
  auto tile_of = [&](int g) { return chunk0 + (g < nA ? nA - 1 - g : g - nA); };
  const uint32_t t_w = tmem;            // W: D columns, M = D
  const uint32_t t_m = tmem + D;        // M: D columns, M = D
  const uint32_t t_o = tmem + 2 * D;    // O: D columns, M = C (d = 128: O^T, C columns, M = D)
  const uint32_t t_sc = tmem + (Cfg::TR ? 2 * D + C : 3 * D);  // scores: C columns, M = C
  const uint32_t t_wbf = tmem + 2 * D + 2 * C;  // d = 128: bf16 W (A operand), D / 2 columns
  const uint32_t t_mbf = t_wbf + D / 2;         // d = 128: bf16 M
  uint8_t* wbf = smem + Cfg::OFF_WBF;
  uint8_t* mbf = smem + Cfg::OFF_MBF;
  uint8_t* k1s = smem + Cfg::OFF_K1;
  uint8_t* k2s = smem + Cfg::OFF_K2;
  uint8_t* qts = smem + Cfg::OFF_QT;
  constexpr int NSA = Cfg::NSA;
  auto ka_off = [&](int k) -> int {  // byte offset of phase-A stage k's K tile; V follows at + TILE
    return k < NST ? k * STAGE + TILE : (k == NST ? Cfg::KA2 : Cfg::KA3);
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      bool dead = false;
      for (int g = 0; g < NI; ++g) {
        const int t0 = tile_of(g) * C;
        if (g < nA) {
          const int k = g % NSA;
          if (g >= NSA && !dead) dead = !mbar_wait(&emptyA[k], ((g / NSA) - 1) & 1, lim);
          mbar_arrive_expect_tx(&fullA[k], 2 * TILE);
          uint8_t* kd = smem + ka_off(k);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb) {
            tma_load_3d(&tmK, &fullA[k], kd + kb * C * 128, kb * 64, t0, bh);
            tma_load_3d(&tmV, &fullA[k], kd + TILE + kb * C * 128, kb * 64, t0, bh);
          }
          continue;
        }
        const int it = g - nA, s = it % NST;
        uint8_t* st = smem + s * STAGE;
        if (it >= NST) {
          if (!dead) dead = !mbar_wait(&empty[s], ((it / NST) - 1) & 1, lim);
        } else if (nA > 0) {
          if (!dead) dead = !mbar_wait(sdone, 0, lim);  // phase A is done with every stage
        }
        mbar_arrive_expect_tx(&full[s], 2 * TILE);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_load_3d(&tmQ, &full[s], st + kb * C * 128, kb * 64, t0, bh);
          tma_load_3d(&tmK, &full[s], st + TILE + kb * C * 128, kb * 64, t0, bh);
        }
        if (it >= NST && !dead) dead = !mbar_wait(&emptyV[s], ((it / NST) - 1) & 1, lim);
        mbar_arrive_expect_tx(&fullV[s], TILE);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) tma_load_3d(&tmV, &fullV[s], st + 2 * TILE + kb * C * 128, kb * 64, t0, bh);
      }
      for (int it = max(0, nB - NST); it < nB; ++it) {
        mbar_wait(&full[it % NST], (it / NST) & 1, lim);
        mbar_wait(&fullV[it % NST], (it / NST) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      bool dead = false;
      constexpr uint32_t ID_SC = idesc_bf16_f32(C, C, false, false);
      constexpr uint32_t ID_O_K = idesc_bf16_f32(C, D, false, false);
      constexpr uint32_t ID_W = idesc_bf16_f32(D, D, true, true);
      // W and M adjacent in TMEM, K1 and K2 adjacent 64-column blocks in shared
      // memory: phase B's state update is one N = 2D MMA per step
      constexpr uint32_t ID_WM = idesc_bf16_f32(D, 2 * D, true, true);
      static_assert(Cfg::OFF_K2 == Cfg::OFF_K1 + TILE, "K1, K2 adjacent");
      constexpr uint32_t ID_O_PV = idesc_bf16_f32(C, D, false, true);
      constexpr uint32_t ID_OT = idesc_bf16_f32(D, C, false, false);     // O^T += Wbf Q^T (A in TMEM)
      constexpr uint32_t ID_OT_PV = idesc_bf16_f32(D, C, true, false);   // O^T += V^T P^T
      const uint64_t d_wbf = sdesc_sw128(sbase + Cfg::OFF_WBF, 16, 1024);
      const uint64_t d_mbf = sdesc_sw128(sbase + Cfg::OFF_MBF, 16, 1024);
      const uint64_t d_k1 = sdesc_sw128(sbase + Cfg::OFF_K1, C * 128, 1024);
      const uint64_t d_k2 = sdesc_sw128(sbase + Cfg::OFF_K2, C * 128, 1024);
      const uint64_t d_k1b = sdesc_sw128(sbase, C * 128, 1024);          // phase A, odd tiles
      const uint64_t d_k2b = sdesc_sw128(sbase + STAGE, C * 128, 1024);
      const uint64_t d_qt = sdesc_sw128(sbase + Cfg::OFF_QT, 16, 1024);
      const uint64_t d_p = sdesc_sw128(sbase + Cfg::OFF_P, 16, 1024);
      for (int g = 0; g < NI; ++g) {
        const int s = g < nA ? g % NSA : (g - nA) % NST;  // phase-A or phase-B stage
        const uint32_t stq = sbase + s * STAGE;
        const uint32_t stv = g < nA ? sbase + ka_off(s) + TILE : stq + 2 * TILE;
        const uint64_t dvm = sdesc_sw128(stv, C * 128, 1024);
        if (g < nA) {
          // segment totals: dW += V^T K1, dM += V^T K2 (fresh at g == 0)
          const int b = g & 1;
          if (!dead) dead = !mbar_wait(&ktA_ready[b], (g >> 1) & 1, lim);
          tc_fence_after();
          const uint64_t dk1 = b ? d_k1b : d_k1, dk2 = b ? d_k2b : d_k2;
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) {
            const uint32_t acc = (g > 0 || kk > 0) ? 1u : 0u;
            mma_bf16_ss(t_w, dvm + mn_step(kk), dk1 + mn_step(kk), ID_W, acc);
            mma_bf16_ss(t_m, dvm + mn_step(kk), dk2 + mn_step(kk), ID_W, acc);
          }
          tc_commit(&emptyA[s]);
          tc_commit(&ktA_free[b]);
          if (g == nA - 1) tc_commit(sdone);
          continue;
        }
        const int it = g - nA;
        const uint64_t dq = sdesc_sw128(stq, 16, 1024), dkk = sdesc_sw128(stq + TILE, 16, 1024);
        if (!dead) dead = !mbar_wait(&full[s], (it / NST) & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_bf16_ss(t_sc, dq + k_step(C, kk), dkk + k_step(C, kk), ID_SC, kk > 0);
        tc_commit(sc_full);
        if (!dead) dead = !mbar_wait(kt_ready, it & 1, lim);
        if (!dead) dead = !mbar_wait(wbf_ready, it & 1, lim);
        if (!dead) dead = !mbar_wait(&fullV[s], (it / NST) & 1, lim);
        tc_fence_after();
        // (3) first: it needs only this tile's K1/K2 and the rewritten W, M
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_w, dvm + mn_step(kk), d_k1 + mn_step(kk), ID_WM, 1);
        tc_commit(kt_free);
        // (2) overwrites O: the previous tile's O must have been read out
        if (it > 0 && !dead) dead = !mbar_wait(o_free, (it - 1) & 1, lim);
        tc_fence_after();
        if constexpr (Cfg::TR) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            mma_bf16_ts(t_o, t_wbf + 8 * kk, dq + k_step(C, kk), ID_OT, kk > 0);
            mma_bf16_ts(t_o, t_mbf + 8 * kk, d_qt + k_step(C, kk), ID_OT, 1);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            mma_bf16_ss(t_o, dq + k_step(C, kk), d_wbf + k_step(D, kk), ID_O_K, kk > 0);
            mma_bf16_ss(t_o, d_qt + k_step(C, kk), d_mbf + k_step(D, kk), ID_O_K, 1);
          }
        }
        tc_commit(sdone);
        tc_commit(&empty[s]);  // Q and K of this tile are read
        if (!dead) dead = !mbar_wait(p_ready, it & 1, lim);
        tc_fence_after();
        if constexpr (Cfg::TR) {
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_o, dvm + mn_step(kk), d_p + k_step(C, kk), ID_OT_PV, 1);
        } else {
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_o, d_p + k_step(C, kk), dvm + mn_step(kk), ID_O_PV, 1);
        }
        tc_commit(o_full);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, lim);
    }
  } else if (warp == 6) {
    // ----------------------------------------------------- O store warp --
    if (lane == 0) {
      bool dead = false;
      for (int it = 0; it < nB; ++it) {
        const int s = it % NST;
        if (!dead) dead = !mbar_wait(&staged[it % NST], (it / NST) & 1, lim);
        const uint8_t* sv = smem + s * STAGE + 2 * TILE;
        const int t0 = (chunk0 + it) * C;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) tma_store_3d(&tmO, sv + kb * C * 128, kb * 64, t0, bh);
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(&emptyV[s]);
      }
      bulk_wait0();
    }
  } else if (warp >= 7) {
    // ------------------- coefficients (warp 7) and K scaling (warps 7-10) --
    // Warp 7 scans the tile's learning rates and writes the row weights;
    // the four scaling warps then each scale 16 rows of K into K1 and K2.
    const int sw = warp - 7;
    bool dead = false;
    const float* eg = p.eta ? p.eta + static_cast<size_t>(bh) * p.T : nullptr;
    const float beta = p.beta, sigma = p.sigma;
    float R = 0.f, Bc = 1.f;  // phase A carries: suffix coefficient after this tile, beta^(tokens after it)
    // eta of rows 2*lane, 2*lane+1 of tile g (0 past the sequence end or past the last tile)
    auto fetch_eta = [&](int g, float& x0, float& x1) {
      x0 = x1 = 0.f;
      if (sw != 0 || g >= NI) return;
      const int ta = tile_of(g) * C + 2 * lane, tb = ta + 1;
      if (ta < p.T) x0 = eg ? __ldg(eg + ta) : p.eta_const;
      if (tb < p.T) x1 = eg ? __ldg(eg + tb) : p.eta_const;
    };
    float en0, en1;
    fetch_eta(0, en0, en1);
    for (int g = 0; g < NI; ++g) {
      const int t0 = tile_of(g) * C;
      uint32_t* wg = wpk + (g & 1) * 2 * C;  // this tile's weights (double-buffered)
      if (sw == 0) {
        // eta of rows 2*lane, 2*lane+1 of this tile (fetched one tile ahead)
        const float e0 = en0, e1 = en1;
        fetch_eta(g + 1, en0, en1);
        // suffix scan over the tile: value at row 2*lane given zero beyond the tile
        float a = e0 + beta * e1, m = beta * beta;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float ah = __shfl_down_sync(0xffffffffu, a, off);
          const float mh = __shfl_down_sync(0xffffffffu, m, off);
          if (lane + off < 32) {
            a = fmaf(m, ah, a);
            m *= mh;
          }
        }
        float an = __shfl_down_sync(0xffffffffu, a, 1);
        if (lane == 31) an = 0.f;
        const float cl0 = a, cl1 = fmaf(beta, an, e1);  // cl at rows 2*lane, 2*lane+1
        if (g >= nA) {
          // phase B: publish the tile's suffix sums for the epilogue, in slot
          // it % NST once the epilogue is done with that slot's previous tile
          const int it = g - nA;
          if (it >= NST && !dead) dead = !mbar_wait(&cl_free[it % NST], ((it / NST) - 1) & 1, lim);
          float* cl = cls + (it % NST) * (C + 1);
          cl[2 * lane] = cl0;
          cl[2 * lane + 1] = cl1;
          if (lane == 0) cl[C] = 0.f;
          __syncwarp();
          if (lane == 0) mbar_arrive(&cl_ready[it % NST]);
        }
        // per-row weights of the two scaled K tiles
        float w1a, w1b, w2a, w2b;
        if (g < nA) {
          w1a = sigma * fmaf(bp[C - 2 * lane], R, cl0);
          w1b = sigma * fmaf(bp[C - 2 * lane - 1], R, cl1);
          w2a = -sigma * bp[C - 1 - 2 * lane] * Bc;
          w2b = -sigma * bp[C - 2 - 2 * lane] * Bc;
          R = fmaf(bp[C], R, __shfl_sync(0xffffffffu, cl0, 0));
          Bc *= bp[C];
          if (g == nA - 1 && lane == 0) {
            segsc[0] = beta * R;  // G: beta * suffix coefficient at the segment's first token
            segsc[1] = Bc;        // B = beta^L
            mbar_arrive(seg_ready);
          }
        } else {
          const int n = min(C, p.T - t0);
          w1a = sigma * cl0;
          w1b = sigma * cl1;
          w2a = (2 * lane < n) ? -sigma * bp[n - 1 - 2 * lane] : 0.f;
          w2b = (2 * lane + 1 < n) ? -sigma * bp[n - 2 - 2 * lane] : 0.f;
        }
        // row weights as bf16 pairs (each product is then rounded to bf16 as
        // the operand itself would be)
        wg[2 * lane] = pack_bf16x2(w1a, w1a);
        wg[2 * lane + 1] = pack_bf16x2(w1b, w1b);
        wg[C + 2 * lane] = pack_bf16x2(w2a, w2a);
        wg[C + 2 * lane + 1] = pack_bf16x2(w2b, w2b);
      }
      // the weights are visible to the four scaling warps; a warp passes this
      // barrier for tile g only after finishing tile g-1, so the other
      // weight buffer is free for warp 7 to fill next
      asm volatile("bar.sync 2, %0;" ::"n"(32 * Cfg::NSCW) : "memory");
      const uint8_t* sk;
      if (g < nA) {
        const int k = g % NSA;
        if (!dead) dead = !mbar_wait(&fullA[k], (g / NSA) & 1, lim);
        sk = smem + ka_off(k);
      } else {
        const int it = g - nA;
        if (!dead) dead = !mbar_wait(&full[it % NST], (it / NST) & 1, lim);
        sk = smem + (it % NST) * STAGE + TILE;
      }
      uint8_t *d1 = k1s, *d2 = k2s;
      if (g < nA) {
        if (g & 1) d1 = smem, d2 = smem + STAGE;
        if (g >= 2 && !dead) dead = !mbar_wait(&ktA_free[g & 1], ((g >> 1) - 1) & 1, lim);
      } else {
        const int it = g - nA;
        if (it > 0) {
          if (!dead) dead = !mbar_wait(kt_free, (it - 1) & 1, lim);
        } else if (nA > 0) {
          if (!dead) dead = !mbar_wait(sdone, 0, lim);  // phase A is done with both sets
        }
      }
      // K1 = diag(w1) K, K2 = diag(w2) K for rows [16 sw, 16 sw + 16), packed bf16 multiplies
      constexpr int PER_LANE = 16 * (D / 8) / 32;
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i) {
        const int idx = lane + 32 * i;
        const int r = 16 * sw + idx / (D / 8), cc = idx % (D / 8);
        const uint32_t off = (cc >> 3) * C * 128 + sw128_off(r, cc & 7);
        const uint32_t f1 = wg[r], f2 = wg[C + r];
        const uint4 u = *reinterpret_cast<const uint4*>(sk + off);
        *reinterpret_cast<uint4*>(d1 + off) =
            make_uint4(mul_bf16x2(u.x, f1), mul_bf16x2(u.y, f1), mul_bf16x2(u.z, f1), mul_bf16x2(u.w, f1));
        *reinterpret_cast<uint4*>(d2 + off) =
            make_uint4(mul_bf16x2(u.x, f2), mul_bf16x2(u.y, f2), mul_bf16x2(u.z, f2), mul_bf16x2(u.w, f2));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(g < nA ? &ktA_ready[g & 1] : kt_ready);
    }
  } else {
    // --------------------------------------------------------- epilogue --
    const int et = threadIdx.x - 64;
    const int g4 = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * g4) << 16;
    const int row128 = 32 * g4 + lane;
    const int row64 = 16 * g4 + lane;
    const bool ok64 = lane < 16;
    const int wrow = (D == 128) ? row128 : row64;
    const bool wrow_ok = (D == 128) || ok64;
    // 64-row tiles read with the whole warp: row 16*g4 + lane%16, column half lane/16
    const int row64h = 16 * g4 + (lane & 15), half = lane >> 4;
    const float beta = p.beta, sigma = p.sigma;
    bool dead = false;
    const size_t DD = static_cast<size_t>(D) * D;

    // ---- phase A result and look-back
    {
      float* me = p.ws ? TTT_AT(p.ws, (static_cast<size_t>(bh) * p.nseg + seg) * 4 * DD, 4 * DD, p.ws_floats_of(D))
                       : nullptr;
      unsigned* flag_me = p.flags ? TTT_AT(p.flags, static_cast<size_t>(bh) * p.nseg + seg, 1, p.flag_words_of()) : nullptr;
      if (nA > 0) {
        if (!dead) dead = !mbar_wait(sdone, 0, lim);
        if (!dead) dead = !mbar_wait(seg_ready, 0, lim);
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t tq = q ? t_m : t_w;
#pragma unroll
          for (int cb = 0; cb < D / 32; ++cb) {
            uint32_t r[32];
            tmem_ld32(tq + lane_off + cb * 32, r);
            tmem_ld_wait();
            if (wrow_ok) {
              float4* d4 = reinterpret_cast<float4*>(me + q * DD);  // quad-major
#pragma unroll
              for (int j = 0; j < 8; ++j)
                __stcg(d4 + qm4<D>(wrow, cb * 8 + j),
                       make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                   __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
            }
          }
        }
        if (et == 0) {
          float* sc = TTT_AT(p.wsc, (static_cast<size_t>(bh) * p.nseg + seg) * 2, 2,
                             p.ws_floats_of(D) - static_cast<size_t>(p.BH) * p.nseg * 4 * DD);
          sc[0] = segsc[0];
          sc[1] = segsc[1];
        }
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (et == 0) st_release(flag_me, 1u);
      }
      const float *bw = nullptr, *bm = nullptr;
      int first = 0;
      bool base_qm = false;  // bw, bm are published (quad-major) states, not the caller's
      if (p.coop && p.nseg > 1) {
        // Cooperative prefix (the grid is one wave, so the head's nseg blocks
        // are resident together): once every segment map is published, block
        // `seg` runs element slice `seg` of (W, M) through all the maps in
        // order, coalesced, writing each segment's start state into its
        // slots 2 and 3; the blocks meet at the head's counter and each then
        // reads its own start state.
        for (int j = et; j < p.nseg - 1; j += 128)
          if (!dead && wait_geq(TTT_AT(p.flags, static_cast<size_t>(bh) * p.nseg + j, 1, p.flag_words_of()), 1u, lim) == 0)
            dead = true;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const int DDi = D * D;
        const int SL = ((DDi + p.nseg - 1) / p.nseg + 31) / 32 * 32;  // slice, a multiple of 32
        const int v1 = min(DDi, (seg + 1) * SL) / 4;
        const int nagg = p.nseg - 1;
        // segment j's four matrices (dW, dM, then W and M at its start)
        auto seg4 = [&](int j) {
          return reinterpret_cast<float4*>(
              TTT_AT(p.ws, (static_cast<size_t>(bh) * p.nseg + j) * 4 * DD, 4 * DD, p.ws_floats_of(D)));
        };
        const size_t Q4 = DD / 4;  // float4 stride between a segment's matrices
        const float* maps = TTT_AT(p.wsc, static_cast<size_t>(bh) * p.nseg * 2, 2 * p.nseg,
                                   p.ws_floats_of(D) - static_cast<size_t>(p.BH) * p.nseg * 4 * DD);
        const size_t nst = static_cast<size_t>(p.BH) * DD;
        const float4* sw4 = p.S_in ? reinterpret_cast<const float4*>(TTT_AT(p.S_in, bh * DD, DD, nst)) : nullptr;
        const float4* sm4 = p.M_in ? reinterpret_cast<const float4*>(TTT_AT(p.M_in, bh * DD, DD, nst)) : nullptr;
        TTT_EXPECT(v1 <= static_cast<int>(DD / 4));
        const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
        // two positions per thread per round, four maps per round
        for (int v0 = seg * SL / 4 + et; v0 < v1; v0 += 256) {
          const int vv[2] = {v0, v0 + 128};
          const bool ok[2] = {true, v0 + 128 < v1};
          float4 w[2], m[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {  // the scratch is quad-major, the caller's states row-major
            w[e] = (sw4 && ok[e]) ? __ldcg(sw4 + qm4_to_rm4<D>(vv[e])) : zero;
            m[e] = (sm4 && ok[e]) ? __ldcg(sm4 + qm4_to_rm4<D>(vv[e])) : zero;
          }
          for (int j = 0; j < nagg; j += 4) {
            float4 dw[2][4], dm[2][4];
            float G[4], B[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (j + u < nagg) {
                G[u] = __ldcg(maps + 2 * (j + u));
                B[u] = __ldcg(maps + 2 * (j + u) + 1);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  if (ok[e]) {
                    dw[e][u] = __ldcg(seg4(j + u) + vv[e]);
                    dm[e][u] = __ldcg(seg4(j + u) + Q4 + vv[e]);
                  }
                }
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (j + u < nagg) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  if (!ok[e]) continue;
                  __stcg(seg4(j + u) + 2 * Q4 + vv[e], w[e]);
                  __stcg(seg4(j + u) + 3 * Q4 + vv[e], m[e]);
                  // (W, M) -> (W - G M + dW, B M + dM)
                  const float4 a = w[e], b = m[e], x = dw[e][u], y = dm[e][u];
                  w[e] = make_float4(fmaf(-G[u], b.x, a.x) + x.x, fmaf(-G[u], b.y, a.y) + x.y,
                                     fmaf(-G[u], b.z, a.z) + x.z, fmaf(-G[u], b.w, a.w) + x.w);
                  m[e] = make_float4(fmaf(B[u], b.x, y.x), fmaf(B[u], b.y, y.y), fmaf(B[u], b.z, y.z),
                                     fmaf(B[u], b.w, y.w));
                }
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            if (!ok[e]) continue;
            __stcg(seg4(nagg) + 2 * Q4 + vv[e], w[e]);
            __stcg(seg4(nagg) + 3 * Q4 + vv[e], m[e]);
          }
        }
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        unsigned* cnt = TTT_AT(p.flags, static_cast<size_t>(p.BH) * p.nseg + 1 + bh, 1, p.flag_words_of());
        if (et == 0) {
          atomicAdd(cnt, 1u);
          if (!dead && wait_geq(cnt, static_cast<unsigned>(p.nseg), lim) == 0) dead = true;
          __threadfence();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        bw = TTT_AT(p.ws, ((static_cast<size_t>(bh) * p.nseg + seg) * 4 + 2) * DD, 2 * DD, p.ws_floats_of(D));
        bm = bw + DD;
        base_qm = true;
        first = seg;
      } else {
        // Decoupled look-back: every predecessor has published at least its
        // map; the nearest one that has also published its inclusive state
        // cuts the composition short.
        if (et == 0) sh_lb[1] = -1;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        for (int j = et; j < seg; j += 128) {
          const unsigned f =
              dead ? 1u : wait_geq(TTT_AT(p.flags, static_cast<size_t>(bh) * p.nseg + j, 1, p.flag_words_of()), 1u, lim);
          if (f == 0) dead = true;
          if (f >= 2) atomicMax(&sh_lb[1], j);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const int incl = sh_lb[1];
        first = incl + 1;
        if (incl >= 0) {
          bw = TTT_AT(p.ws, ((static_cast<size_t>(bh) * p.nseg + incl) * 4 + 2) * DD, 2 * DD, p.ws_floats_of(D));
          bm = bw + DD;
          base_qm = true;
        } else {
          if (p.S_in) bw = TTT_AT(p.S_in, bh * DD, DD, static_cast<size_t>(p.BH) * DD);
          if (p.M_in) bm = TTT_AT(p.M_in, bh * DD, DD, static_cast<size_t>(p.BH) * DD);
        }
      }
      const float Gme = (nA > 0) ? segsc[0] : 0.f, Bme = (nA > 0) ? segsc[1] : 1.f;
      // With few segments every block reads all its predecessors' totals (at
      // most a few maps); publishing inclusive states as well would double
      // the scratch writes, which cost more than the reads they save.
      const bool pub_incl = !p.coop && nA > 0 && p.nseg > 8;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        float w[32], mm[32];
        const size_t off = static_cast<size_t>(wrow) * D + cb * 32;
#pragma unroll
        for (int j = 0; j < 32; ++j) w[j] = mm[j] = 0.f;
        if (wrow_ok) {
          if (bw) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float8 x = base_qm ? ld_cg_f8_qm<D>(bw, wrow, cb * 8 + 2 * j) : ld_cg_f8(bw + off + 8 * j);
#pragma unroll
              for (int e = 0; e < 8; ++e) w[8 * j + e] = x.v[e];
            }
          }
          if (bm) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float8 x = base_qm ? ld_cg_f8_qm<D>(bm, wrow, cb * 8 + 2 * j) : ld_cg_f8(bm + off + 8 * j);
#pragma unroll
              for (int e = 0; e < 8; ++e) mm[8 * j + e] = x.v[e];
            }
          }
          // apply the published segment maps in order
          for (int jj = first; jj < seg; ++jj) {
            const float* dw = TTT_AT(p.ws, (static_cast<size_t>(bh) * p.nseg + jj) * 4 * DD, 2 * DD, p.ws_floats_of(D));
            const float* dm = dw + DD;
            const float* gb = TTT_AT(p.wsc, (static_cast<size_t>(bh) * p.nseg + jj) * 2, 2,
                                     p.ws_floats_of(D) - static_cast<size_t>(p.BH) * p.nseg * 4 * DD);
            const float G = __ldcg(gb), B = __ldcg(gb + 1);
            float8 xw[4], xm[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              xw[j] = ld_cg_f8_qm<D>(dw, wrow, cb * 8 + 2 * j);
              xm[j] = ld_cg_f8_qm<D>(dm, wrow, cb * 8 + 2 * j);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int c = 8 * j + e;
                w[c] = fmaf(-G, mm[c], w[c]) + xw[j].v[e];
                mm[c] = fmaf(B, mm[c], xm[j].v[e]);
              }
            }
          }
        }
        uint32_t r[32], r2[32];
        if (pub_incl) {  // inclusive state after this segment, from its totals in TMEM
          tmem_ld32(t_w + lane_off + cb * 32, r);
          tmem_ld32(t_m + lane_off + cb * 32, r2);
          tmem_ld_wait();
          if (wrow_ok) {
            float4* iw = reinterpret_cast<float4*>(me + 2 * DD);  // quad-major
            float4* im = reinterpret_cast<float4*>(me + 3 * DD);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              iw[qm4<D>(wrow, cb * 8 + j / 4)] = make_float4(fmaf(-Gme, mm[j], w[j]) + __uint_as_float(r[j]),
                                      fmaf(-Gme, mm[j + 1], w[j + 1]) + __uint_as_float(r[j + 1]),
                                      fmaf(-Gme, mm[j + 2], w[j + 2]) + __uint_as_float(r[j + 2]),
                                      fmaf(-Gme, mm[j + 3], w[j + 3]) + __uint_as_float(r[j + 3]));
              im[qm4<D>(wrow, cb * 8 + j / 4)] = make_float4(fmaf(Bme, mm[j], __uint_as_float(r2[j])),
                                      fmaf(Bme, mm[j + 1], __uint_as_float(r2[j + 1])),
                                      fmaf(Bme, mm[j + 2], __uint_as_float(r2[j + 2])),
                                      fmaf(Bme, mm[j + 3], __uint_as_float(r2[j + 3])));
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          r[j] = __float_as_uint(w[j]);
          r2[j] = __float_as_uint(mm[j]);
        }
        tmem_st32(t_w + lane_off + cb * 32, r);
        tmem_st32(t_m + lane_off + cb * 32, r2);
      }
      tmem_st_wait();
      if (pub_incl) {
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (et == 0) st_release(flag_me, 2u);
      }
      // look-back: count the blocks that are done reading W_0 and M_0, which
      // the last segment's W_T and M_T may overwrite (in place)
      if (!p.coop && p.nseg > 1 && seg < p.nseg - 1) {
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (et == 0) atomicAdd(TTT_AT(p.flags, static_cast<size_t>(p.BH) * p.nseg + 1 + bh, 1, p.flag_words_of()), 1u);
      }
    }

    // ---- phase B
    auto step_w = [&](int it) {
      const int s = it % NST;
      const int n = min(C, p.T - (chunk0 + it) * C);
      uint8_t* st = smem + s * STAGE;
      const float* cl = cls + (it % NST) * (C + 1);
      // Step W: Wbf, Mbf from the state entering this tile; W -= g_end M; M *= beta^n; Q~ = diag(-g) Q
      if (!dead) dead = !mbar_wait(&cl_ready[it % NST], (it / NST) & 1, lim);  // the tile's cl is in smem
      if (!dead) dead = !mbar_wait(&full[s], (it / NST) & 1, lim);  // its Q has landed
      if (it > 0 && !dead) dead = !mbar_wait(sdone, ((nA > 0 ? 1 : 0) + it - 1) & 1, lim);
      tc_fence_after();
      const float gend = beta * cl[0];
      const float bn = bp[n];
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t r[32], r2[32];
        tmem_ld32(t_w + lane_off + cb * 32, r);
        tmem_ld32(t_m + lane_off + cb * 32, r2);
        tmem_ld_wait();
        if constexpr (Cfg::TR) {
          // bf16 pairs along k: the A-operand layout of an M = 128 MMA (row = lane)
          uint32_t pw[16], pm[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            pw[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
            pm[j] = pack_bf16x2(__uint_as_float(r2[2 * j]), __uint_as_float(r2[2 * j + 1]));
          }
          tmem_st16(t_wbf + lane_off + cb * 16, pw);
          tmem_st16(t_mbf + lane_off + cb * 16, pm);
        } else if (wrow_ok) {
          store_row32_bf16(wbf, D * 128, wrow, cb * 32, r);
          store_row32_bf16(mbf, D * 128, wrow, cb * 32, r2);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float wv = __uint_as_float(r[j]), mv = __uint_as_float(r2[j]);
          r[j] = __float_as_uint(fmaf(-gend, mv, wv));
          r2[j] = __float_as_uint(bn * mv);
        }
        tmem_st32(t_w + lane_off + cb * 32, r);
        tmem_st32(t_m + lane_off + cb * 32, r2);
      }
      {
        // this thread's half of row row64h of Q~ = diag(-g) Q
        const float f = -beta * fmaf(-bp[row64h + 1], cl[row64h + 1], cl[0]);
        const uint32_t f2 = pack_bf16x2(f, f);
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
          const int cc = half * (D / 16) + i;
          const uint32_t off = (cc >> 3) * C * 128 + sw128_off(row64h, cc & 7);
          const uint4 u = *reinterpret_cast<const uint4*>(st + off);
          *reinterpret_cast<uint4*>(qts + off) =
              make_uint4(mul_bf16x2(u.x, f2), mul_bf16x2(u.y, f2), mul_bf16x2(u.z, f2), mul_bf16x2(u.w, f2));
        }
      }
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(wbf_ready);
    };
    auto step_p = [&](int it) {
      const float* cl = cls + (it % NST) * (C + 1);
      // Step P: P_ij = sigma * c_ij * Sc_ij for j <= i (this thread: half of row row64h)
      {
        if (!dead) dead = !mbar_wait(sc_full, it & 1, lim);
        tc_fence_after();
        uint32_t r[32];
        tmem_ld_half32(t_sc + lane_off, r);
        tmem_ld_wait();
        const float cnext = cl[row64h + 1];
        const uint32_t pdst = sbase + Cfg::OFF_P;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 8 * i + 2 * e, col = 32 * half + j;
            float a0 = 0.f, a1 = 0.f;
            if (col <= row64h) a0 = sigma * fmaf(-bp[row64h + 1 - col], cnext, cl[col]) * __uint_as_float(r[j]);
            if (col + 1 <= row64h)
              a1 = sigma * fmaf(-bp[row64h - col], cnext, cl[col + 1]) * __uint_as_float(r[j + 1]);
            w[e] = pack_bf16x2(a0, a1);
          }
          st_shared_v4(pdst + sw128_off(row64h, 4 * half + i), w[0], w[1], w[2], w[3]);
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(p_ready);
        mbar_arrive(&cl_free[it % NST]);  // last use of this tile's coefficients
      }
    };
    auto step_o = [&](int it) {
      // Step O (this thread: half of row row64h)
      {
        const uint32_t sv = sbase + (it % NST) * STAGE + 2 * TILE;
        if (!dead) dead = !mbar_wait(o_full, it & 1, lim);
        tc_fence_after();
        if constexpr (Cfg::TR) {
          // O^T: this thread holds output column d = row128 for the C tokens.
          // Lane pairs (d even, d + 1) swap halves so that each writes two
          // adjacent columns of one token: the even lane tokens 2m, the odd
          // lane tokens 2m + 1.
          uint32_t r[32], r2[32];
          tmem_ld32(t_o + lane_off, r);
          tmem_ld32(t_o + lane_off + 32, r2);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(o_free);
          const bool odd = lane & 1;
          const int de = row128 & ~1;
          const uint32_t cbase = sv + (de >> 6) * C * 128 + (de & 7) * 2;
          const uint32_t c16 = (de & 63) >> 3;
          auto put = [&](int m, uint32_t x0, uint32_t x1) {  // tokens 2m, 2m + 1 of column d
            const float a = __uint_as_float(x0), b = __uint_as_float(x1);
            const float got = __shfl_xor_sync(0xffffffffu, odd ? a : b, 1);
            st_shared_b32(cbase + sw128_off(2 * m + (odd ? 1 : 0), c16), odd ? pack_bf16x2(got, b) : pack_bf16x2(a, got));
          };
#pragma unroll
          for (int m = 0; m < 16; ++m) put(m, r[2 * m], r[2 * m + 1]);
#pragma unroll
          for (int m = 0; m < 16; ++m) put(16 + m, r2[2 * m], r2[2 * m + 1]);
        } else {
          uint32_t r[32];
          tmem_ld_half32(t_o + lane_off, r);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(o_free);
          store_row32_bf16(sv, C * 128, row64h, 32 * half, r);
        }
        fence_async_smem();
        mbar_arrive(&staged[it % NST]);
      }
    };
    // Order: the next tile's Step W as soon as this tile's readout is done
    // (it gates the next MMAs), then this tile's Step O (its readout frees
    // O in TMEM for the next (2)), then the next tile's Step P.
    if (nB > 0) {
      step_w(0);
      step_p(0);
    }
    for (int it = 0; it < nB; ++it) {
      if (it + 1 < nB) step_w(it + 1);
      step_o(it);
      if (it + 1 < nB) step_p(it + 1);
    }

    // final state (last segment)
    if (seg == p.nseg - 1 && (p.S_out != nullptr || p.M_out != nullptr)) {
      // look-back: W_T, M_T may overwrite W_0, M_0 (in place) once every
      // other block has its start state (the cooperative prefix has already
      // met at the same counter)
      if (!p.coop && p.nseg > 1 && et == 0 && !dead &&
          wait_geq(TTT_AT(p.flags, static_cast<size_t>(p.BH) * p.nseg + 1 + bh, 1, p.flag_words_of()),
                   static_cast<unsigned>(p.nseg - 1), lim) == 0)
        dead = true;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!dead) dead = !mbar_wait(sdone, ((nA > 0 ? 1 : 0) + nB - 1) & 1, lim);
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float* dst = q ? p.M_out : p.S_out;
        const uint32_t tq = q ? t_m : t_w;
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t r[32];
          tmem_ld32(tq + lane_off + cb * 32, r);
          tmem_ld_wait();
          if (dst && wrow_ok) {
            float4* d4 = reinterpret_cast<float4*>(TTT_AT(dst, bh * DD, DD, static_cast<size_t>(p.BH) * DD) +
                                                   static_cast<size_t>(wrow) * D + cb * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              d4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                  __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::TCOLS);
}

}  // namespace ttt
