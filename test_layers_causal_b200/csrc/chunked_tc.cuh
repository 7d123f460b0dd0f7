// chunked_tc.cuh -- chunk-parallel forward of the TTT layer on the sm_100a
// tensor cores (tcgen05 + TMEM, operands staged by TMA), bf16 in, fp32
// accumulate, no momentum.
//
// The layer, written as learned linear attention (kualia.ai explainer
// "Test Time Training as Linear Attention", section "The Linear Attention
// Equivalence"; "fully parallel formulations" in the abstract of "Test-Time
// Training with KV Binding Is Secretly Linear Attention"): per (b, h) and for a
// chunk of C tokens with local indices i, j, with K~ = diag(sigma * eta) K,
//   O_c = tril(Q_c K~_c^T) V_c + Q_c W^T        (update-then-read: j <= i)
//   W  <- W + V_c^T K~_c
// where W (d_v x d_k, fp32) is the fast weight carried in from earlier chunks.
//
// One launch per forward.  A (b, h) sequence is cut into `nseg` segments of
// whole chunks so that B*H*nseg blocks fill the SMs in one wave.  A block
// takes its tile (segment, head) from an atomic counter; then
//   phase A (all but the last segment): dW_p = sum over the segment of
//           V^T K~ in one TMEM accumulator (chunks taken last to first),
//           published as fp32 with a flag;
//   start:   W_start(p) = W_0 + sum_{p' < p} dW_p', either by a decoupled
//           look-back (segment p sums the totals after the nearest
//           predecessor that has published its own start + total; tiles
//           are taken in segment order, so it never waits for a block that
//           has not started) or, when that would read many totals and the
//           grid is one wave, by a cooperative prefix (the head's blocks
//           each sum one slice of the state over all totals, then meet at a
//           counter);
//   phase B: the chunk loop above from W_start(p); its first K and V tiles
//           are the ones phase A read last (the likeliest to hit in L2).
//
// Block = 8 warps: warp 0 issues TMA loads, warp 1 owns TMEM and issues the
// MMAs (one thread, descriptors precomputed), warps 2-5 (128 threads, one
// TMEM lane each) mask scores, convert fp32 accumulators into bf16 operands
// and stage O, warp 6 stores O with TMA, warp 7 scales every K tile by the
// learning rate as it lands (fetching eta two chunks ahead).  Per phase-B
// chunk the MMA thread issues
//   (1) Sc    = Q K~^T              [TMEM, M=C,   N=C]
//   (2) O[b]  = Q Wbf^T             [TMEM, M=C,   N=d_v]   Wbf = bf16(W) in smem
//   (3) W    += V^T K~              [TMEM, M=d_v, N=d_k]   (after Wbf was taken)
//   (4) O[b] += P V                 P = bf16(masked Sc) in smem
// O is double-buffered in TMEM (b = chunk parity) so that chunk c+1's (2)-(3)
// overlap the read-out of chunk c.  P is written over the Q (and K) slots once
// (1)-(3) have read them and O is staged in the V slot once (4) has read it,
// so one stage holds just Q, K, V.  Every wait is bounded (common.cuh); a
// thread whose wait runs out stops waiting but keeps arriving, so the block
// always drains and exits.
#pragma once
#include "common.cuh"

namespace ttt {

struct TcParams {
  int BH, T, nchunks, cps, nseg;  // cps = chunks per segment
  const float* eta;               // [BH, T] or nullptr
  float eta_const, sigma;
  const float* S_in;              // [BH, dv, dk] initial state or nullptr
  float* ws;                      // [BH, nseg, 2, dv, dk]: segment totals, segment start states
  unsigned* flags;                // [BH * nseg] flags, tile counter, [BH] head counters (zeroed per call)
  int coop;                       // 1: cooperative prefix (one wave), 0: decoupled look-back
  float* S_out;                   // [BH, dv, dk] final state or nullptr
  uint64_t limit_ns;
};

template <int C, int D>
struct TcCfg {
  static constexpr int TILE = C * D * 2;                     // bytes of one bf16 C x D tile
  // 64 x 64 tiles fuse (1) and (2) into one N = C + D MMA, [Sc | O] = Q [K~; Wbf]^T:
  // the K region of a stage then holds K~ and that chunk's Wbf as adjacent rows
  // of one operand (order alternating with the chunk's parity, see below).
  static constexpr bool MRG = (C == 64 && D == 64);
  static constexpr int KWR = MRG ? C + D : C;                // rows per 64-column block of the K region
  static constexpr int KREG = KWR * D * 2;
  static constexpr int OK = TILE, OV = TILE + KREG;          // Q at 0, K region, V
  static constexpr int STAGE = 2 * TILE + KREG;
  static constexpr int NST = (C == 128 && D == 128) ? 2 : 3;
  static constexpr int SBF = MRG ? 0 : D * D * 2;            // bf16 copy of W (B operand)
  // P gets its own buffer, written as soon as the scores land, except for the
  // 128 x 128 tile, where it reuses the Q/K slots once (1)-(3) have read them.
  static constexpr bool PSEP = !(C == 128 && D == 128);
  static constexpr int PBUF = PSEP ? C * C * 2 : 0;
  static constexpr int BIG = NST * STAGE + SBF + PBUF;
  static constexpr int NBAR = 4 * NST + 10;
  static constexpr int SMALL = NBAR * 8 + NST * C * 4 + 32;
  static constexpr int SMEM = BIG + SMALL + 1024;            // + alignment slack
  static constexpr int TCOLS_USED = C + 3 * D;               // W, scores, O x 2
  static constexpr int TCOLS = TCOLS_USED <= 256 ? 256 : 512;
  static constexpr int MINB = (C == 64 && D == 64) ? 2 : 1;  // blocks per SM
  static_assert(C == 64 || C == 128, "chunk");
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(C <= 2 * D, "P must fit in the Q and K slots");
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(TCOLS_USED <= 512, "tensor memory");
};

// K-major operand (rows x 64-element k-blocks, SW128): descriptor of the
// 16-wide k-step kk.
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int rows, int kk) {
  return sdesc_sw128(base + static_cast<uint32_t>((kk >> 2) * rows * 128 + (kk & 3) * 32), 16, 1024);
}
// MN-major operand stored token-major ([C tokens][64-col blocks], SW128),
// contracted over tokens: descriptor of the 16-token step kk.
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int C, int kk) {
  return sdesc_sw128(base + static_cast<uint32_t>(kk * 2048), static_cast<uint32_t>(C * 128), 1024);
}

// Offset (in the descriptor's 16-byte address units) of the MN-major step kk.
__host__ __device__ constexpr uint64_t mn_step(int kk) { return static_cast<uint64_t>(kk * 2048 >> 4); }

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Waits until *p >= target (bounded); returns the value seen, 0 on timeout.
// A slow path, kept out of line so that it costs the callers no registers.
__device__ __noinline__ unsigned wait_geq(const unsigned* p, unsigned target, uint64_t limit_ns) {
  unsigned v = ld_acquire(p);
  if (v >= target) return v;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(64);
    v = ld_acquire(p);
    if (v >= target) return v;
    if (globaltimer_ns() - t0 > limit_ns) {
      record_timeout();
      return 0;
    }
  }
}


// Packs 32 fp32 values (as raw bits) into bf16 and writes them as four
// 16-byte units of row `row` of a 128B-swizzled K-major tile (shared address
// `tile`) whose 64-column blocks are `blk` bytes apart, starting at column
// `col0` (multiple of 32).
__device__ __forceinline__ void store_row32_bf16(uint32_t tile, int blk, int row, int col0, const uint32_t (&r)[32]) {
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const int col = col0 + q4 * 8;
    st_shared_v4(tile + (col >> 6) * blk + sw128_off(row, (col & 63) >> 3),
                 pack_bf16x2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1])),
                 pack_bf16x2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3])),
                 pack_bf16x2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5])),
                 pack_bf16x2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7])));
  }
}
__device__ __forceinline__ void store_row32_bf16(uint8_t* tile, int blk, int row, int col0, const uint32_t (&r)[32]) {
  store_row32_bf16(smem_u32(tile), blk, row, col0, r);
}

// Same for 64 values starting at column `col0` (multiple of 64): one
// 128-byte row of one 64-column block.
__device__ __forceinline__ void store_row64_bf16(uint32_t tile, int blk, int row, int col0, const uint32_t (&r)[64]) {
#pragma unroll
  for (int q8 = 0; q8 < 8; ++q8)
    st_shared_v4(tile + (col0 >> 6) * blk + sw128_off(row, q8),
                 pack_bf16x2(__uint_as_float(r[q8 * 8 + 0]), __uint_as_float(r[q8 * 8 + 1])),
                 pack_bf16x2(__uint_as_float(r[q8 * 8 + 2]), __uint_as_float(r[q8 * 8 + 3])),
                 pack_bf16x2(__uint_as_float(r[q8 * 8 + 4]), __uint_as_float(r[q8 * 8 + 5])),
                 pack_bf16x2(__uint_as_float(r[q8 * 8 + 6]), __uint_as_float(r[q8 * 8 + 7])));
}
__device__ __forceinline__ void store_row64_bf16(uint8_t* tile, int blk, int row, int col0, const uint32_t (&r)[64]) {
  store_row64_bf16(smem_u32(tile), blk, row, col0, r);
}

template <int C, int D>
__global__ void __launch_bounds__(256, TcCfg<C, D>::MINB)
    chunked_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                      const TcParams p) {
  using Cfg = TcCfg<C, D>;
  constexpr int NST = Cfg::NST, TILE = Cfg::TILE, STAGE = Cfg::STAGE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BIG);
  uint64_t* full = bars;                // [NST] TMA landed
  uint64_t* kready = bars + NST;        // [NST] K scaled by the scaler warp
  uint64_t* empty = bars + 2 * NST;     // [NST] stage free
  uint64_t* staged = bars + 3 * NST;    // [NST] O of phase-B chunk it staged (index it % NST)
  uint64_t* sc_full = bars + 4 * NST;   // scores in TMEM
  uint64_t* sdone = sc_full + 1;        // (2),(3) done / phase-A total done
  uint64_t* wbf_ready = sc_full + 2;    // Wbf written
  uint64_t* p_ready = sc_full + 3;      // P written
  uint64_t* o_full = sc_full + 4;       // [2] O[b] complete in TMEM
  uint64_t* o_free = sc_full + 6;       // [2] O[b] read out of TMEM
  uint64_t* drain = sc_full + 8;        // final MMA drain
  float* es = reinterpret_cast<float*>(smem + Cfg::BIG + Cfg::NBAR * 8);  // [NST][C] sigma*eta
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(es + NST * C);
  int* sh_tile = reinterpret_cast<int*>(tmem_holder + 1);
  int* sh_lb = sh_tile + 1;             // decoupled look-back: [1] nearest inclusive predecessor or -1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&kready[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&staged[s], 128);
    }
    mbar_init(sc_full, 1);
    mbar_init(sdone, 1);
    mbar_init(wbf_ready, 128);
    mbar_init(p_ready, 128);
    mbar_init(&o_full[0], 1);
    mbar_init(&o_full[1], 1);
    mbar_init(&o_free[0], 128);
    mbar_init(&o_free[1], 128);
    mbar_init(drain, 1);
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
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The tile is taken only once this block holds its tensor memory, so a block
  // that others may wait for never waits for tensor memory itself.
  if (threadIdx.x == 0)
    *sh_tile = p.flags ? static_cast<int>(atomicAdd(p.flags + p.BH * p.nseg, 1u)) : static_cast<int>(blockIdx.x);
  __syncthreads();
  const uint32_t tmem = *tmem_holder;
  const int tile = *sh_tile;
  const int seg = tile / p.BH, bh = tile % p.BH;  // segment-major: predecessors have smaller tiles
  const int chunk0 = seg * p.cps;
  const int nch = min(p.cps, p.nchunks - chunk0);
  const int nA = (p.nseg > 1 && seg < p.nseg - 1) ? nch : 0;  // phase-A chunks
  const int nB = nch;
  const int NI = nA + nB;
  // Row offsets inside the K region (merged tiles): even phase-B chunks hold
  // [K~ ; Wbf], odd ones [Wbf ; K~], so that the fused MMA writes [Sc | O0] or
  // [O1 | Sc] and O stays double-buffered around one score region in TMEM.
  // Phase A walks its chunks last to first, so the K/V tiles phase B starts
  // with are the ones read most recently.
  auto chunk_of = [&](int g) { return g >= nA ? chunk0 + g - nA : chunk0 + nA - 1 - g; };
  auto krow_of = [&](int g) { return (Cfg::MRG && g >= nA && ((g - nA) & 1)) ? D : 0; };
  auto wrow_of = [&](int it) { return (it & 1) ? 0 : C; };
  // TMEM column map
  //   separate (1),(2): [W | Sc | O0 | O1]     merged: [W | O1 | Sc | O0]
  const uint32_t t_w = tmem;                                  // W: D columns, M = D
  const uint32_t t_sc = Cfg::MRG ? tmem + 2 * D : tmem + D;   // scores: C columns, M = C
  auto t_o_of = [&](int b) -> uint32_t {                      // O[b]: D columns, M = C
    return Cfg::MRG ? (b ? tmem + D : tmem + 2 * D + C) : tmem + D + C + b * D;
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      bool dead = false;
      // Every tile is loaded as evict-first: the only re-read (K and V of a
      // segment, phase A then phase B) gains nothing measurable from being
      // kept, and the streamed tiles then leave L2 to the state totals.
      const uint64_t pol_once = l2_policy_evict_first();
      for (int g = 0; g < NI; ++g) {
        const int s = g % NST;
        if (g >= NST && !dead) dead = !mbar_wait(&empty[s], ((g / NST) - 1) & 1, lim);
        const bool pb = g >= nA;
        const int t0 = chunk_of(g) * C;
        mbar_arrive_expect_tx(&full[s], pb ? 3 * TILE : 2 * TILE);
        uint8_t* st = smem + s * STAGE;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          if (pb) tma_load_3d_hint(&tmQ, &full[s], st + kb * C * 128, kb * 64, t0, bh, pol_once);
          tma_load_3d_hint(&tmK, &full[s], st + Cfg::OK + (kb * Cfg::KWR + krow_of(g)) * 128, kb * 64, t0, bh,
                           pol_once);
          tma_load_3d_hint(&tmV, &full[s], st + Cfg::OV + kb * C * 128, kb * 64, t0, bh, pol_once);
        }
      }
      for (int g = max(0, NI - NST); g < NI; ++g) mbar_wait(&full[g % NST], (g / NST) & 1, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      bool dead = false;
      constexpr uint32_t ID_SC = idesc_bf16_f32(C, C, false, false);
      constexpr uint32_t ID_O_QW = idesc_bf16_f32(C, D, false, false);
      constexpr uint32_t ID_W = idesc_bf16_f32(D, D, true, true);
      constexpr uint32_t ID_O_PV = idesc_bf16_f32(C, D, false, true);
      // Descriptors are built once per tile and advanced by constant offsets
      // (the start address is the low field; no carry leaves it below 256 KB).
      const uint64_t d_wbf = sdesc_sw128(sbase + NST * STAGE, 16, 1024);
      const uint64_t d_pbuf = sdesc_sw128(sbase + NST * STAGE + Cfg::SBF, 16, 1024);
      // phase A: segment total of V^T K~
      for (int g = 0; g < nA; ++g) {
        const int s = g % NST;
        const uint32_t stk = sbase + s * STAGE + Cfg::OK, stv = sbase + s * STAGE + Cfg::OV;
        const uint64_t dkm = sdesc_sw128(stk, Cfg::KWR * 128, 1024), dvm = sdesc_sw128(stv, C * 128, 1024);
        if (!dead) dead = !mbar_wait(&kready[s], (g / NST) & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          mma_bf16_ss(t_w, dvm + mn_step(kk), dkm + mn_step(kk), ID_W, (g > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      if (nA > 0) tc_commit(sdone);
      // phase B
      for (int it = 0; it < nB; ++it) {
        const int g = nA + it, s = g % NST, b = it & 1;
        const uint32_t stq = sbase + s * STAGE, stk = stq + Cfg::OK, stv = stq + Cfg::OV;
        const uint64_t dq = sdesc_sw128(stq, 16, 1024), dkk = sdesc_sw128(stk, 16, 1024);
        const uint64_t dkm = sdesc_sw128(stk + krow_of(g) * 128, Cfg::KWR * 128, 1024);
        const uint64_t dvm = sdesc_sw128(stv, C * 128, 1024);
        const uint64_t dp = Cfg::PSEP ? d_pbuf : dq;
        const uint32_t t_o = t_o_of(b);
        if (!dead) dead = !mbar_wait(&kready[s], (g / NST) & 1, lim);
        if (Cfg::MRG) {
          // [Sc | O] in one N = C + D MMA: needs this chunk's Wbf and a free O[b]
          if (!dead) dead = !mbar_wait(wbf_ready, it & 1, lim);
          if (it >= 2 && !dead) dead = !mbar_wait(&o_free[b], ((it - 2) >> 1) & 1, lim);
          tc_fence_after();
          constexpr uint32_t ID_SCO = idesc_bf16_f32(C, C + D, false, false);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(b ? t_o : t_sc, dq + k_step(C, kk), dkk + k_step(Cfg::KWR, kk), ID_SCO, kk > 0);
          tc_commit(sc_full);
        } else {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(t_sc, dq + k_step(C, kk), dkk + k_step(C, kk), ID_SC, kk > 0);
          tc_commit(sc_full);
          if (!dead) dead = !mbar_wait(wbf_ready, it & 1, lim);
          if (it >= 2 && !dead) dead = !mbar_wait(&o_free[b], ((it - 2) >> 1) & 1, lim);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(t_o, dq + k_step(C, kk), d_wbf + k_step(D, kk), ID_O_QW, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_w, dvm + mn_step(kk), dkm + mn_step(kk), ID_W, 1);
        tc_commit(sdone);
        if (!dead) dead = !mbar_wait(p_ready, it & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_o, dp + k_step(C, kk), dvm + mn_step(kk), ID_O_PV, 1);
        tc_commit(&o_full[b]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, lim);
    }
  } else if (warp == 6) {
    // ----------------------------------------------------- O store warp --
    if (lane == 0) {
      bool dead = false;
      for (int it = 0; it < nB; ++it) {
        const int g = nA + it, s = g % NST;
        if (!dead) dead = !mbar_wait(&staged[it % NST], (it / NST) & 1, lim);
        const uint8_t* sv = smem + s * STAGE + Cfg::OV;
        const int t0 = (chunk0 + it) * C;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) tma_store_3d(&tmO, sv + kb * C * 128, kb * 64, t0, bh);
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(&empty[s]);
      }
      bulk_wait0();
    }
  } else if (warp == 7) {
    // ------------------------------------------------------- K scaler --
    // K~ = diag(sigma * eta) K for every tile as it lands (phase A and B),
    // in place, swizzle-aware; eta is fetched two chunks ahead.
    bool dead = false;
    constexpr int RPL = C / 32;  // rows of a chunk whose eta this lane fetches
    const float* eg = p.eta ? p.eta + static_cast<size_t>(bh) * p.T : nullptr;
    auto fetch = [&](int g, float (&dst)[RPL]) {
      const int c0 = chunk_of(g) * C;
#pragma unroll
      for (int j = 0; j < RPL; ++j) {
        const int t = c0 + lane + 32 * j;
        dst[j] = (g < NI && t < p.T) ? (eg ? __ldg(eg + t) : p.eta_const) : 0.f;
      }
    };
    float er[RPL], en[RPL];
    fetch(0, er);
    fetch(1, en);
    constexpr int PER_LANE = C * (D / 8) / 32;  // 16-byte units of the K tile per lane
    constexpr int BATCH = 8;
    for (int g = 0; g < NI; ++g) {
      const int s = g % NST;
      float* ess = es + s * C;
#pragma unroll
      for (int j = 0; j < RPL; ++j) ess[lane + 32 * j] = p.sigma * er[j];
#pragma unroll
      for (int j = 0; j < RPL; ++j) er[j] = en[j];
      fetch(g + 2, en);
      __syncwarp();
      if (!dead) dead = !mbar_wait(&full[s], (g / NST) & 1, lim);
      uint8_t* sk = smem + s * STAGE + Cfg::OK + krow_of(g) * 128;
#pragma unroll 1
      for (int b0 = 0; b0 < PER_LANE; b0 += BATCH) {
        uint4 u[BATCH];
        uint32_t off[BATCH];
        float e[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const int idx = lane + 32 * (b0 + i);
          const int r = idx / (D / 8), cc = idx % (D / 8);
          off[i] = (cc >> 3) * Cfg::KWR * 128 + sw128_off(r, cc & 7);
          e[i] = ess[r];
          u[i] = *reinterpret_cast<const uint4*>(sk + off[i]);
        }
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          // packed bf16 multiply: eta_r is rounded to bf16 once, then each
          // product is rounded to bf16 as the operand itself would be
          const uint32_t e2 = pack_bf16x2(e[i], e[i]);
          u[i].x = mul_bf16x2(u[i].x, e2);
          u[i].y = mul_bf16x2(u[i].y, e2);
          u[i].z = mul_bf16x2(u[i].z, e2);
          u[i].w = mul_bf16x2(u[i].w, e2);
          *reinterpret_cast<uint4*>(sk + off[i]) = u[i];
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&kready[s]);
    }
  } else {
    // --------------------------------------------------------- epilogue --
    const int et = threadIdx.x - 64;               // 0..127
    const int g4 = warp & 3;                       // TMEM lane group of this warp
    const uint32_t lane_off = static_cast<uint32_t>(32 * g4) << 16;
    const int row128 = 32 * g4 + lane;
    const int row64 = 16 * g4 + lane;
    const bool ok64 = lane < 16;
    const int wrow = (D == 128) ? row128 : row64;  // W row (d_v index)
    const bool wrow_ok = (D == 128) || ok64;
    const int qrow = (C == 128) ? row128 : row64;  // query row of scores / O
    const bool qrow_ok = (C == 128) || ok64;
    // M = 64 tiles read with the whole warp: row 16*g4 + lane%16, column half lane/16
    const int row64h = 16 * g4 + (lane & 15), half = lane >> 4;
    bool dead = false;

    // --------------------------------------------- look-back, W_start
    {
      const size_t DD = static_cast<size_t>(D) * D;
      float* agg_me = p.ws ? p.ws + (static_cast<size_t>(bh) * p.nseg + seg) * 2 * DD : nullptr;
      unsigned* flag_me = p.flags ? p.flags + bh * p.nseg + seg : nullptr;
      if (nA > 0) {
        if (!dead) dead = !mbar_wait(sdone, 0, lim);
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t r[32];
          tmem_ld32(t_w + lane_off + cb * 32, r);
          tmem_ld_wait();
          if (wrow_ok) {
            float4* a4 = reinterpret_cast<float4*>(agg_me);  // quad-major
#pragma unroll
            for (int j = 0; j < 8; ++j)
              __stcg(a4 + qm4<D>(wrow, cb * 8 + j),
                     make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
          }
        }
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (et == 0) st_release(flag_me, 1u);
      }
      // W_start = W_0 + the totals of all earlier segments, in one of two ways.
      const float* base = p.S_in ? p.S_in + static_cast<size_t>(bh) * DD : nullptr;
      if (p.nseg > 1 && p.coop) {
        // Cooperative prefix: the grid is a single wave, so the nseg blocks
        // of a head are resident together.  Once every total is published,
        // block `seg` prefix-sums element slice `seg` over all segments
        // (coalesced) into the start-state slots; then the blocks meet at the
        // head's counter and each reads its own start state.
        for (int j = et; j < p.nseg - 1; j += 128)
          if (!dead && wait_geq(p.flags + bh * p.nseg + j, 1u, lim) == 0) dead = true;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const int DDi = D * D;
        const int SL = ((DDi + p.nseg - 1) / p.nseg + 31) / 32 * 32;  // slice, a multiple of 32
        const int v1 = min(DDi, (seg + 1) * SL) / 4;
        const int nagg = p.nseg - 1;
        float4* w4 = reinterpret_cast<float4*>(p.ws + static_cast<size_t>(bh) * p.nseg * 2 * DD);
        const size_t SEG4 = 2 * DD / 4;  // float4 stride between segments; start states at +DD/4
        const float4* s4 = reinterpret_cast<const float4*>(base);
        // two vectors per thread per round, four totals per round
        for (int v = seg * SL / 4 + et; v < v1; v += 256) {
          const bool two = v + 128 < v1;
          // the scratch is quad-major, the caller's W_0 row-major
          float4 run0 = s4 ? __ldcg(s4 + qm4_to_rm4<D>(v)) : make_float4(0.f, 0.f, 0.f, 0.f);
          float4 run1 = (s4 && two) ? __ldcg(s4 + qm4_to_rm4<D>(v + 128)) : make_float4(0.f, 0.f, 0.f, 0.f);
          for (int j = 0; j < nagg; j += 4) {
            float4 a0[4], a1[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (j + u < nagg) {
                a0[u] = __ldcg(w4 + (j + u) * SEG4 + v);
                if (two) a1[u] = __ldcg(w4 + (j + u) * SEG4 + v + 128);
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (j + u < nagg) {
                __stcg(w4 + (j + u) * SEG4 + DD / 4 + v, run0);
                run0 = f4_add(run0, a0[u]);
                if (two) {
                  __stcg(w4 + (j + u) * SEG4 + DD / 4 + v + 128, run1);
                  run1 = f4_add(run1, a1[u]);
                }
              }
            }
          }
          __stcg(w4 + nagg * SEG4 + DD / 4 + v, run0);
          if (two) __stcg(w4 + nagg * SEG4 + DD / 4 + v + 128, run1);
        }
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        unsigned* cnt = p.flags + p.BH * p.nseg + 1 + bh;
        if (et == 0) {
          atomicAdd(cnt, 1u);
          if (!dead && wait_geq(cnt, static_cast<unsigned>(p.nseg), lim) == 0) dead = true;
          __threadfence();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        base = p.ws + (static_cast<size_t>(bh) * p.nseg + seg) * 2 * DD + DD;
        // this thread's row of W_start; with d = 128 all loads are issued
        // before any store (one round trip), with d = 64 one 32-column block
        // per round (register budget of two blocks per SM)
        constexpr int G = (D == 128) ? D / 32 : 1;
#pragma unroll
        for (int cb0 = 0; cb0 < D / 32; cb0 += G) {
          float row[G * 32];
#pragma unroll
          for (int c = 0; c < G * 8; ++c) {
            const float4 x = wrow_ok ? __ldcg(reinterpret_cast<const float4*>(base) + qm4<D>(wrow, cb0 * 8 + c))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            row[4 * c] = x.x, row[4 * c + 1] = x.y, row[4 * c + 2] = x.z, row[4 * c + 3] = x.w;
          }
#pragma unroll
          for (int cb = 0; cb < G; ++cb) {
            uint32_t r[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(row[cb * 32 + j]);
            tmem_st32(t_w + lane_off + (cb0 + cb) * 32, r);  // W accumulator := W_start
            if (wrow_ok) {
              if (Cfg::MRG)
                store_row32_bf16(sbase + (nA % NST) * STAGE + Cfg::OK + wrow_of(0) * 128, Cfg::KWR * 128, wrow,
                                 (cb0 + cb) * 32, r);
              else
                store_row32_bf16(sbase + NST * STAGE, D * 128, wrow, (cb0 + cb) * 32, r);
            }
          }
        }
        tmem_st_wait();
      } else {
        // Decoupled look-back: every predecessor has published at least its
        // total; the nearest one that has also published its inclusive state
        // (start + total) cuts the sum short.  One thread per predecessor
        // reads the flags.
        int first = 0;
        bool base_qm = false;  // base is a published (quad-major) state, not the caller's W_0
        if (seg > 0) {
          if (et == 0) sh_lb[1] = -1;
          asm volatile("bar.sync 1, 128;" ::: "memory");
          for (int j = et; j < seg; j += 128) {
            const unsigned f = dead ? 1u : wait_geq(p.flags + bh * p.nseg + j, 1u, lim);
            if (f == 0) dead = true;
            if (f >= 2) atomicMax(&sh_lb[1], j);
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
          const int incl = sh_lb[1];
          if (incl >= 0) {
            base = p.ws + ((static_cast<size_t>(bh) * p.nseg + incl) * 2 + 1) * DD;
            base_qm = true;
          }
          first = incl + 1;
        }
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          float acc[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[j] = 0.f;
          if (wrow_ok) {
            if (base) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float8 x = base_qm ? ld_cg_f8_qm<D>(base, wrow, cb * 8 + 2 * j)
                                         : ld_cg_f8(base + static_cast<size_t>(wrow) * D + cb * 32 + 8 * j);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[8 * j + e] = x.v[e];
              }
            }
            // NR totals per round (4 x NR x 2 independent 16-byte loads in
            // flight; two for 64-wide rows, within their register budget)
            constexpr int NR = (D == 128) ? 4 : 2;
            int jj = first;
            for (; jj + NR <= seg; jj += NR) {
              float8 x[NR][4];
#pragma unroll
              for (int u = 0; u < NR; ++u) {
                const float* ag = p.ws + (static_cast<size_t>(bh) * p.nseg + jj + u) * 2 * DD;
#pragma unroll
                for (int j = 0; j < 4; ++j) x[u][j] = ld_cg_f8_qm<D>(ag, wrow, cb * 8 + 2 * j);
              }
#pragma unroll
              for (int u = 0; u < NR; ++u)
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                  for (int e = 0; e < 8; ++e) acc[8 * j + e] += x[u][j].v[e];
            }
            for (; jj < seg; ++jj) {
              const float* ag = p.ws + (static_cast<size_t>(bh) * p.nseg + jj) * 2 * DD;
              float8 x[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) x[j] = ld_cg_f8_qm<D>(ag, wrow, cb * 8 + 2 * j);
#pragma unroll
              for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[8 * j + e] += x[j].v[e];
            }
          }
          uint32_t r[32];
          if (nA > 0) {  // this segment's total is still in t_w: publish the inclusive state
            tmem_ld32(t_w + lane_off + cb * 32, r);
            tmem_ld_wait();
            if (wrow_ok) {
              float4* d4 = reinterpret_cast<float4*>(agg_me + DD);  // quad-major
#pragma unroll
              for (int j = 0; j < 8; ++j)
                __stcg(d4 + qm4<D>(wrow, cb * 8 + j),
                       make_float4(acc[4 * j] + __uint_as_float(r[4 * j]), acc[4 * j + 1] + __uint_as_float(r[4 * j + 1]),
                                   acc[4 * j + 2] + __uint_as_float(r[4 * j + 2]),
                                   acc[4 * j + 3] + __uint_as_float(r[4 * j + 3])));
            }
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(acc[j]);
          tmem_st32(t_w + lane_off + cb * 32, r);  // W accumulator := W_start
          if (wrow_ok) {
            if (Cfg::MRG)
              store_row32_bf16(sbase + (nA % NST) * STAGE + Cfg::OK + wrow_of(0) * 128, Cfg::KWR * 128, wrow, cb * 32, r);
            else
              store_row32_bf16(sbase + NST * STAGE, D * 128, wrow, cb * 32, r);
          }
        }
        tmem_st_wait();
        if (nA > 0) {
          __threadfence();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (et == 0) st_release(flag_me, 2u);
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(wbf_ready);
    }

    // ---------------------------------------------------------- phase B
    const int hasA = nA > 0 ? 1 : 0;
    for (int it = 0; it < nB; ++it) {
      const int g = nA + it, s = g % NST, b = it & 1;
      uint8_t* st = smem + s * STAGE;
      // P = bf16(tril(scores)) into the Q (and K) slots
      {
        if (!dead) dead = !mbar_wait(sc_full, it & 1, lim);
        tc_fence_after();
        if constexpr (C == 64) {
          // this thread's 32 columns (half) of row row64h, straight into the
          // separate P buffer (free since the previous tile's (4): o_full,
          // waited in the previous O step)
          static_assert(Cfg::PSEP, "64-token tiles keep P in its own buffer");
          uint32_t r[32];
          tmem_ld_half32(t_sc + lane_off, r);
          tmem_ld_wait();
          const uint32_t pdst = sbase + NST * STAGE + Cfg::SBF;
          const int jmax = row64h - 32 * half;  // last unmasked column of this half
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 8 * i + 2 * e;
              w[e] = pack_bf16x2((j <= jmax) ? __uint_as_float(r[j]) : 0.f,
                                 (j + 1 <= jmax) ? __uint_as_float(r[j + 1]) : 0.f);
            }
            st_shared_v4(pdst + sw128_off(row64h, 4 * half + i), w[0], w[1], w[2], w[3]);
          }
        } else {
          uint32_t pk[C / 2];
#pragma unroll
          for (int cb = 0; cb < C / 64; ++cb) {
            uint32_t r[64];
            tmem_ld64(t_sc + lane_off + cb * 64, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const int col = cb * 64 + j;
              const float a0 = (col <= qrow) ? __uint_as_float(r[j]) : 0.f;
              const float a1 = (col + 1 <= qrow) ? __uint_as_float(r[j + 1]) : 0.f;
              pk[col >> 1] = pack_bf16x2(a0, a1);
            }
          }
          // the overlaid P must wait until (1)-(3) have read the Q and K
          // slots; a separate P buffer only until (4) of the previous tile
          // (o_full, waited in the previous O step)
          uint8_t* pdst = Cfg::PSEP ? smem + NST * STAGE + Cfg::SBF : st;
          if (!Cfg::PSEP && !dead) dead = !mbar_wait(sdone, (hasA + it) & 1, lim);
          if (qrow_ok) {
#pragma unroll
            for (int c16 = 0; c16 < C / 8; ++c16) {
              uint4 u = make_uint4(pk[c16 * 4 + 0], pk[c16 * 4 + 1], pk[c16 * 4 + 2], pk[c16 * 4 + 3]);
              *reinterpret_cast<uint4*>(pdst + (c16 >> 3) * C * 128 + sw128_off(qrow, c16 & 7)) = u;
            }
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      // next chunk's Wbf (W after this chunk's (3)) while (4) runs
      if (it + 1 < nB) {
        if (Cfg::PSEP && !dead) dead = !mbar_wait(sdone, (hasA + it) & 1, lim);
        tc_fence_after();
        const uint32_t wdst =
            Cfg::MRG ? sbase + ((g + 1) % NST) * STAGE + Cfg::OK + wrow_of(it + 1) * 128 : sbase + NST * STAGE;
        const int wblk = Cfg::MRG ? Cfg::KWR * 128 : D * 128;
        if constexpr (D == 64) {
          uint32_t r[32];
          tmem_ld_half32(t_w + lane_off, r);
          tmem_ld_wait();
          store_row32_bf16(wdst, wblk, row64h, 32 * half, r);
        } else {
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            uint32_t r[64];
            tmem_ld64(t_w + lane_off + cb * 64, r);
            tmem_ld_wait();
            store_row64_bf16(wdst, wblk, wrow, cb * 64, r);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(wbf_ready);
      }
      // O[b]: TMEM -> bf16 -> V slot, then the store warp takes it
      {
        const uint32_t sv = sbase + s * STAGE + Cfg::OV;
        if (!dead) dead = !mbar_wait(&o_full[b], (it >> 1) & 1, lim);
        tc_fence_after();
        const uint32_t t_o = t_o_of(b);
        if constexpr (C == 64 && D == 64) {
          uint32_t r[32];
          tmem_ld_half32(t_o + lane_off, r);
          tmem_ld_wait();
          store_row32_bf16(sv, C * 128, row64h, 32 * half, r);
        } else if constexpr (C == 64) {
          uint32_t r[64];
          tmem_ld_half64(t_o + lane_off, r);
          tmem_ld_wait();
          store_row64_bf16(sv, C * 128, row64h, 64 * half, r);
        } else {
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            uint32_t r[64];
            tmem_ld64(t_o + lane_off + cb * 64, r);
            tmem_ld_wait();
            if (qrow_ok) store_row64_bf16(sv, C * 128, qrow, cb * 64, r);
          }
        }
        tc_fence_before();
        mbar_arrive(&o_free[b]);
        fence_async_smem();
        mbar_arrive(&staged[it % NST]);
      }
    }

    // final state of the sequence (last segment)
    if (seg == p.nseg - 1 && p.S_out != nullptr) {
      if (!dead) dead = !mbar_wait(sdone, (hasA + nB - 1) & 1, lim);
      tc_fence_after();
      float* dst = p.S_out + static_cast<size_t>(bh) * D * D;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t r[32];
        tmem_ld32(t_w + lane_off + cb * 32, r);
        tmem_ld_wait();
        if (wrow_ok) {
          float4* d4 = reinterpret_cast<float4*>(dst + static_cast<size_t>(wrow) * D + cb * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            d4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
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
