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
// Sequence split.  A (b, h) sequence is cut into `nseg` segments of whole
// chunks so that B*H*nseg blocks fill the 148 SMs:
//   pass 1 (OUT = false, segments 0..nseg-2): dW_p = sum over the segment of
//          V^T K~ (one TMEM accumulator), written as fp32;
//   pass 2 (scan kernel): W_start(p) = W_0 + sum_{p' < p} dW_p';
//   pass 3 (OUT = true, every segment): the chunk loop above starting from
//          W_start(p); the last segment writes the final state.
//
// Block = 6 warps: warp 0 issues TMA loads, warp 1 owns TMEM and issues the
// MMAs (one thread), warps 2-5 (128 threads, one TMEM lane each) scale K by
// the learning rate, mask the scores, convert fp32 accumulators to bf16
// operands and stage O for the TMA store.  Per chunk the MMA thread issues
//   (1) Sc  = Q K~^T              [TMEM, M=C,   N=C]
//   (2) O   = Q Wbf^T             [TMEM, M=C,   N=d_v]   Wbf = bf16(W) in smem
//   (3) W  += V^T K~              [TMEM, M=d_v, N=d_k]   (after Wbf was taken)
//   (4) O  += P V                 P = bf16(masked Sc) in smem
// P is written over the Q (and K) slots once (2)-(3) have read them, and O is
// staged in the V slot once (4) has read it, so one stage holds Q, K, V only.
// Every wait is bounded (see common.cuh); a thread whose wait runs out stops
// waiting but keeps arriving, so the block always drains and exits.
#pragma once
#include "common.cuh"

namespace ttt {

struct TcParams {
  int BH, T, nchunks, cps, nseg;  // cps = chunks per segment
  const float* eta;               // [BH, T] or nullptr
  float eta_const, sigma;
  const float* S_in;              // [BH, dv, dk] initial state (nseg == 1) or nullptr
  float* ws;                      // [BH, nseg, dv, dk]: pass 1 writes dW_p, pass 2 turns it into W_start(p)
  float* S_out;                   // [BH, dv, dk] final state or nullptr
  uint64_t limit_ns;
};

template <int C, int D, bool OUT>
struct TcCfg {
  static constexpr int TILE = C * D * 2;                     // bytes of one bf16 C x D tile
  static constexpr int NT = OUT ? 3 : 2;                     // tiles per stage (Q,K,V or K,V)
  static constexpr int STAGE = NT * TILE;
  static constexpr int NST = OUT ? ((C == 128 && D == 128) ? 2 : (C == 64 && D == 64 ? 4 : 3))
                                 : (196608 / STAGE < 4 ? 196608 / STAGE : 4);
  static constexpr int SBF = OUT ? D * D * 2 : 0;            // bf16 copy of W (B operand)
  static constexpr int BIG = NST * STAGE + SBF;
  static constexpr int NBAR = 3 * NST + 8;
  static constexpr int SMALL = NBAR * 8 + NST * C * 4 + 16;
  static constexpr int SMEM = BIG + SMALL + 1024;            // + alignment slack
  // TMEM columns: scores C, O D, W D (pass 3); W D (pass 1)
  static constexpr int TCOLS_USED = OUT ? (C + 2 * D) : D;
  static constexpr int TCOLS = TCOLS_USED <= 32 ? 32 : TCOLS_USED <= 64 ? 64 : TCOLS_USED <= 128 ? 128
                               : TCOLS_USED <= 256 ? 256 : 512;
  static_assert(C == 64 || C == 128, "chunk");
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(C <= 2 * D, "P must fit in the Q and K slots");
  static_assert(SMEM <= 232448, "shared memory");
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

template <int C, int D, bool OUT>
__global__ void __launch_bounds__(192, 1)
    chunked_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                      const TcParams p) {
  using Cfg = TcCfg<C, D, OUT>;
  constexpr int NST = Cfg::NST, TILE = Cfg::TILE, STAGE = Cfg::STAGE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BIG);
  uint64_t* full = bars;               // [NST] TMA landed
  uint64_t* kready = bars + NST;       // [NST] K scaled by the epilogue
  uint64_t* empty = bars + 2 * NST;    // [NST] stage free
  uint64_t* sc_full = bars + 3 * NST;  // scores in TMEM
  uint64_t* sdone = sc_full + 1;       // (2),(3) done: Wbf and Q/K slots free, W updated
  uint64_t* wbf_ready = sc_full + 2;   // Wbf written
  uint64_t* p_ready = sc_full + 3;     // P written
  uint64_t* o_full = sc_full + 4;      // O complete in TMEM
  uint64_t* o_free = sc_full + 5;      // O read out of TMEM
  uint64_t* drain = sc_full + 6;       // final MMA drain
  float* es = reinterpret_cast<float*>(smem + Cfg::BIG + Cfg::NBAR * 8);  // [NST][C] sigma*eta
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(es + NST * C);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / (OUT ? p.nseg : (p.nseg - 1));
  const int seg = blockIdx.x % (OUT ? p.nseg : (p.nseg - 1));
  const int chunk0 = seg * p.cps;
  const int nch = min(p.cps, p.nchunks - chunk0);
  const uint64_t lim = p.limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&kready[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(sc_full, 1);
    mbar_init(sdone, 1);
    mbar_init(wbf_ready, 128);
    mbar_init(p_ready, 128);
    mbar_init(o_full, 1);
    mbar_init(o_free, 128);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::TCOLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    if (OUT) prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (OUT) prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // TMEM column map
  const uint32_t t_w = tmem;                    // W accumulator: D columns, M = D
  const uint32_t t_sc = tmem + D;               // scores: C columns, M = C (pass 3)
  const uint32_t t_o = tmem + D + C;            // O: D columns, M = C (pass 3)

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      bool dead = false;
      for (int it = 0; it < nch; ++it) {
        const int s = it % NST;
        if (it >= NST && !dead) dead = !mbar_wait(&empty[s], ((it / NST) - 1) & 1, lim);
        mbar_arrive_expect_tx(&full[s], STAGE);
        const int t0 = (chunk0 + it) * C;
        uint8_t* st = smem + s * STAGE;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          if (OUT) tma_load_3d(&tmQ, &full[s], st + kb * C * 128, kb * 64, t0, bh);
          tma_load_3d(&tmK, &full[s], st + (OUT ? TILE : 0) + kb * C * 128, kb * 64, t0, bh);
          tma_load_3d(&tmV, &full[s], st + (OUT ? 2 : 1) * TILE + kb * C * 128, kb * 64, t0, bh);
        }
      }
      // drain: every issued load has landed before the block may exit
      for (int it = max(0, nch - NST); it < nch; ++it) mbar_wait(&full[it % NST], (it / NST) & 1, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      bool dead = false;
      constexpr uint32_t ID_SC = idesc_bf16_f32(C, C, false, false);
      constexpr uint32_t ID_O_QW = idesc_bf16_f32(C, D, false, false);
      constexpr uint32_t ID_W = idesc_bf16_f32(D, D, true, true);
      constexpr uint32_t ID_O_PV = idesc_bf16_f32(C, D, false, true);
      for (int it = 0; it < nch; ++it) {
        const int s = it % NST;
        const uint32_t stq = sbase + s * STAGE;
        const uint32_t stk = stq + (OUT ? TILE : 0);
        const uint32_t stv = stq + (OUT ? 2 : 1) * TILE;
        if (!dead) dead = !mbar_wait(&kready[s], (it / NST) & 1, lim);
        tc_fence_after();
        if (OUT) {
          // (1) scores
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(t_sc, desc_k(stq, C, kk), desc_k(stk, C, kk), ID_SC, kk > 0);
          tc_commit(sc_full);
          // (2) O = Q Wbf^T, (3) W += V^T K~
          if (!dead) dead = !mbar_wait(wbf_ready, it & 1, lim);
          if (it > 0 && !dead) dead = !mbar_wait(o_free, (it - 1) & 1, lim);
          tc_fence_after();
          const uint32_t sbf = sbase + NST * STAGE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(t_o, desc_k(stq, C, kk), desc_k(sbf, D, kk), ID_O_QW, kk > 0);
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_w, desc_mn(stv, C, kk), desc_mn(stk, C, kk), ID_W, 1);
          tc_commit(sdone);
          // (4) O += P V
          if (!dead) dead = !mbar_wait(p_ready, it & 1, lim);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk)
            mma_bf16_ss(t_o, desc_k(stq, C, kk), desc_mn(stv, C, kk), ID_O_PV, 1);
          tc_commit(o_full);
        } else {
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk)
            mma_bf16_ss(t_w, desc_mn(stv, C, kk), desc_mn(stk, C, kk), ID_W, (it > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
          if (it == nch - 1) tc_commit(sdone);
        }
      }
      tc_commit(drain);
      mbar_wait(drain, 0, lim);
    }
  } else {
    // --------------------------------------------------------- epilogue --
    const int et = threadIdx.x - 64;          // 0..127
    const int g = warp & 3;                   // TMEM lane group of this warp
    const uint32_t lane_off = static_cast<uint32_t>(32 * g) << 16;
    // row held by this thread in an M=128 accumulator / an M=64 accumulator
    const int row128 = 32 * g + lane;
    const int row64 = 16 * g + lane;
    const bool ok64 = lane < 16;
    const int wrow = (D == 128) ? row128 : row64;  // W row (d_v index)
    const bool wrow_ok = (D == 128) || ok64;
    const int qrow = (C == 128) ? row128 : row64;  // query row of scores / O
    const bool qrow_ok = (C == 128) || ok64;
    const float* eg = p.eta ? p.eta + static_cast<size_t>(bh) * p.T : nullptr;
    bool dead = false;

    for (int it = 0; it < nch; ++it) {
      const int s = it % NST;
      const int t0 = (chunk0 + it) * C;
      uint8_t* st = smem + s * STAGE;
      uint8_t* sk = st + (OUT ? TILE : 0);
      float* ess = es + s * C;
      // learning rate of the chunk's tokens (0 past the end of the sequence)
      for (int r = et; r < C; r += 128) {
        const int t = t0 + r;
        ess[r] = (t < p.T) ? p.sigma * (eg ? eg[t] : p.eta_const) : 0.f;
      }
      if (!dead) dead = !mbar_wait(&full[s], (it / NST) & 1, lim);
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // K~ = diag(sigma * eta) K, in place (16-byte units, swizzle-aware)
      for (int idx = et; idx < C * (D / 8); idx += 128) {
        const int r = idx / (D / 8), cc = idx % (D / 8);
        uint4* ptr = reinterpret_cast<uint4*>(sk + (cc >> 3) * C * 128 + sw128_off(r, cc & 7));
        uint4 u = *ptr;
        const float e = ess[r];
        float2 a;
        a = unpack_bf16x2(u.x); u.x = pack_bf16x2(a.x * e, a.y * e);
        a = unpack_bf16x2(u.y); u.y = pack_bf16x2(a.x * e, a.y * e);
        a = unpack_bf16x2(u.z); u.z = pack_bf16x2(a.x * e, a.y * e);
        a = unpack_bf16x2(u.w); u.w = pack_bf16x2(a.x * e, a.y * e);
        *ptr = u;
      }
      fence_async_smem();
      mbar_arrive(&kready[s]);

      if (!OUT) continue;

      // ---- Wbf = bf16(W entering this chunk); W accumulator initialised at it == 0
      {
        uint8_t* sbf = smem + NST * STAGE;
        uint32_t r[32];
        if (it == 0) {
          const float* src = nullptr;
          if (p.nseg > 1) src = p.ws + (static_cast<size_t>(bh) * p.nseg + seg) * D * D;
          else if (p.S_in) src = p.S_in + static_cast<size_t>(bh) * D * D;
#pragma unroll
          for (int cb = 0; cb < D / 32; ++cb) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              r[j] = __float_as_uint((src && wrow_ok) ? src[static_cast<size_t>(wrow) * D + cb * 32 + j] : 0.f);
            tmem_st32(t_w + lane_off + cb * 32, r);
            if (wrow_ok) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const int col = cb * 32 + q4 * 8;
                uint4 u;
                u.x = pack_bf16x2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
                u.y = pack_bf16x2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
                u.z = pack_bf16x2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
                u.w = pack_bf16x2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
                *reinterpret_cast<uint4*>(sbf + (col >> 6) * D * 128 + sw128_off(wrow, (col & 63) >> 3)) = u;
              }
            }
          }
          tmem_st_wait();
        } else {
          if (!dead) dead = !mbar_wait(sdone, (it - 1) & 1, lim);
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < D / 32; ++cb) {
            tmem_ld32(t_w + lane_off + cb * 32, r);
            tmem_ld_wait();
            if (wrow_ok) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const int col = cb * 32 + q4 * 8;
                uint4 u;
                u.x = pack_bf16x2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
                u.y = pack_bf16x2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
                u.z = pack_bf16x2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
                u.w = pack_bf16x2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
                *reinterpret_cast<uint4*>(sbf + (col >> 6) * D * 128 + sw128_off(wrow, (col & 63) >> 3)) = u;
              }
            }
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(wbf_ready);
      }

      // ---- P = bf16(tril(scores)) into the Q (and K) slots
      {
        uint32_t pk[C / 2];
        if (!dead) dead = !mbar_wait(sc_full, it & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < C / 32; ++cb) {
          uint32_t r[32];
          tmem_ld32(t_sc + lane_off + cb * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const int col = cb * 32 + j;
            const float a0 = (col <= qrow) ? __uint_as_float(r[j]) : 0.f;
            const float a1 = (col + 1 <= qrow) ? __uint_as_float(r[j + 1]) : 0.f;
            pk[(cb * 32 + j) >> 1] = pack_bf16x2(a0, a1);
          }
        }
        if (!dead) dead = !mbar_wait(sdone, it & 1, lim);  // Q, K slots no longer read
        if (qrow_ok) {
#pragma unroll
          for (int c16 = 0; c16 < C / 8; ++c16) {
            uint4 u = make_uint4(pk[c16 * 4 + 0], pk[c16 * 4 + 1], pk[c16 * 4 + 2], pk[c16 * 4 + 3]);
            *reinterpret_cast<uint4*>(st + (c16 >> 3) * C * 128 + sw128_off(qrow, c16 & 7)) = u;
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(p_ready);
      }

      // ---- O: TMEM -> bf16 -> V slot -> TMA store
      {
        uint8_t* sv = st + 2 * TILE;
        if (!dead) dead = !mbar_wait(o_full, it & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t r[32];
          tmem_ld32(t_o + lane_off + cb * 32, r);
          tmem_ld_wait();
          if (qrow_ok) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int col = cb * 32 + q4 * 8;
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
              u.y = pack_bf16x2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
              u.z = pack_bf16x2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
              u.w = pack_bf16x2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
              *reinterpret_cast<uint4*>(sv + (col >> 6) * C * 128 + sw128_off(qrow, (col & 63) >> 3)) = u;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(o_free);
        fence_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (et == 0) {
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb) tma_store_3d(&tmO, sv + kb * C * 128, kb * 64, t0, bh);
          bulk_commit();
          bulk_wait_read0();
          mbar_arrive(&empty[s]);
        }
      }
    }

    // ---- segment result: final W (pass 3, last segment) or dW_p (pass 1)
    const bool write_w = OUT ? (seg == p.nseg - 1 && p.S_out != nullptr) : true;
    if (write_w && nch > 0) {
      // pass 3 commits sdone once per chunk; pass 1 once, after its last chunk
      if (!dead) dead = !mbar_wait(sdone, OUT ? ((nch - 1) & 1) : 0, lim);
      tc_fence_after();
      float* dst = OUT ? p.S_out + static_cast<size_t>(bh) * D * D
                       : p.ws + (static_cast<size_t>(bh) * p.nseg + seg) * D * D;
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
    if (OUT && et == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::TCOLS);
}

// W_start(p) = W_0 + sum_{p' < p} dW_p', in place over the pass-1 results.
__global__ void segment_scan_kernel(float* ws, const float* S_in, int nseg, int DD) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= DD) return;
  float run = S_in ? S_in[static_cast<size_t>(bh) * DD + e] : 0.f;
  for (int s = 0; s < nseg; ++s) {
    float* w = ws + (static_cast<size_t>(bh) * nseg + s) * DD + e;
    const float d = (s < nseg - 1) ? *w : 0.f;
    *w = run;
    run += d;
  }
}

}  // namespace ttt
