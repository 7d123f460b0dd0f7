// feature_map.cuh -- the frozen feature map phi(x) = silu(W1 x) * (W3 x) of
// keys and queries, on the fifth-generation tensor cores (sm_100a).
//
// Variants 1-2 of Table 2 in the thelatestinai.com listing of "Test-Time
// Training with KV Binding Is Secretly Linear Attention" update only the last
// layer of the fast-weight MLP, so the layers before it are fixed for the
// sequence and act as a feature map of the keys and queries.  Here that fixed
// part is one gated hidden layer of the "GLU Variants Improve Transformer"
// form; per head h and token,
//   phi(x) = silu(W1[h] x) * (W3[h] x),   silu(a) = a / (1 + exp(-a)).
//
// Design.  A tile is 128 tokens of one (input, b, h).  W1[h] and W3[h] are
// stacked into one K-major B operand [W1; W3] of 2 d_out rows, so a single
// chain of d_in / 16 MMAs writes [x W1^T | x W3^T] (128 lanes x 2 d_out fp32
// columns) into TMEM.  TMEM holds two (d_out 128) or four (d_out 64) such
// accumulators, so the epilogue of one tile overlaps the MMAs of the next
// ones, and up to eight x stages keep that many tiles of loads in flight.  The
// grid is persistent, one CTA per SM, and walks the tiles in head-major order
// in contiguous ranges, so a CTA's tiles mostly share one head and its stacked
// weights stay in shared memory.
//
// Warp roles (576 threads):
//   warp 0     TMA producer: the stacked weights on a head change, x tiles
//   warp 1     MMA issuer; owns the TMEM allocation
//   warps 2-17 epilogue, two groups of eight taking alternate tiles: a warp
//              reads one TMEM lane quadrant and half of the output columns,
//              applies the gate and rounds to bf16 into its group's
//              128B-swizzled tile; one thread of the group stores the tile
//              with TMA (rows past T are clipped by the map).
//
// Bound: HBM.  Per token it reads d_in and writes d_out bf16 values; the
// weights (2 d_out d_in bf16 per head) come from L2.
#pragma once
#include "common.cuh"

namespace ttt {

struct FmapParams {
  int H, B, T;
  int ntile;    // 128-token tiles per sequence
  int ninputs;  // 1 or 2
  int total;    // H * ninputs * B * ntile
  uint64_t limit_ns;
};

template <int DIN, int DOUT>
struct FmapCfg {
  static_assert(DIN == 64 || DIN == 128, "input width");
  static_assert(DOUT == 64 || DOUT == 128, "output width");
  static constexpr int ROWS = 128;            // tokens per tile (MMA M)
  static constexpr int N = 2 * DOUT;          // [W1; W3] rows (MMA N)
  static constexpr int XT = ROWS * DIN * 2;   // x tile bytes
  static constexpr int WT = N * DIN * 2;      // stacked weight bytes
  static constexpr int YT = ROWS * DOUT * 2;  // output tile bytes
  static constexpr int fits(int nst, int yb) { return 1024 + WT + nst * XT + 2 * yb * YT + 256 <= 232448; }
  // output tiles per epilogue group: two (the next tile is written while the
  // last one is stored) when that still leaves four x stages
  static constexpr int YB = fits(4, 2) ? 2 : 1;
  // as many x stages as shared memory holds, up to 8 (bytes in flight per SM)
  static constexpr int NST = fits(8, YB) ? 8 : fits(6, YB) ? 6 : fits(5, YB) ? 5 : fits(4, YB) ? 4 : fits(3, YB) ? 3 : 2;
  static constexpr int NACC = 512 / N;        // accumulators in TMEM: 4 (d_out 64) or 2 (d_out 128)
  static constexpr int OFF_X = WT;
  static constexpr int OFF_Y = OFF_X + NST * XT;
  static constexpr int OFF_BAR = OFF_Y + 2 * YB * YT;
  static constexpr int NBAR = 2 * NST + 3 + 2 * NACC;  // full, empty, w_full, w_empty, drain, acc_full, acc_empty
  static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
  static constexpr int TCOLS = NACC * N;      // all 512 columns
  static constexpr int EPI_WARPS = 16;        // two groups of eight
  static constexpr int GROUP_WARPS = 8;       // the warps that read one tile
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int CW = DOUT / 2;         // output columns per epilogue thread and tile
  static constexpr int SUBS = CW / 32;        // 32-column pieces of them
  static_assert(SMEM <= 232448, "shared memory");
};

// Named barrier `id` over `n` threads (the epilogue groups).
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Packed fp32 arithmetic (sm_100): one instruction applies the operation to
// both halves of a pair, each rounded to nearest as the scalar form would be.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// silu(a) * b = a b / (1 + e^-a) for a pair of elements, packed as bf16x2.
// e^-a comes from the special-function unit, which bounded the first
// version of this kernel; the reciprocal stays on the FMA pipe: Newton-
// Raphson, r <- r + r (1 - d r), from the seed obtained by subtracting the bit
// pattern of d from 0x7F000000.  For d = 2^E m, 1 <= m < 2, that seed is
// 2^(-E-1) (3 - m), within [1/d, 1.125/d]; each step squares the relative
// error (2^-3, 2^-6, 2^-12, 2^-24), so three steps reach single precision.
// The exponent is clamped at 80 so that d < 2^116 stays in the seed's range;
// past the clamp the quotient is below 1e-34 of a b anyway.  The work runs on
// negated denominators, nd = -(1 + e), so that 1 - d r is one fused step.
__device__ __forceinline__ uint32_t swiglu2_bf16(float a0, float a1, float b0, float b1) {
  const float2 e = make_float2(__expf(-fmaxf(a0, -80.f)), __expf(-fmaxf(a1, -80.f)));
  const float2 m1 = make_float2(-1.f, -1.f), one = make_float2(1.f, 1.f);
  const float2 nd = fma2(e, m1, m1);  // -(1 + e)
  // seed of 1/d from -d: 0x7F000000 - bits(d) = 0xFF000000 - bits(-d) (mod 2^32)
  float2 r = make_float2(__uint_as_float(0xFF000000u - __float_as_uint(nd.x)),
                         __uint_as_float(0xFF000000u - __float_as_uint(nd.y)));
#pragma unroll
  for (int k = 0; k < 3; ++k) r = fma2(r, fma2(nd, r, one), r);
  const float2 y = mul2(mul2(make_float2(a0, a1), make_float2(b0, b1)), r);
  return pack_bf16x2(y.x, y.y);
}

template <int DIN, int DOUT>
__global__ void __launch_bounds__(FmapCfg<DIN, DOUT>::THREADS, 1)
    feature_map_kernel(const __grid_constant__ CUtensorMap tmX0, const __grid_constant__ CUtensorMap tmX1,
                       const __grid_constant__ CUtensorMap tmY0, const __grid_constant__ CUtensorMap tmY1,
                       const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW3,
                       const FmapParams p) {
  using Cfg = FmapCfg<DIN, DOUT>;
  constexpr int NST = Cfg::NST, ROWS = Cfg::ROWS, N = Cfg::N;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* full = bars;                 // [NST] x tile landed
  uint64_t* empty = bars + NST;          // [NST] x stage consumed by the MMAs
  uint64_t* w_full = bars + 2 * NST;     // stacked weights landed
  uint64_t* w_empty = w_full + 1;        // MMAs on the previous weights done
  uint64_t* drain = w_full + 2;          // every MMA of this CTA done
  uint64_t* acc_full = w_full + 3;       // [NACC] accumulator written
  uint64_t* acc_empty = acc_full + Cfg::NACC;  // [NACC] accumulator read out
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + Cfg::NBAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.limit_ns;
  // Contiguous range of tiles, head-major: tile i -> (head, input, b, t).
  const int lo = static_cast<int>(static_cast<long long>(blockIdx.x) * p.total / gridDim.x);
  const int hi = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.total / gridDim.x);
  const int per_head = p.ninputs * p.B * p.ntile;
  auto head_of = [&](int i) { return i / per_head; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(w_full, 1);
    mbar_init(w_empty, 1);
    for (int a = 0; a < Cfg::NACC; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], Cfg::GROUP_WARPS);  // one arrival per warp of the reading group
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::TCOLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX0);
    prefetch_tmap(&tmX1);
    prefetch_tmap(&tmY0);
    prefetch_tmap(&tmY1);
    prefetch_tmap(&tmW1);
    prefetch_tmap(&tmW3);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();  // x is read once
      bool dead = false;
      int cur = -1, nw = 0;
      for (int i = lo, li = 0; i < hi && !dead; ++i, ++li) {
        const int head = head_of(i), r = i % per_head;
        const int inp = r / (p.B * p.ntile), b = (r / p.ntile) % p.B, t = r % p.ntile;
        if (head != cur) {
          if (nw > 0) dead = !mbar_wait(w_empty, (nw - 1) & 1, lim);
          if (dead) break;
          mbar_arrive_expect_tx(w_full, Cfg::WT);
#pragma unroll
          for (int kb = 0; kb < DIN / 64; ++kb) {
            tma_load_3d(&tmW1, w_full, smem + kb * N * 128, kb * 64, 0, head);
            tma_load_3d(&tmW3, w_full, smem + kb * N * 128 + DOUT * 128, kb * 64, 0, head);
          }
          cur = head;
          ++nw;
        }
        const int s = li % NST;
        if (li >= NST) dead = !mbar_wait(&empty[s], ((li / NST) - 1) & 1, lim);
        if (dead) break;
        mbar_arrive_expect_tx(&full[s], Cfg::XT);
        const CUtensorMap* mx = inp ? &tmX1 : &tmX0;
        uint8_t* xs = smem + Cfg::OFF_X + s * Cfg::XT;
#pragma unroll
        for (int kb = 0; kb < DIN / 64; ++kb)
          tma_load_3d_hint(mx, &full[s], xs + kb * ROWS * 128, kb * 64, t * ROWS, b * p.H + head, pol);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t ID = idesc_bf16_f32(ROWS, N, false, false);
      const uint64_t dw = sdesc_sw128(sbase, 16, 1024);
      bool dead = false;
      int cur = -1, nw = 0;
      for (int i = lo, li = 0; i < hi && !dead; ++i, ++li) {
        const int head = head_of(i);
        if (head != cur) {
          if (nw > 0) tc_commit(w_empty);
          dead = !mbar_wait(w_full, nw & 1, lim);
          if (dead) break;
          cur = head;
          ++nw;
        }
        const int s = li % NST, a = li % Cfg::NACC;
        dead = !mbar_wait(&full[s], (li / NST) & 1, lim);
        if (!dead && li >= Cfg::NACC) dead = !mbar_wait(&acc_empty[a], ((li / Cfg::NACC) - 1) & 1, lim);
        if (dead) break;
        tc_fence_after();
        const uint64_t dx = sdesc_sw128(sbase + Cfg::OFF_X + s * Cfg::XT, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < DIN / 16; ++kk)
          mma_bf16_ss(tmem + a * N, dx + k_step(ROWS, kk), dw + k_step(N, kk), ID, kk > 0 ? 1u : 0u);
        tc_commit(&empty[s]);
        tc_commit(&acc_full[a]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, lim);
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    // Two groups of eight warps take alternate tiles, so one group's TMEM
    // reads, barriers and store overlap the other's arithmetic.  In a group,
    // warp w reads lane quadrant w % 4 and half (w / 4) % 2 of the output
    // columns; the group shares one 128B-swizzled output tile, stored by one
    // thread after a group barrier.
    const int ew = warp - 2, grp = ew >> 3, quad = warp & 3, half = (ew >> 2) & 1;
    const int row = quad * 32 + lane;
    const bool issuer = ((ew & 7) == 0 && lane == 0);
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t ys0 = Cfg::OFF_Y + grp * Cfg::YB * Cfg::YT;  // the group's output tiles
    bool dead = false;  // warp-uniform: a wait ran out, later tiles are skipped
    for (int i = lo + grp, li = grp; i < hi; i += 2, li += 2) {
      const int head = head_of(i), r = i % per_head;
      const int inp = r / (p.B * p.ntile), b = (r / p.ntile) % p.B, t = r % p.ntile;
      const int a = li % Cfg::NACC;
      const uint32_t yoff = ys0 + ((li >> 1) % Cfg::YB) * Cfg::YT, ys = sbase + yoff;
      // every thread of the group reaches both barriers of every tile: a
      // timed-out wait only skips the work
      if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&acc_full[a], (li / Cfg::NACC) & 1, lim));
      const bool ok = !dead;
      // this output tile's previous store (YB tiles of the group ago) must have read it
      if (issuer) asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(Cfg::YB - 1) : "memory");
      named_bar_sync(1 + grp, 32 * Cfg::GROUP_WARPS);
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int j = 0; j < Cfg::SUBS; ++j) {
          uint32_t ra[32], rb[32], out[16];
          const int c0 = half * Cfg::CW + j * 32;
          const uint32_t tb = tmem + a * N + lane_off + c0;
          tmem_ld32(tb, ra);
          tmem_ld32(tb + DOUT, rb);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            out[e] = swiglu2_bf16(__uint_as_float(ra[2 * e]), __uint_as_float(ra[2 * e + 1]),
                                  __uint_as_float(rb[2 * e]), __uint_as_float(rb[2 * e + 1]));
          const uint32_t blk = ys + (c0 >> 6) * (ROWS * 128);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(blk + sw128_off(row, ((c0 & 63) >> 3) + q), out[4 * q], out[4 * q + 1], out[4 * q + 2],
                         out[4 * q + 3]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[a]);
        fence_async_smem();
      }
      named_bar_sync(1 + grp, 32 * Cfg::GROUP_WARPS);
      if (issuer && ok) {
        const CUtensorMap* my = inp ? &tmY1 : &tmY0;
#pragma unroll
        for (int blk = 0; blk < DOUT / 64; ++blk)
          tma_store_3d(my, smem + yoff + blk * ROWS * 128, blk * 64, t * ROWS, b * p.H + head);
        bulk_commit();
      }
    }
    if (issuer) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::TCOLS);
}

}  // namespace ttt
