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
// One launch per forward.  P blocks work on each (b, h) sequence so that
// B*H*P blocks fill the SMs in one wave.  A block computes a run of chunks in
// two phases: phase A sums V^T K~ over the run (its total T, the run's whole
// effect on W) into one TMEM accumulator, chunks last to first; phase B is the
// chunk loop above from the run's start state, which is W_0 plus the totals
// of all earlier runs.  The start states come from one of two schedules:
//
//   decoupled look-back (grids of any size): the sequence is cut into P
//     segments, one run each.  A block takes its (segment, head) tile from an
//     atomic counter in segment order, publishes its total, then sums the
//     totals after the nearest predecessor that has published its inclusive
//     state (start + total), and publishes its own inclusive state.
//   waves (the grid is one wave, launched cooperatively): the sequence is cut
//     into `nwave` waves of P runs each, run p of every wave belonging to
//     block p.  Iteration i of a block runs phase A of its run of wave i, then
//     phase B of its run of wave i-1, so the K and V tiles phase B reads were
//     loaded one iteration earlier and are still in L2 (two waves of K and V
//     are live at a time, against the whole sequence for one pass of each
//     phase).  Between, block p is the owner of element slice p of the state:
//     it scans the P totals of wave i-1 at its slice in place into the runs'
//     start states, carrying the state at the wave's end to the next wave in
//     scratch; the blocks then meet at a per-head counter.  The last scan
//     gives the final state.
//
// Block = 8 warps: warp 0 issues TMA loads, warp 1 owns TMEM and issues the
// MMAs (one thread, descriptors precomputed), warps 2-5 (128 threads, one
// TMEM lane each) mask scores, convert fp32 accumulators into bf16 operands,
// stage O and exchange states, warp 6 stores O with TMA, warp 7 scales every
// K tile by a per-token learning rate as it lands (fetching eta two tiles
// ahead; a constant rate is folded into P and the bf16 copy of W instead).
// Per phase-A chunk the MMA thread issues T += V^T K~ into the score region
// of TMEM (free outside phase B), so the next run's start state can be loaded
// into W while phase A runs; per phase-B chunk
//   (1) Sc    = Q K~^T              [TMEM, M=C,   N=C]
//   (2) O[b]  = Q Wbf^T             [TMEM, M=C,   N=d_v]   Wbf = bf16(W) in smem
//   (3) W    += V^T K~              [TMEM, M=d_v, N=d_k]   (after Wbf was taken)
//   (4) O[b] += P V                 P = bf16(masked Sc) in smem
// O is double-buffered in TMEM (b = phase-B chunk parity) so that chunk c+1's
// (2)-(3) overlap the read-out of chunk c.  P is written over the Q (and K)
// slots once (1)-(3) have read them and O is staged in the V slot once (4)
// has read it, so one stage holds just Q, K, V.  Every wait is bounded
// (common.cuh); a thread whose wait runs out stops waiting but keeps arriving,
// so the block always drains and exits.
#pragma once
#include "common.cuh"

namespace ttt {

struct TcParams {
  int BH, T, nchunks, cps, nseg;  // cps = chunks per segment (look-back); nseg = P, blocks per sequence
  int nwave;                      // waves (cooperative schedule; every run of every wave >= 1 chunk); 1 otherwise
  const float* eta;               // [BH, T] or nullptr
  float eta_const, sigma;
  const float* S_in;              // [BH, dv, dk] initial state or nullptr
  // look-back: [BH, nseg, 2, dv, dk] segment totals and inclusive states;
  // waves: [BH, 2, nseg, dv, dk] run totals / start states (slot = wave parity), then [BH, dv, dk] wave-end state
  float* ws;
  // look-back: [BH * nseg] flags, tile counter; waves: [BH * nseg] published-wave counts, [BH] head counters
  unsigned* flags;                // (zeroed per call)
  int coop;                       // 1: waves (launched cooperatively), 0: decoupled look-back
  int keep;                       // phase A: K, V of a run's first `keep` chunks loaded evict-last (phase B reads
                                  // them first), the rest evict-first
  float* S_out;                   // [BH, dv, dk] final state or nullptr
  // BWD only: rows [BH, T, dv] (bf16) dotted with O for the per-token
  // learning-rate gradient deta [BH, T] (both nullptr: no deta)
  const void* vdot;
  float* deta;
  uint64_t limit_ns;
  // Scratch bounds of the debug checks, from the sizes above (kept out of the
  // parameter struct, which a few bytes more made measurably slower in the
  // momentum kernel).
  __device__ __forceinline__ size_t ws_floats_of(int D) const {
    return static_cast<size_t>(BH) * (2 * nseg + (coop ? 1 : 0)) * static_cast<size_t>(D) * D;
  }
  __device__ __forceinline__ size_t flag_words_of() const { return static_cast<size_t>(BH) * nseg + 1 + BH; }
};

// BWD (the backward's two reverse-time passes, see backward_chunked.cuh):
// the chunks are walked last to first (logical chunk c is chunk N-1-c of the
// sequence) with the anti-causal mask j >= i inside a chunk, so the state
// carried in is the sum over the later tokens; K is used unscaled (the pass
// runs with eta = 1, sigma = +1, so `eta`, `eta_const` and `sigma` carry
// the layer's own); the state is read out as bf16(W) + bf16(W - bf16(W)),
// two MMAs whose sum carries W to about 2^-17; and the epilogue writes
// sigma * eta_t * O_t (dv or dk, bf16, through the O map) and, when `deta`
// is set, deta_t = sigma * vdot_t . O_t from O in fp32.
template <int C, int D, bool BWD = false>
struct TcCfg {
  static constexpr int TILE = C * D * 2;                     // bytes of one bf16 C x D tile
  // 64 x 64 tiles fuse (1) and (2) into one N = C + D MMA, [Sc | O] = Q [K~; Wbf]^T:
  // the K region of a stage then holds K~ and that chunk's Wbf as adjacent rows
  // of one operand (order alternating with the chunk's parity, see below).
  static constexpr bool MRG = (C == 64 && D == 64 && !BWD);
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
  static constexpr int SBF_LO = BWD ? D * D * 2 : 0;         // bf16 residual of W (split readout)
  static constexpr int BIG = NST * STAGE + SBF + PBUF + SBF_LO;
  // The 128 x 128 tile streams phase A through three K/V slots (A3): the two
  // stages' K and V regions and a third made of their Q regions, which phase
  // A leaves idle; they have barriers of their own.
  static constexpr bool A3 = (C == 128 && D == 128);
  static constexpr int NBAR = 4 * NST + 12 + (A3 ? 9 : 0);
  static constexpr int SMALL = NBAR * 8 + NST * C * 4 + 32;
  static constexpr int SMEM = BIG + SMALL + 1024;            // + alignment slack
  // W, O x 2 and the scores, which phase A's D-column total shares: C + 3D
  // columns, or 4D when the score region has to grow to hold the total
  static constexpr int TCOLS_USED = (C > D ? C : D) + 3 * D;
  static constexpr int TCOLS = TCOLS_USED <= 256 ? 256 : 512;
  static constexpr int MINB = (C == 64 && D == 64) ? 2 : 1;  // blocks per SM
  static_assert(C == 64 || C == 128, "chunk");
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(C <= 2 * D, "P must fit in the Q and K slots");
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(TCOLS_USED <= 512, "tensor memory");
  static_assert(!BWD || D == 64 || C == 64, "the reverse passes' tiles");
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

// A run of whole chunks: the first chunk and the count.
struct TcSpan {
  int c0, n;
};

// The run of block `seg` in wave w (wave schedule: the wave is chunks
// [w N / nwave, (w + 1) N / nwave), split evenly over the nseg blocks) or its
// segment (look-back: cps chunks from seg * cps, the last one shorter).
__device__ __forceinline__ TcSpan tc_span(const TcParams& p, int seg, int w) {
  TcSpan s;
  if (!p.coop) {
    s.c0 = seg * p.cps;
    s.n = max(0, min(p.cps, p.nchunks - s.c0));
    return s;
  }
  const long long N = p.nchunks;
  const int a = static_cast<int>(w * N / p.nwave), b = static_cast<int>((w + 1) * N / p.nwave);
  const long long L = b - a;
  s.c0 = a + static_cast<int>(seg * L / p.nseg);
  s.n = a + static_cast<int>((seg + 1) * L / p.nseg) - s.c0;
  return s;
}

// Iteration it of a block runs phase A of wave it (look-back: iteration 0,
// every segment but the last) and phase B of wave it - 1.
__device__ __forceinline__ TcSpan tc_span_a(const TcParams& p, int seg, int it) {
  if (it >= p.nwave || (!p.coop && (p.nseg <= 1 || seg == p.nseg - 1))) return TcSpan{0, 0};
  return tc_span(p, seg, it);
}
__device__ __forceinline__ TcSpan tc_span_b(const TcParams& p, int seg, int it) {
  if (it < 1 || it > p.nwave) return TcSpan{0, 0};
  return tc_span(p, seg, it - 1);
}

// Walks the tiles of one block in the order every warp role handles them:
// per iteration, its phase-A chunks last to first, then its phase-B chunks
// first to last.
struct TcCursor {
  int it, k;
  TcSpan A, B;
  __device__ __forceinline__ void settle(const TcParams& p, int seg) {
    while (it <= p.nwave && k >= A.n + B.n) {
      ++it;
      k = 0;
      A = tc_span_a(p, seg, it);
      B = tc_span_b(p, seg, it);
    }
  }
  __device__ __forceinline__ void init(const TcParams& p, int seg) {
    it = 0;
    k = 0;
    A = tc_span_a(p, seg, 0);
    B = tc_span_b(p, seg, 0);
    settle(p, seg);
  }
  __device__ __forceinline__ void next(const TcParams& p, int seg) {
    ++k;
    settle(p, seg);
  }
  __device__ __forceinline__ bool valid(const TcParams& p) const { return it <= p.nwave; }
  __device__ __forceinline__ bool is_b() const { return k >= A.n; }
  __device__ __forceinline__ int chunk() const { return k >= A.n ? B.c0 + (k - A.n) : A.c0 + A.n - 1 - k; }
};

// Writes the bf16 residual x - bf16(x) of each of n fp32 values (raw bits) in place.
template <int N>
__device__ __forceinline__ void to_residual(uint32_t (&r)[N]) {
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float x = __uint_as_float(r[j]);
    r[j] = __float_as_uint(x - __bfloat162float(__float2bfloat16_rn(x)));
  }
}

template <int C, int D, bool BWD = false>
__global__ void __launch_bounds__(256, TcCfg<C, D, BWD>::MINB)
    chunked_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                      const TcParams p) {
  using Cfg = TcCfg<C, D, BWD>;
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
  uint64_t* sdone = sc_full + 1;        // (2),(3) of a phase-B chunk done
  uint64_t* wbf_ready = sc_full + 2;    // Wbf written
  uint64_t* p_ready = sc_full + 3;      // P written
  uint64_t* o_full = sc_full + 4;       // [2] O[b] complete in TMEM
  uint64_t* o_free = sc_full + 6;       // [2] O[b] read out of TMEM
  uint64_t* drain = sc_full + 8;        // final MMA drain
  uint64_t* adone = sc_full + 9;        // a run's phase-A total complete in TMEM
  uint64_t* a_read = sc_full + 10;      // that total read out of TMEM (its columns free again)
  uint64_t* fullA = sc_full + 11;       // [3] phase-A slot landed (A3)
  uint64_t* kreadyA = sc_full + 14;     // [3] its K scaled
  uint64_t* emptyA = sc_full + 17;      // [3] slot free
  float* es = reinterpret_cast<float*>(smem + Cfg::BIG + Cfg::NBAR * 8);  // [NST][C] sigma*eta
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(es + NST * C);
  int* sh_tile = reinterpret_cast<int*>(tmem_holder + 1);
  int* sh_lb = sh_tile + 1;             // decoupled look-back: [1] nearest inclusive predecessor or -1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.limit_ns;
  // Constant learning rate: K~ = c K with one scalar c = sigma * eta, so the
  // kernel uses K itself and folds c in where fp32 values become bf16 operands
  // (P = bf16(c Sc), Wbf = bf16(c W')) and where states cross the boundary.
  // The W accumulator, the phase-A totals and every published or scanned
  // state then hold W' = W / c; W_0 is divided by c as it is read, W_T
  // multiplied by c as it is written.  This removes the K scaler's pass over
  // every K tile (a 32 KB read and write of shared memory per 128 x 128 tile).
  bool fold = false;
  if constexpr (!BWD) fold = p.eta == nullptr && fabsf(p.sigma * p.eta_const) >= 1e-30f;
  const float fc = fold ? p.sigma * p.eta_const : 1.f;  // c, or 1 without the fold
  const float finv = fold ? 1.f / fc : 1.f;

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
    mbar_init(adone, 1);
    mbar_init(a_read, 128);
    if constexpr (Cfg::A3)
      for (int x = 0; x < 3; ++x) {
        mbar_init(&fullA[x], 1);
        mbar_init(&kreadyA[x], 1);
        mbar_init(&emptyA[x], 1);
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
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Look-back: the tile is taken only once this block holds its tensor
  // memory, so a block that others may wait for never waits for tensor memory
  // itself.  Waves: the grid is resident as a whole (cooperative launch).
  if (threadIdx.x == 0)
    *sh_tile = (p.flags && !p.coop) ? static_cast<int>(atomicAdd(p.flags + p.BH * p.nseg, 1u))
                                    : static_cast<int>(blockIdx.x);
  __syncthreads();
  const uint32_t tmem = *tmem_holder;
  const int tile = *sh_tile;
  const int seg = tile / p.BH, bh = tile % p.BH;  // segment-major: predecessors have smaller tiles
  TTT_EXPECT(tile >= 0 && tile < p.BH * p.nseg);
  // Chunk of the sequence that logical chunk c is (reverse time for BWD).
  auto phys = [&](int c) { return BWD ? p.nchunks - 1 - c : c; };
  // Row offsets inside the K region (merged tiles): even phase-B chunks hold
  // [K~ ; Wbf], odd ones [Wbf ; K~], so that the fused MMA writes [Sc | O0] or
  // [O1 | Sc] and O stays double-buffered around one score region in TMEM.
  // Phase-A tiles keep K~ in the first rows.
  auto krow_of = [&](bool pb, int itb) { return (Cfg::MRG && pb && (itb & 1)) ? D : 0; };
  auto wrow_of = [&](int itb) { return (itb & 1) ? 0 : C; };
  // TMEM column map (phase A's total t_a shares the score columns)
  //   merged: [W | O1 | Sc | O0]   C = 64, D = 128: [W | O0 | O1 | Sc + 64 spare]   else: [W | Sc | O0 | O1]
  constexpr bool SC_LAST = (C < D);
  const uint32_t t_w = tmem;  // W: D columns, M = D
  const uint32_t t_sc = Cfg::MRG ? tmem + 2 * D : SC_LAST ? tmem + 3 * D : tmem + D;  // scores: C columns, M = C
  const uint32_t t_a = t_sc;  // phase-A total: D columns, M = D
  auto t_o_of = [&](int b) -> uint32_t {  // O[b]: D columns, M = C
    return Cfg::MRG ? (b ? tmem + D : tmem + 2 * D + C) : SC_LAST ? tmem + D + b * D : tmem + D + C + b * D;
  };
  // Three phase-A slots (A3 tile, when every phase-A chunk of the block comes
  // before its phase-B ones: a single wave).  Phase-A chunk ia goes to slot
  // ia % 3: slot x < 2 is stage x's K and V regions, slot 2 keeps K in stage
  // 0's Q region and V in stage 1's.  Phase-B chunk itb then uses stage
  // itb % NST, whose first use waits for the phase-A slots it overlaps.
  const bool a3 = Cfg::A3 && p.nwave == 1;
  const int nA0 = tc_span_a(p, seg, 0).n;  // the block's phase-A chunks (a single wave)
  auto a_koff = [](int x) { return x == 2 ? 0 : x * STAGE + Cfg::OK; };
  auto a_voff = [](int x) { return x == 2 ? STAGE : x * STAGE + Cfg::OV; };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      bool dead = false;
      // Q and phase-B K and V are read for the last time: evict-first.
      // Phase A walks a run last to first, so its final loads are the chunks
      // phase B reads first: the K and V of a run's first `keep` chunks are
      // loaded evict-last (the planner sizes `keep` so that they fit in L2
      // beside the streams), the rest evict-first.
      const uint64_t pol_once = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      int g = 0, itb = 0, ia = 0;
      TcCursor cur;
      for (cur.init(p, seg); cur.valid(p); cur.next(p, seg), ++g) {
        const bool pb = cur.is_b();
        const int t0 = phys(cur.chunk()) * C;
        TTT_EXPECT(cur.chunk() >= 0 && cur.chunk() < p.nchunks);
        const uint64_t pol_kv = (!pb && cur.chunk() - cur.A.c0 < p.keep) ? pol_keep : pol_once;
        if (a3 && !pb) {
          const int x = ia % 3, u = ia / 3;
          if (u > 0 && !dead) dead = !mbar_wait(&emptyA[x], (u - 1) & 1, lim);
          mbar_arrive_expect_tx(&fullA[x], 2 * TILE);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb) {
            tma_load_3d_hint(&tmK, &fullA[x], smem + a_koff(x) + kb * C * 128, kb * 64, t0, bh, pol_kv);
            tma_load_3d_hint(&tmV, &fullA[x], smem + a_voff(x) + kb * C * 128, kb * 64, t0, bh, pol_kv);
          }
          ++ia;
          continue;
        }
        const int s = (a3 ? itb : g) % NST, u = (a3 ? itb : g) / NST;
        if (a3 && u == 0) {
          // first use of stage s: the phase-A slots on it (slot s; slot 2 in the Q regions) are free
          const int on_stage[2] = {s, 2};
          for (int i = 0; i < 2; ++i) {
            const int x = on_stage[i], uses = nA0 / 3 + (x < nA0 % 3 ? 1 : 0);
            if (uses > 0 && !dead) dead = !mbar_wait(&emptyA[x], (uses - 1) & 1, lim);
          }
        } else if (u > 0 && !dead) {
          dead = !mbar_wait(&empty[s], (u - 1) & 1, lim);
        }
        mbar_arrive_expect_tx(&full[s], pb ? 3 * TILE : 2 * TILE);
        uint8_t* st = smem + s * STAGE;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          if (pb) tma_load_3d_hint(&tmQ, &full[s], st + kb * C * 128, kb * 64, t0, bh, pol_once);
          uint8_t* kd = st + Cfg::OK + (kb * Cfg::KWR + krow_of(pb, itb)) * 128;
          uint8_t* vd = st + Cfg::OV + kb * C * 128;
          tma_load_3d_hint(&tmK, &full[s], kd, kb * 64, t0, bh, pol_kv);
          tma_load_3d_hint(&tmV, &full[s], vd, kb * 64, t0, bh, pol_kv);
        }
        if (pb) ++itb;
      }
      const int nst_items = a3 ? itb : g;  // loads on the stage barriers
      for (int j = max(0, nst_items - NST); j < nst_items; ++j) mbar_wait(&full[j % NST], (j / NST) & 1, lim);
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
      const uint64_t d_wlo = sdesc_sw128(sbase + NST * STAGE + Cfg::SBF + Cfg::PBUF, 16, 1024);
      int g = 0, itb = 0, nread = 0, ia = 0;
      bool pending_read = false;  // a phase-A total sits in the score columns, not yet read out
      auto free_scores = [&]() {
        if (pending_read) {
          if (!dead) dead = !mbar_wait(a_read, nread & 1, lim);
          ++nread;
          pending_read = false;
        }
      };
      TcCursor cur;
      for (cur.init(p, seg); cur.valid(p); cur.next(p, seg), ++g) {
        if (!cur.is_b()) {
          // phase A: T (+)= V^T K~ into the score columns
          const int x = ia % 3, s = g % NST;
          const uint32_t stk = a3 ? sbase + a_koff(x) : sbase + s * STAGE + Cfg::OK;
          const uint32_t stv = a3 ? sbase + a_voff(x) : sbase + s * STAGE + Cfg::OV;
          const uint64_t dkm = sdesc_sw128(stk, Cfg::KWR * 128, 1024), dvm = sdesc_sw128(stv, C * 128, 1024);
          if (cur.k == 0) free_scores();
          // (BWD: K is used as loaded and the scaler warp sits out)
          if (!dead) dead = !mbar_wait(a3 ? &kreadyA[x] : BWD ? &full[s] : &kready[s], ((a3 ? ia / 3 : g / NST)) & 1, lim);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk)
            mma_bf16_ss(t_a, dvm + mn_step(kk), dkm + mn_step(kk), ID_W, (cur.k > 0 || kk > 0) ? 1u : 0u);
          tc_commit(a3 ? &emptyA[x] : &empty[s]);
          ++ia;
          if (cur.k == cur.A.n - 1) {
            tc_commit(adone);
            pending_read = true;
          }
          continue;
        }
        // phase B
        const int b = itb & 1, s = (a3 ? itb : g) % NST, u = (a3 ? itb : g) / NST;
        const uint32_t stq = sbase + s * STAGE, stk = stq + Cfg::OK, stv = stq + Cfg::OV;
        const uint64_t dq = sdesc_sw128(stq, 16, 1024), dkk = sdesc_sw128(stk, 16, 1024);
        const uint64_t dkm = sdesc_sw128(stk + krow_of(true, itb) * 128, Cfg::KWR * 128, 1024);
        const uint64_t dvm = sdesc_sw128(stv, C * 128, 1024);
        const uint64_t dp = Cfg::PSEP ? d_pbuf : dq;
        const uint32_t t_o = t_o_of(b);
        if (!dead) dead = !mbar_wait(BWD ? &full[s] : &kready[s], u & 1, lim);
        free_scores();
        if (Cfg::MRG) {
          // [Sc | O] in one N = C + D MMA: needs this chunk's Wbf and a free O[b]
          if (!dead) dead = !mbar_wait(wbf_ready, itb & 1, lim);
          if (itb >= 2 && !dead) dead = !mbar_wait(&o_free[b], ((itb - 2) >> 1) & 1, lim);
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
          if (!dead) dead = !mbar_wait(wbf_ready, itb & 1, lim);
          if (itb >= 2 && !dead) dead = !mbar_wait(&o_free[b], ((itb - 2) >> 1) & 1, lim);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(t_o, dq + k_step(C, kk), d_wbf + k_step(D, kk), ID_O_QW, kk > 0);
          if constexpr (BWD) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) mma_bf16_ss(t_o, dq + k_step(C, kk), d_wlo + k_step(D, kk), ID_O_QW, 1);
          }
        }
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_w, dvm + mn_step(kk), dkm + mn_step(kk), ID_W, 1);
        tc_commit(sdone);
        if (!dead) dead = !mbar_wait(p_ready, itb & 1, lim);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) mma_bf16_ss(t_o, dp + k_step(C, kk), dvm + mn_step(kk), ID_O_PV, 1);
        tc_commit(&o_full[b]);
        ++itb;
      }
      free_scores();
      tc_commit(drain);
      mbar_wait(drain, 0, lim);
    }
  } else if (warp == 6) {
    // ----------------------------------------------------- O store warp --
    if (lane == 0) {
      bool dead = false;
      int g = 0, itb = 0;
      const uint64_t pol_out = l2_policy_evict_first();
      TcCursor cur;
      for (cur.init(p, seg); cur.valid(p); cur.next(p, seg), ++g) {
        if (!cur.is_b()) continue;
        const int s = (a3 ? itb : g) % NST;
        if (!dead) dead = !mbar_wait(&staged[itb % NST], (itb / NST) & 1, lim);
        {
          const uint8_t* sv = smem + s * STAGE + Cfg::OV;
          const int t0 = phys(cur.chunk()) * C;
          // O is not read again: evict-first, so that it does not push out
          // the K and V phase B still reads from L2
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb) tma_store_3d_hint(&tmO, sv + kb * C * 128, kb * 64, t0, bh, pol_out);
          bulk_commit();
          bulk_wait_read0();
        }
        mbar_arrive(&empty[s]);
        ++itb;
      }
      bulk_wait0();
    }
  } else if (warp == 7) {
    // ------------------------------------------------------- K scaler --
    // K~ = diag(sigma * eta) K for every tile as it lands (phase A and B),
    // in place, swizzle-aware; eta is fetched two tiles ahead.  (BWD: no
    // scaling.)
    if constexpr (!BWD) {
      bool dead = false;
      constexpr int RPL = C / 32;  // rows of a chunk whose eta this lane fetches
      const float* eg = p.eta ? p.eta + static_cast<size_t>(bh) * p.T : nullptr;
      auto fetch = [&](const TcCursor& c, float (&dst)[RPL]) {
        const bool ok = c.valid(p);
        const int c0 = ok ? c.chunk() * C : 0;
#pragma unroll
        for (int j = 0; j < RPL; ++j) {
          const int t = c0 + lane + 32 * j;
          dst[j] = (ok && t < p.T) ? (eg ? __ldg(eg + t) : p.eta_const) : 0.f;
        }
      };
      TcCursor cur, ahead;
      cur.init(p, seg);
      ahead = cur;
      float er[RPL], en[RPL];
      fetch(ahead, er);
      if (ahead.valid(p)) ahead.next(p, seg);
      fetch(ahead, en);
      if (ahead.valid(p)) ahead.next(p, seg);
      constexpr int PER_LANE = C * (D / 8) / 32;  // 16-byte units of the K tile per lane
      constexpr int BATCH = 8;
      int g = 0, itb = 0, ia = 0;
      for (; cur.valid(p); cur.next(p, seg), ++g) {
        const bool pb = cur.is_b();
        const bool slotA = a3 && !pb;  // a three-slot phase-A chunk
        const int x = ia % 3;
        const int s = slotA ? x % NST : (a3 ? itb : g) % NST;
        const int u = slotA ? ia / 3 : (a3 ? itb : g) / NST;
        uint64_t* fb = slotA ? &fullA[x] : &full[s];
        uint64_t* kb_ready = slotA ? &kreadyA[x] : &kready[s];
        float* ess = es + s * C;
#pragma unroll
        for (int j = 0; j < RPL; ++j) ess[lane + 32 * j] = p.sigma * er[j];
#pragma unroll
        for (int j = 0; j < RPL; ++j) er[j] = en[j];
        fetch(ahead, en);
        if (ahead.valid(p)) ahead.next(p, seg);
        __syncwarp();
        if (!dead) dead = !mbar_wait(fb, u & 1, lim);
        uint8_t* sk = slotA ? smem + a_koff(x) : smem + s * STAGE + Cfg::OK + krow_of(pb, itb) * 128;
#pragma unroll 1
        for (int b0 = 0; b0 < (fold ? 0 : PER_LANE); b0 += BATCH) {
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
        if (lane == 0) mbar_arrive(kb_ready);
        if (pb) ++itb;
        if (slotA) ++ia;
      }
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
    constexpr size_t DD = static_cast<size_t>(D) * D;
    // a row of W' as the bf16 operand Wbf = bf16(c W') (no-op without the fold)
    auto wscale = [&](auto& r) {
#pragma unroll
      for (auto& x : r) x = __float_as_uint(fc * __uint_as_float(x));
    };
    // The merged 64 x 64 tile (two blocks per SM, 128 registers a thread)
    // runs the decoupled look-back only.
    bool waves = false;
    if constexpr (!Cfg::MRG) waves = p.coop != 0;
    int g0 = 0;     // tile index of the iteration's first tile
    int itb = 0;    // phase-B chunks so far
    int nadone = 0;

    // Reads the phase-A total out of TMEM into quad-major fp32 at `dst` (this
    // thread's row), then frees the score columns for the MMA thread.
    auto publish_total = [&](float* dst, bool release_columns) {
      if (!dead) dead = !mbar_wait(adone, nadone & 1, lim);
      ++nadone;
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t r[32];
        tmem_ld32(t_a + lane_off + cb * 32, r);
        tmem_ld_wait();
        if (wrow_ok) {
          float4* a4 = reinterpret_cast<float4*>(dst);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcg(a4 + qm4<D>(wrow, cb * 8 + j),
                   make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                               __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
        }
      }
      if (release_columns) {
        tc_fence_before();
        mbar_arrive(a_read);
      }
    };
    // Writes this thread's row of a start state (quad-major fp32 at `src`)
    // into the W accumulator and, as bf16, into the Wbf operand of phase-B
    // chunk `itb` (tile index gb); with d = 128 all loads are issued before any
    // store (one round trip), with d = 64 one 32-column block per round
    // (register budget of two blocks per SM).
    auto load_start_qm = [&](const float* src, int gb) {
      constexpr int G = (D == 128) ? D / 32 : 1;
#pragma unroll
      for (int cb0 = 0; cb0 < D / 32; cb0 += G) {
        float row[G * 32];
#pragma unroll
        for (int c = 0; c < G * 8; ++c) {
          const float4 x = wrow_ok ? __ldcg(reinterpret_cast<const float4*>(src) + qm4<D>(wrow, cb0 * 8 + c))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
          row[4 * c] = x.x, row[4 * c + 1] = x.y, row[4 * c + 2] = x.z, row[4 * c + 3] = x.w;
        }
#pragma unroll
        for (int cb = 0; cb < G; ++cb) {
          uint32_t r[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(row[cb * 32 + j]);
          tmem_st32(t_w + lane_off + (cb0 + cb) * 32, r);  // W accumulator := start
          if (fold) wscale(r);
          if (wrow_ok) {
            if (Cfg::MRG)
              store_row32_bf16(sbase + (gb % NST) * STAGE + Cfg::OK + wrow_of(itb) * 128, Cfg::KWR * 128, wrow,
                               (cb0 + cb) * 32, r);
            else
              store_row32_bf16(sbase + NST * STAGE, D * 128, wrow, (cb0 + cb) * 32, r);
            if constexpr (BWD) {
              to_residual(r);
              store_row32_bf16(sbase + NST * STAGE + Cfg::SBF + Cfg::PBUF, D * 128, wrow, (cb0 + cb) * 32, r);
            }
          }
        }
      }
      tmem_st_wait();
    };

    // (the merged 64 x 64 tile always runs one wave: a constant trip count
    // lets the compiler lay its two iterations out straight)
    const int nwave = Cfg::MRG ? 1 : p.nwave;
#pragma unroll(Cfg::MRG ? 2 : 1)
    for (int it = 0; it <= nwave; ++it) {
      const TcSpan A = tc_span_a(p, seg, it), Bs = tc_span_b(p, seg, it);
      const int gb0 = g0 + A.n;  // tile index of the first phase-B chunk
      g0 += A.n + Bs.n;
      if (waves) {
        // ================================================ wave schedule ==
        const int P = p.nseg;
        float4* ws4 = reinterpret_cast<float4*>(p.ws);
        const size_t DD4 = DD / 4, ws4n = p.ws_floats_of(D) / 4;
        unsigned* wflag = TTT_AT(p.flags, static_cast<size_t>(bh) * P, P, p.flag_words_of());  // [P] published-wave counts
        unsigned* cnt = TTT_AT(p.flags, static_cast<size_t>(p.BH) * P + 1 + bh, 1, p.flag_words_of());
        auto tot4 = [&](int slot, int j) {
          return TTT_AT(ws4, ((static_cast<size_t>(bh) * 2 + slot) * P + j) * DD4, DD4, ws4n);
        };
        if (it >= 1) {
          // (a) owner of slice `seg`: in-place exclusive scan of wave it-1's
          // totals into its runs' start states, carrying the wave-end state
          const int slot = (it - 1) & 1;
          for (int j = et; j < P; j += 128)
            if (!dead && wait_geq(wflag + j, static_cast<unsigned>(it), lim) == 0) dead = true;
          asm volatile("bar.sync 1, 128;" ::: "memory");
          const int SL = static_cast<int>((DD4 + P - 1) / P);
          const int v1 = min(static_cast<int>(DD4), (seg + 1) * SL);
          float4* send = TTT_AT(ws4, static_cast<size_t>(p.BH) * 2 * P * DD4 + static_cast<size_t>(bh) * DD4, DD4, ws4n);
          const size_t nst4 = static_cast<size_t>(p.BH) * DD4;
          const float4* s4 = p.S_in ? TTT_AT(reinterpret_cast<const float4*>(p.S_in), bh * DD4, DD4, nst4) : nullptr;
          float4* o4 = p.S_out ? TTT_AT(reinterpret_cast<float4*>(p.S_out), bh * DD4, DD4, nst4) : nullptr;
          TTT_EXPECT(v1 <= static_cast<int>(DD4));
          // Two positions per thread (v0 and v0 + 128), up to NB totals per
          // round with every load of the round issued before its stores: the
          // scan costs a few L2 round trips (its adds are cheap; its latency
          // sits between phase A and phase B of every wave; more totals per
          // round spill registers).
          constexpr int NB = 4;
          const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int v0 = seg * SL + et; v0 < v1; v0 += 256) {
            const bool ok1 = v0 + 128 < v1;
            // the scratch is quad-major, the caller's W_0 and W_T row-major
            float4 run0 = (it > 1) ? __ldcg(send + v0) : (s4 ? f4_scale(finv, __ldcg(s4 + qm4_to_rm4<D>(v0))) : zero);
            float4 run1 = !ok1 ? zero
                               : (it > 1) ? __ldcg(send + v0 + 128)
                                          : (s4 ? f4_scale(finv, __ldcg(s4 + qm4_to_rm4<D>(v0 + 128))) : zero);
            for (int j0 = 0; j0 < P; j0 += NB) {
              float4 a0[NB], a1[NB];
#pragma unroll
              for (int u = 0; u < NB; ++u) {
                if (j0 + u < P) {
                  const float4* tj = tot4(slot, j0 + u) + v0;  // run j0 + u's total at this position
                  a0[u] = __ldcg(tj);
                  if (ok1) a1[u] = __ldcg(tj + 128);
                }
              }
#pragma unroll
              for (int u = 0; u < NB; ++u) {
                if (j0 + u < P) {
                  float4* tj = tot4(slot, j0 + u) + v0;
                  __stcg(tj, run0);
                  run0 = f4_add(run0, a0[u]);
                  if (ok1) {
                    __stcg(tj + 128, run1);
                    run1 = f4_add(run1, a1[u]);
                  }
                }
              }
            }
            __stcg(send + v0, run0);
            if (ok1) __stcg(send + v0 + 128, run1);
            if (it == p.nwave && o4) {
              o4[qm4_to_rm4<D>(v0)] = f4_scale(fc, run0);
              if (ok1) o4[qm4_to_rm4<D>(v0 + 128)] = f4_scale(fc, run1);
            }
          }
          __threadfence();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (et == 0) {
            atomicAdd(cnt, 1u);
            // every owner has scanned wave it-1: the start states are final,
            // and the other slot may be written again
            if (!dead && wait_geq(cnt, static_cast<unsigned>(P * it), lim) == 0) dead = true;
            __threadfence();
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
        }
        // (c) this block's start state for its run of wave it-1, loaded while
        // phase A of wave it runs: W and the Wbf buffer are free by then (the
        // merged 64 x 64 tile, which keeps Wbf in rows a phase-A tile may
        // still occupy, never runs this schedule)
        if (it >= 1 && Bs.n > 0) {
          load_start_qm(reinterpret_cast<const float*>(tot4((it - 1) & 1, seg)), gb0);
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(wbf_ready);
        }
        if (it < p.nwave) {
          // (b) publish this block's total of wave it
          if (A.n > 0) publish_total(reinterpret_cast<float*>(tot4(it & 1, seg)), true);
          __threadfence();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (et == 0) st_release(wflag + seg, static_cast<unsigned>(it + 1));
        }
      } else if (it == 0) {
        // ============================================ decoupled look-back ==
        // publish this segment's total (its state leaves t_a only once the
        // inclusive state is out, in iteration 1)
        if (A.n > 0) {
          float* agg_me = TTT_AT(p.ws, (static_cast<size_t>(bh) * p.nseg + seg) * 2 * DD, DD, p.ws_floats_of(D));
          publish_total(agg_me, false);
          __threadfence();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (et == 0) st_release(TTT_AT(p.flags, static_cast<size_t>(bh) * p.nseg + seg, 1, p.flag_words_of()), 1u);
        }
      } else {
        // W_start = W_0 + the totals of the segments after the nearest
        // predecessor that has published its inclusive state (start + total).
        // One thread per predecessor reads the flags.
        const bool hasA = tc_span_a(p, seg, 0).n > 0;
        float* agg_me = hasA ? TTT_AT(p.ws, (static_cast<size_t>(bh) * p.nseg + seg) * 2 * DD, 2 * DD, p.ws_floats_of(D))
                             : nullptr;
        const float* base = p.S_in ? TTT_AT(p.S_in, bh * DD, DD, static_cast<size_t>(p.BH) * DD) : nullptr;
        int first = 0;
        bool base_qm = false;  // base is a published (quad-major) state, not the caller's W_0
        if (seg > 0) {
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
          if (incl >= 0) {
            base = TTT_AT(p.ws, ((static_cast<size_t>(bh) * p.nseg + incl) * 2 + 1) * DD, DD, p.ws_floats_of(D));
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
                const float sc = base_qm ? 1.f : finv;  // the caller's W_0 enters as W_0 / c
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[8 * j + e] = sc * x.v[e];
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
                const float* ag = TTT_AT(p.ws, (static_cast<size_t>(bh) * p.nseg + jj + u) * 2 * DD, DD, p.ws_floats_of(D));
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
              const float* ag = TTT_AT(p.ws, (static_cast<size_t>(bh) * p.nseg + jj) * 2 * DD, DD, p.ws_floats_of(D));
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
          if (hasA) {  // this segment's total is still in t_a: publish the inclusive state
            tmem_ld32(t_a + lane_off + cb * 32, r);
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
          if (fold) wscale(r);
          if (wrow_ok) {
            if (Cfg::MRG)
              store_row32_bf16(sbase + (gb0 % NST) * STAGE + Cfg::OK + wrow_of(itb) * 128, Cfg::KWR * 128, wrow,
                               cb * 32, r);
            else
              store_row32_bf16(sbase + NST * STAGE, D * 128, wrow, cb * 32, r);
            if constexpr (BWD) {
              to_residual(r);
              store_row32_bf16(sbase + NST * STAGE + Cfg::SBF + Cfg::PBUF, D * 128, wrow, cb * 32, r);
            }
          }
        }
        tmem_st_wait();
        if (hasA) {
          tc_fence_before();
          mbar_arrive(a_read);  // the score columns are free for phase B
          __threadfence();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (et == 0) st_release(TTT_AT(p.flags, static_cast<size_t>(bh) * p.nseg + seg, 1, p.flag_words_of()), 2u);
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(wbf_ready);
      }

      // ---------------------------------------------------------- phase B
      for (int j = 0; j < Bs.n; ++j, ++itb) {
        const int g = gb0 + j, s = (a3 ? itb : g) % NST, b = itb & 1;
        uint8_t* st = smem + s * STAGE;
        // P = bf16(tril(scores)) into the Q (and K) slots (BWD: triu, j >= i)
        {
          if (!dead) dead = !mbar_wait(sc_full, itb & 1, lim);
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
            const int jd = row64h - 32 * half;  // the diagonal's column in this half
            auto keep = [&](int jj) { return BWD ? jj >= jd : jj <= jd; };
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int jj = 8 * i + 2 * e;
                w[e] = pack_bf16x2(keep(jj) ? fc * __uint_as_float(r[jj]) : 0.f,
                                   keep(jj + 1) ? fc * __uint_as_float(r[jj + 1]) : 0.f);
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
              for (int jj = 0; jj < 64; jj += 2) {
                const int col = cb * 64 + jj;
                const bool k0 = BWD ? col >= qrow : col <= qrow, k1 = BWD ? col + 1 >= qrow : col + 1 <= qrow;
                const float a0 = k0 ? fc * __uint_as_float(r[jj]) : 0.f;
                const float a1 = k1 ? fc * __uint_as_float(r[jj + 1]) : 0.f;
                pk[col >> 1] = pack_bf16x2(a0, a1);
              }
            }
            // the overlaid P must wait until (1)-(3) have read the Q and K
            // slots; a separate P buffer only until (4) of the previous tile
            // (o_full, waited in the previous O step)
            uint8_t* pdst = Cfg::PSEP ? smem + NST * STAGE + Cfg::SBF : st;
            if (!Cfg::PSEP && !dead) dead = !mbar_wait(sdone, itb & 1, lim);
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
        if (j + 1 < Bs.n) {
          if (Cfg::PSEP && !dead) dead = !mbar_wait(sdone, itb & 1, lim);
          tc_fence_after();
          const uint32_t wdst =
              Cfg::MRG ? sbase + ((g + 1) % NST) * STAGE + Cfg::OK + wrow_of(itb + 1) * 128 : sbase + NST * STAGE;
          const int wblk = Cfg::MRG ? Cfg::KWR * 128 : D * 128;
          const uint32_t wlo = sbase + NST * STAGE + Cfg::SBF + Cfg::PBUF;
          if constexpr (D == 64) {
            uint32_t r[32];
            tmem_ld_half32(t_w + lane_off, r);
            tmem_ld_wait();
            if (fold) wscale(r);
            store_row32_bf16(wdst, wblk, row64h, 32 * half, r);
            if constexpr (BWD) {
              to_residual(r);
              store_row32_bf16(wlo, wblk, row64h, 32 * half, r);
            }
          } else {
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
              uint32_t r[64];
              tmem_ld64(t_w + lane_off + cb * 64, r);
              tmem_ld_wait();
              if (fold) wscale(r);
              store_row64_bf16(wdst, wblk, wrow, cb * 64, r);
              if constexpr (BWD) {
                to_residual(r);
                store_row64_bf16(wlo, wblk, wrow, cb * 64, r);
              }
            }
          }
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(wbf_ready);
        }
        // O[b]: TMEM -> bf16 -> V slot, then the store warp takes it
        {
          const uint32_t sv = sbase + s * STAGE + Cfg::OV;
          // BWD: this thread's token (row crow of the chunk, NV columns from
          // c0: a whole row of 128-token tiles, half a row of 64-token ones),
          // its sigma * eta and its NV values of vdot, fetched before the wait
          // (rows past T give zeros, which the TMA store drops)
          constexpr int NV = (C == 128) ? D : D / 2, NU = NV / 8;
          [[maybe_unused]] const int crow = (C == 128) ? qrow : row64h;
          [[maybe_unused]] const int c0 = (C == 128) ? 0 : NV * half;
          [[maybe_unused]] size_t rowi = 0;
          [[maybe_unused]] bool live = false;
          [[maybe_unused]] float es_t = 0.f;
          [[maybe_unused]] uint4 vv[NU];
          if constexpr (BWD) {
            const int tok = phys(Bs.c0 + j) * C + crow;
            const size_t ntok = static_cast<size_t>(p.BH) * p.T;
            live = tok < p.T;
            rowi = static_cast<size_t>(bh) * p.T + tok;
            es_t = live ? p.sigma * (p.eta ? __ldg(TTT_AT(p.eta, rowi, 1, ntok)) : p.eta_const) : 0.f;
#pragma unroll
            for (int i = 0; i < NU; ++i) vv[i] = make_uint4(0u, 0u, 0u, 0u);
            if (p.deta && live) {
              const uint4* src = TTT_AT(static_cast<const uint4*>(p.vdot), (rowi * D + c0) / 8, NU, ntok * D / 8);
#pragma unroll
              for (int i = 0; i < NU; ++i) vv[i] = __ldg(src + i);
            }
          }
          if (!dead) dead = !mbar_wait(&o_full[b], (itb >> 1) & 1, lim);
          tc_fence_after();
          const uint32_t t_o = t_o_of(b);
          if constexpr (BWD) {
            uint32_t r[NV];
            if constexpr (C == 128)
              tmem_ld64(t_o + lane_off, r);
            else if constexpr (NV == 64)
              tmem_ld_half64(t_o + lane_off, r);
            else
              tmem_ld_half32(t_o + lane_off, r);
            tmem_ld_wait();
            if (p.deta) {
              float dot = 0.f;
#pragma unroll
              for (int i = 0; i < NU; ++i) {
                const uint32_t w[4] = {vv[i].x, vv[i].y, vv[i].z, vv[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  dot = fmaf(__uint_as_float(w[e] << 16), __uint_as_float(r[8 * i + 2 * e]), dot);
                  dot = fmaf(__uint_as_float(w[e] & 0xffff0000u), __uint_as_float(r[8 * i + 2 * e + 1]), dot);
                }
              }
              if constexpr (C == 64) dot += __shfl_xor_sync(0xffffffffu, dot, 16);  // the row's other half
              if (live && (C == 128 || half == 0)) *TTT_AT(p.deta, rowi, 1, static_cast<size_t>(p.BH) * p.T) = p.sigma * dot;
            }
#pragma unroll
            for (int i = 0; i < NV; ++i) r[i] = __float_as_uint(es_t * __uint_as_float(r[i]));
            if constexpr (NV == 64)
              store_row64_bf16(sv, C * 128, crow, c0, r);
            else
              store_row32_bf16(sv, C * 128, crow, c0, r);
          } else if constexpr (C == 64 && D == 64) {
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
          mbar_arrive(&staged[itb % NST]);
        }
      }
    }

    // final state of the sequence (look-back: the last segment's W; the wave
    // schedule writes it in its last scan)
    if (!p.coop && seg == p.nseg - 1 && p.S_out != nullptr && itb > 0) {
      // W_T may overwrite W_0 (in place): first every predecessor must have
      // read W_0, which it has once its inclusive state is out (flag 2)
      for (int j = et; j < seg; j += 128)
        if (!dead && wait_geq(TTT_AT(p.flags, static_cast<size_t>(bh) * p.nseg + j, 1, p.flag_words_of()), 2u, lim) == 0)
          dead = true;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!dead) dead = !mbar_wait(sdone, (itb - 1) & 1, lim);
      tc_fence_after();
      float* dst = TTT_AT(p.S_out, bh * DD, DD, static_cast<size_t>(p.BH) * DD);
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t r[32];
        tmem_ld32(t_w + lane_off + cb * 32, r);
        tmem_ld_wait();
        if (wrow_ok) {
          float4* d4 = reinterpret_cast<float4*>(dst + static_cast<size_t>(wrow) * D + cb * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            d4[j] = make_float4(fc * __uint_as_float(r[4 * j]), fc * __uint_as_float(r[4 * j + 1]),
                                fc * __uint_as_float(r[4 * j + 2]), fc * __uint_as_float(r[4 * j + 3]));
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
