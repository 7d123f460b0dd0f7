// seqshard.cuh -- pieces for splitting one sequence over several devices
// along T (the exchange step of the sequence-split scan).
//
// A run of L tokens acts on the carried state (W, M) as the affine map
//   (W, M) -> (W - G M + dW, B M + dM)
// (the chunked form of "Test-Time Training with KV Binding Is Secretly
// Linear Attention", thelatestinai.com listing, Table 2, Variant 3), where
// dW, dM are the state the run leaves from W = M = 0, and
//   G = sum_{t=1..L} eta_t beta^t,   B = beta^L
// (M enters W through every later step; M_t = beta M_{t-1} + grad_t).  Without
// momentum G = 0 and B = 1.  A device holding a slice of the sequence
// computes its slice's map, the maps are exchanged, and each device composes
// the maps of the slices before its own into its start state.
#pragma once
#include "common.cuh"

namespace ttt {

struct MapScalarParams {
  int BH, T;
  const float* eta;  // [BH, T] or nullptr
  float eta_const, beta;
  float* GB;         // [BH, 2]: G, B
};

// One warp per (b,h).  Lane l takes a contiguous block of tokens and forms
// (s_l, p_l) = (sum_j eta_{t0+j} beta^(j+1), beta^len); the blocks then
// combine as s_0 + p_0 (s_1 + p_1 (s_2 + ...)), a suffix scan over lanes.
__global__ void __launch_bounds__(256) segment_scalars_kernel(const MapScalarParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= p.BH) return;
  const int per = (p.T + 31) / 32;
  const int t0 = lane * per, t1 = min(p.T, t0 + per);
  const float* e = p.eta ? p.eta + static_cast<size_t>(warp) * p.T : nullptr;
  float s = 0.f, pw = 1.f;
  for (int t = t0; t < t1; ++t) {
    pw *= p.beta;
    s = fmaf(e ? __ldg(e + t) : p.eta_const, pw, s);
  }
  // suffix combine: (s, pw) of lanes l..31
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float sh = __shfl_down_sync(0xffffffffu, s, off);
    const float ph = __shfl_down_sync(0xffffffffu, pw, off);
    if (lane + off < 32) {
      s = fmaf(pw, sh, s);
      pw *= ph;
    }
  }
  if (lane == 0) {
    p.GB[2 * warp] = s;
    p.GB[2 * warp + 1] = pw;
  }
}

struct ComposeParams {
  int nmaps;
  long long n;       // BH * d_v * d_k
  int DD;            // d_v * d_k
  const float* dW;   // [nmaps, BH, d_v, d_k]
  const float* dM;   // [nmaps, BH, d_v, d_k] or nullptr (no momentum)
  const float* GB;   // [nmaps, BH, 2] or nullptr (G = 0, B = 1)
  const float* W0;   // [BH, d_v, d_k] or nullptr (zeros)
  const float* M0;
  float* W_out;
  float* M_out;      // or nullptr
};

// Elementwise: (W, M) from (W0, M0) through maps 0..nmaps-1 in order.
__global__ void __launch_bounds__(256) compose_maps_kernel(const ComposeParams p) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < p.n; i += stride) {
    const long long bh = i / p.DD;
    float w = p.W0 ? p.W0[i] : 0.f, m = p.M0 ? p.M0[i] : 0.f;
    for (int j = 0; j < p.nmaps; ++j) {
      const size_t o = static_cast<size_t>(j) * p.n + i;
      const float G = p.GB ? p.GB[(static_cast<size_t>(j) * (p.n / p.DD) + bh) * 2] : 0.f;
      const float B = p.GB ? p.GB[(static_cast<size_t>(j) * (p.n / p.DD) + bh) * 2 + 1] : 1.f;
      w = fmaf(-G, m, w) + p.dW[o];
      m = p.dM ? fmaf(B, m, p.dM[o]) : m;
    }
    p.W_out[i] = w;
    if (p.M_out) p.M_out[i] = m;
  }
}

}  // namespace ttt
