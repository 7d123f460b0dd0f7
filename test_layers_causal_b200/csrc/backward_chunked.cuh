// backward_chunked.cuh -- pieces of the chunk-parallel backward of the layer
// without momentum.
//
// The gradient of the plain layer (update, then read; W_t = W_{t-1} +
// sigma eta_t v_t k_t^T, o_t = W_t q_t) is three runs of the forward layer
// itself, each computed by the chunked forward:
//   dq_t = W_t^T do_t       the forward on (q, k, v) := (do, v, k) from W_0^T,
//                           same eta and sigma;
//   u_t  = G_t k_t          the forward on the time-reversed sequence of
//                           (q, k, v) := (k, q, do), eta = 1, sigma = +1,
//                           from dL/dW_T; its final state is dL/dW_0 = G_1;
//   r_t  = G_t^T v_t        the same on (v, do, q) from (dL/dW_T)^T;
// with G_t = dL/dW_T + sum_{t' >= t} do_t' q_t'^T.  Then
//   dv_t = sigma eta_t u_t,  dk_t = sigma eta_t r_t,  deta_t = sigma v_t . u_t.
// In bf16 the two reverse-time passes run on the tensor cores straight over
// the inputs, chunks last to first with the anti-causal mask (chunked_tc.cuh,
// BWD), and their epilogues apply that last step.  The fp32 path runs them
// on copies reversed along T and applies it in a finishing kernel.  Both
// transpose W_0 and dL/dW_T with the kernel here.  (The gradient of "Test-Time Training with KV Binding
// Is Secretly Linear Attention"'s layer, needed for the training of its
// Figure 4, thelatestinai.com listing.)
#pragma once
#include "common.cuh"

namespace ttt {

// Up to four [BH][T][row_bytes] tensors copied with the token order reversed
// within every (b, h): dst[bh][T-1-t] = src[bh][t].  Rows are whole 16-byte
// units (row_bytes a multiple of 16).
struct ReverseParams {
  int n, BH, T, units;  // tensors, sequences, tokens, 16-byte units per row
  const uint4* src[4];
  uint4* dst[4];
};

__global__ void __launch_bounds__(256) reverse_tokens_kernel(const ReverseParams p) {
  const long long per = static_cast<long long>(p.BH) * p.T * p.units;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < per; i += stride) {
    const long long row = i / p.units;  // bh * T + t
    const int u = static_cast<int>(i - row * p.units);
    const long long bh = row / p.T;
    const int t = static_cast<int>(row - bh * p.T);
    const long long o = (bh * p.T + (p.T - 1 - t)) * p.units + u;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (j < p.n) p.dst[j][o] = __ldcs(p.src[j] + i);
  }
}

// Up to four [BH][R][C] fp32 matrices transposed to [BH][C][R].
struct TransposeParams {
  int n, BH, R, C;
  const float* src[4];
  float* dst[4];
  float* zero;       // zeroed here as well (zero_n floats), or nullptr
  long long zero_n;
};

__global__ void __launch_bounds__(256) transpose_states_kernel(const TransposeParams p) {
  const long long per = static_cast<long long>(p.BH) * p.R * p.C;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < per; i += stride) {
    const long long bh = i / (static_cast<long long>(p.R) * p.C);
    const int rc = static_cast<int>(i - bh * p.R * p.C);
    const int r = rc / p.C, c = rc % p.C;
    const long long o = bh * p.R * p.C + static_cast<long long>(c) * p.R + r;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (j < p.n) p.dst[j][o] = p.src[j][i];
  }
  if (p.zero)
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < p.zero_n; i += stride)
      p.zero[i] = 0.f;
}

// dv_t = sigma eta_t u_t, dk_t = sigma eta_t r_t, deta_t = sigma v_t . u_t,
// with u and r stored in fp32 in reversed token order (the fp32 path).  One
// warp per (b, h, t).
struct FinishParams {
  int BH, T, dk, dv;
  const float* u_rev; // [BH][T][dv]
  const float* r_rev; // [BH][T][dk]
  const float* v;     // [BH][T][dv]
  const float* eta;   // [BH][T] or nullptr
  float eta_const, sigma;
  float* dk_out;      // [BH][T][dk]
  float* dv_out;      // [BH][T][dv]
  float* deta;        // [BH][T] or nullptr
};

__global__ void __launch_bounds__(256) backward_finish_kernel(const FinishParams p) {
  const long long warp = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= static_cast<long long>(p.BH) * p.T) return;
  const long long bh = warp / p.T;
  const int t = static_cast<int>(warp - bh * p.T);
  const long long fwd = warp, rev = bh * p.T + (p.T - 1 - t);
  const float s = p.sigma * (p.eta ? p.eta[fwd] : p.eta_const);
  const float* u = p.u_rev + rev * p.dv;
  const float* r = p.r_rev + rev * p.dk;
  const float* v = p.v + fwd * p.dv;
  float* dv = p.dv_out + fwd * p.dv;
  float* dk = p.dk_out + fwd * p.dk;
  float vu = 0.f;
  for (int c = lane; c < p.dv; c += 32) {
    const float uc = u[c];
    vu = fmaf(v[c], uc, vu);
    dv[c] = s * uc;
  }
  for (int c = lane; c < p.dk; c += 32) dk[c] = s * r[c];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) vu += __shfl_xor_sync(0xffffffffu, vu, off);
  if (lane == 0 && p.deta) p.deta[fwd] = p.sigma * vu;
}

}  // namespace ttt
