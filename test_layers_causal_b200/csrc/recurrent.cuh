// recurrent.cuh -- token-by-token forward of the TTT layer ("Recurrent
// Impl." column of Table 2 in the thelatestinai.com listing of "Test-Time
// Training with KV Binding Is Secretly Linear Attention").
//
// Each (b, h) sequence is split over blocks by rows of W: row n of W only
// ever meets feature n of v and produces feature n of o, so rows are
// independent.  Within a block a row is held in registers by TPR = d_k/4
// lanes (one float4 each; the momentum buffer likewise), and every thread
// owns RPT rows so that RPT dot-product reductions overlap.  Tokens are
// staged through shared memory TB at a time.  Arithmetic is fp32 throughout.
#pragma once
#include "common.cuh"

namespace ttt {

struct SeqParams {
  int B, H, T, dk, dv;
  const void* q;
  const void* k;
  const void* v;
  const float* eta;
  float eta_const, beta, sigma;
  const float* S_in;
  float* S_out;
  const float* M_in;
  float* M_out;
  void* o;
};

template <int DK>
struct RecurrentShape {
  static constexpr int TPR = DK / 4, RPW = 32 / TPR, RPT = 4, WARPS = 4;
  static constexpr int ROWS = WARPS * RPW * RPT;  // rows of W per block
  static constexpr int TB = 32;                   // tokens per staging step
};

template <int DK, typename T, bool MOM>
__global__ void __launch_bounds__(128) recurrent_kernel(const SeqParams p) {
  using Sh = RecurrentShape<DK>;
  constexpr int TPR = Sh::TPR, RPW = Sh::RPW, RPT = Sh::RPT, ROWS = Sh::ROWS, TB = Sh::TB;
  __shared__ __align__(16) float qs[TB][DK];
  __shared__ __align__(16) float ks[TB][DK];
  __shared__ float vs[TB][ROWS];
  __shared__ float es[TB];

  const int bh = blockIdx.x;
  const int row0 = blockIdx.y * ROWS;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / TPR, c4 = lane % TPR;
  const T* qg = static_cast<const T*>(p.q) + static_cast<size_t>(bh) * p.T * DK;
  const T* kg = static_cast<const T*>(p.k) + static_cast<size_t>(bh) * p.T * DK;
  const T* vg = static_cast<const T*>(p.v) + static_cast<size_t>(bh) * p.T * p.dv;
  const float* eg = p.eta ? p.eta + static_cast<size_t>(bh) * p.T : nullptr;
  T* og = static_cast<T*>(p.o) + static_cast<size_t>(bh) * p.T * p.dv;

  int lrow[RPT];  // row within the block
  float4 w[RPT], m[RPT];
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    lrow[u] = (warp * RPT + u) * RPW + sub;
    const int row = row0 + lrow[u];
    w[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    m[u] = w[u];
    if (row < p.dv) {
      const size_t off = (static_cast<size_t>(bh) * p.dv + row) * DK + 4 * c4;
      if (p.S_in) w[u] = *reinterpret_cast<const float4*>(p.S_in + off);
      if (MOM && p.M_in) m[u] = *reinterpret_cast<const float4*>(p.M_in + off);
    }
  }

  for (int t0 = 0; t0 < p.T; t0 += TB) {
    const int n = min(TB, p.T - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < TB * (DK / 4); i += blockDim.x) {
      const int t = i / (DK / 4), c = i % (DK / 4);
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (t < n) {
        a = load4(qg + static_cast<size_t>(t0 + t) * DK + 4 * c);
        b = load4(kg + static_cast<size_t>(t0 + t) * DK + 4 * c);
      }
      *reinterpret_cast<float4*>(&qs[t][4 * c]) = a;
      *reinterpret_cast<float4*>(&ks[t][4 * c]) = b;
    }
    for (int i = threadIdx.x; i < TB * ROWS; i += blockDim.x) {
      const int t = i / ROWS, r = i % ROWS;
      vs[t][r] = (t < n && row0 + r < p.dv) ? to_f(vg[static_cast<size_t>(t0 + t) * p.dv + row0 + r]) : 0.f;
    }
    if (threadIdx.x < TB) es[threadIdx.x] = (threadIdx.x < n) ? (eg ? eg[t0 + threadIdx.x] : p.eta_const) : 0.f;
    __syncthreads();

    for (int t = 0; t < n; ++t) {
      const float4 kk = *reinterpret_cast<const float4*>(&ks[t][4 * c4]);
      const float4 qq = *reinterpret_cast<const float4*>(&qs[t][4 * c4]);
      const float eta = es[t];
      float dot[RPT];
#pragma unroll
      for (int u = 0; u < RPT; ++u) {
        const float vv = vs[t][lrow[u]];
        if (MOM) {
          const float g = -p.sigma * vv;
          m[u].x = fmaf(p.beta, m[u].x, g * kk.x);
          m[u].y = fmaf(p.beta, m[u].y, g * kk.y);
          m[u].z = fmaf(p.beta, m[u].z, g * kk.z);
          m[u].w = fmaf(p.beta, m[u].w, g * kk.w);
          w[u].x = fmaf(-eta, m[u].x, w[u].x);
          w[u].y = fmaf(-eta, m[u].y, w[u].y);
          w[u].z = fmaf(-eta, m[u].z, w[u].z);
          w[u].w = fmaf(-eta, m[u].w, w[u].w);
        } else {
          const float a = p.sigma * eta * vv;
          w[u].x = fmaf(a, kk.x, w[u].x);
          w[u].y = fmaf(a, kk.y, w[u].y);
          w[u].z = fmaf(a, kk.z, w[u].z);
          w[u].w = fmaf(a, kk.w, w[u].w);
        }
        dot[u] = w[u].x * qq.x + w[u].y * qq.y + w[u].z * qq.z + w[u].w * qq.w;
      }
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) {
#pragma unroll
        for (int u = 0; u < RPT; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], off);
      }
      if (c4 == 0) {
#pragma unroll
        for (int u = 0; u < RPT; ++u) {
          const int row = row0 + lrow[u];
          if (row < p.dv) og[static_cast<size_t>(t0 + t) * p.dv + row] = from_f<T>(dot[u]);
        }
      }
    }
  }

#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    const int row = row0 + lrow[u];
    if (row < p.dv) {
      const size_t off = (static_cast<size_t>(bh) * p.dv + row) * DK + 4 * c4;
      if (p.S_out) *reinterpret_cast<float4*>(p.S_out + off) = w[u];
      if (MOM && p.M_out) *reinterpret_cast<float4*>(p.M_out + off) = m[u];
    }
  }
}

}  // namespace ttt
