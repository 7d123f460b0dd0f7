// decode.cuh -- one decode step of the TTT layer for N sequences x H heads.
//
// For every (n, h) the fast weight W (d_v x d_k fp32) takes the single-token
// gradient step on the key-value binding loss and is read out with the query
// (Table 2 of the thelatestinai.com listing of "Test-Time Training with KV
// Binding Is Secretly Linear Attention", Variants 3-5; recurrent form):
//   plain:    W += sigma * eta * v k^T
//   momentum: M  = beta * M - sigma * v k^T ;  W -= eta * M
//   o = W q
// The state is far larger than L2 (256 MiB at 256 x 16 heads x 128 x 128), so
// the step is a pure HBM stream: every element of W (and M) is read once and
// written once with 16-byte streaming accesses (ld.global.cs / st.global.cs).
//
// Work decomposition: the rows of all W matrices form one flat list of
// N*H*d_v rows of d_k floats.  A row is owned by TPR = d_k/4 consecutive
// lanes, each holding one float4; a warp covers 32/TPR rows per pass and U
// passes per iteration (U independent 16-byte loads in flight per lane),
// striding over the list so that every SM stays busy to the end.
#pragma once
#include "common.cuh"

namespace ttt {

struct DecodeParams {
  int N, H, dk, dv;
  const void* q;
  const void* k;
  const void* v;
  const float* eta;
  float eta_const, beta, sigma;
  float* S;
  float* M;
  void* o;
};

template <int DK, typename T, bool MOM, int U>
__global__ void __launch_bounds__(256) decode_step_kernel(const DecodeParams p) {
  constexpr int TPR = DK / 4;   // lanes per row
  constexpr int RPW = 32 / TPR; // rows per warp per pass
  constexpr int STEP = RPW * U; // rows per warp per iteration
  const int lane = threadIdx.x & 31;
  const int sub = lane / TPR, c4 = lane % TPR;
  const int rows = p.N * p.H * p.dv;  // host guarantees < 2^31
  const int warp_gid = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  const T* qg = static_cast<const T*>(p.q);
  const T* kg = static_cast<const T*>(p.k);
  const T* vg = static_cast<const T*>(p.v);
  T* og = static_cast<T*>(p.o);

  for (int base = warp_gid * STEP; base < rows; base += nwarps * STEP) {
    float4 s[U], m[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * RPW + sub;
      if (row < rows) {
        s[u] = __ldcs(reinterpret_cast<const float4*>(p.S + static_cast<size_t>(row) * DK) + c4);
        if (MOM) m[u] = __ldcs(reinterpret_cast<const float4*>(p.M + static_cast<size_t>(row) * DK) + c4);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * RPW + sub;
      float dot = 0.f;
      if (row < rows) {
        const int head = row / p.dv;
        const float4 kk = load4(kg + static_cast<size_t>(head) * DK + 4 * c4);
        const float4 qq = load4(qg + static_cast<size_t>(head) * DK + 4 * c4);
        const float vv = to_f(vg[row]);  // v is [N,H,d_v]: flat index == row
        const float eta = p.eta ? p.eta[head] : p.eta_const;
        float4 w = s[u];
        if (MOM) {
          const float g = -p.sigma * vv;  // gradient row factor: grad = -sigma v k^T
          float4 mm = m[u];
          mm.x = fmaf(p.beta, mm.x, g * kk.x);
          mm.y = fmaf(p.beta, mm.y, g * kk.y);
          mm.z = fmaf(p.beta, mm.z, g * kk.z);
          mm.w = fmaf(p.beta, mm.w, g * kk.w);
          w.x = fmaf(-eta, mm.x, w.x);
          w.y = fmaf(-eta, mm.y, w.y);
          w.z = fmaf(-eta, mm.z, w.z);
          w.w = fmaf(-eta, mm.w, w.w);
          __stcs(reinterpret_cast<float4*>(p.M + static_cast<size_t>(row) * DK) + c4, mm);
        } else {
          const float a = p.sigma * eta * vv;
          w.x = fmaf(a, kk.x, w.x);
          w.y = fmaf(a, kk.y, w.y);
          w.z = fmaf(a, kk.z, w.z);
          w.w = fmaf(a, kk.w, w.w);
        }
        __stcs(reinterpret_cast<float4*>(p.S + static_cast<size_t>(row) * DK) + c4, w);
        dot = w.x * qq.x + w.y * qq.y + w.z * qq.z + w.w * qq.w;
      }
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      if (row < rows && c4 == 0) og[row] = from_f<T>(dot);
    }
  }
}

}  // namespace ttt
