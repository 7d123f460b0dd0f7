// backward.cuh -- token-by-token backward of the TTT layer (the gradient
// needed to train it, Figure 4 of the thelatestinai.com listing of
// "Test-Time Training with KV Binding Is Secretly Linear Attention").
//
// Forward (update, then read; sigma = +1 descent, -1 ascent):
//   momentum:  M_t = beta M_{t-1} - sigma v_t k_t^T ;  W_t = W_{t-1} - eta_t M_t
//   plain:     W_t = W_{t-1} + sigma eta_t v_t k_t^T
//   o_t = W_t q_t
// Backward over the tokens in reverse, with G_t = dL/dW_t and H_t = dL/dM_t:
//   G_t = G_{t+1} + do_t q_t^T                       (G_{T+1} = dL/dW_T)
//   H_t = beta H_{t+1} - eta_t G_t,  H_T = dL/dM_T - eta_T G_T
//   dq_t = W_t^T do_t
//   momentum: dv_t = -sigma H_t k_t,  dk_t = -sigma H_t^T v_t,  deta_t = -<G_t, M_t>
//   plain:    dv_t = sigma eta_t G_t k_t,  dk_t = sigma eta_t G_t^T v_t,
//             deta_t = sigma v_t^T G_t k_t
//   dW_0 = G_1,  dM_0 = beta H_1.
//
// One block per (b, h): dq, dk and deta sum over the rows of W, so all rows
// live in one block.  A row is held by TPR = d_k / 4 lanes (one float4 each)
// and every thread owns RPT rows, as in the recurrent forward.  The states
// W_t, M_t are needed in reverse order; undoing the momentum update would
// divide by beta and amplify rounding, so the kernel replays instead:
//   sweep 1: forward over the sequence, saving (W, M) at the start of every
//            chunk of CK tokens (workspace);
//   sweep 2: chunks in reverse; each is replayed from its checkpoint, every
//            thread writing its own rows of W_t (and M_t) for the chunk's
//            tokens to a per-block history (workspace) that it alone reads
//            back, then walked backwards.
// Per token, the row sums of dq and dk are reduced across the warp with
// shuffles and across warps with shared-memory atomics.  fp32 throughout.
#pragma once
#include "common.cuh"

namespace ttt {

struct BwdParams {
  int BH, T, dk, dv;
  const void* q;
  const void* k;
  const void* v;
  const float* eta;
  float eta_const, beta, sigma;
  const float* S_in;
  const float* M_in;
  const void* dO;
  const float* dS;  // dL/dW_T or nullptr
  const float* dM;  // dL/dM_T or nullptr
  void* dq;
  void* dk_out;
  void* dv_out;
  float* deta;      // or nullptr
  float* dS_in;     // or nullptr
  float* dM_in;     // or nullptr
  float* ckpt;      // [BH][nck][NS][dv][dk]
  float* hist;      // [BH][CK][NS][dv][dk]
  int nck;
};

template <int DK>
struct BwdShape {
  static constexpr int TPR = DK / 4, RPW = 32 / TPR, RPT = 4;
  static constexpr int CK = 32;  // tokens per checkpoint chunk
  static constexpr int ROWS_PER_WARP = RPW * RPT;
};

// Shared floats of one block: q, k, dq, dk [CK][DK]; v, dO [CK][dv]; eta, deta [CK].
__host__ __device__ inline size_t bwd_smem_floats(int DK, int dv, int CK) {
  return static_cast<size_t>(CK) * (4 * DK + 2 * dv + 2);
}

__device__ __forceinline__ float4 f4_fma(float a, float4 x, float4 y) {
  return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}
__device__ __forceinline__ float f4_dot(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }

template <int DK, typename T, bool MOM>
__global__ void __launch_bounds__(1024) backward_recurrent_kernel(const BwdParams p) {
  using Sh = BwdShape<DK>;
  constexpr int TPR = Sh::TPR, RPW = Sh::RPW, RPT = Sh::RPT, CK = Sh::CK;
  constexpr int NS = MOM ? 2 : 1;
  extern __shared__ __align__(16) float bsm[];
  float* qs = bsm;               // [CK][DK]
  float* ks = qs + CK * DK;      // [CK][DK]
  float* dqs = ks + CK * DK;     // [CK][DK]
  float* dks = dqs + CK * DK;    // [CK][DK]
  float* vs = dks + CK * DK;     // [CK][dv]
  float* dos = vs + CK * p.dv;   // [CK][dv]
  float* es = dos + CK * p.dv;   // [CK]
  float* des = es + CK;          // [CK]

  const int bh = blockIdx.x, dv = p.dv, nT = p.T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / TPR, c4 = lane % TPR;
  const size_t DD = static_cast<size_t>(dv) * DK;
  const T* qg = static_cast<const T*>(p.q) + static_cast<size_t>(bh) * nT * DK;
  const T* kg = static_cast<const T*>(p.k) + static_cast<size_t>(bh) * nT * DK;
  const T* vg = static_cast<const T*>(p.v) + static_cast<size_t>(bh) * nT * dv;
  const T* dog = static_cast<const T*>(p.dO) + static_cast<size_t>(bh) * nT * dv;
  const float* eg = p.eta ? p.eta + static_cast<size_t>(bh) * nT : nullptr;
  float* ck = p.ckpt + static_cast<size_t>(bh) * p.nck * NS * DD;
  float* hs = p.hist + static_cast<size_t>(bh) * CK * NS * DD;

  int row[RPT];
  bool ok[RPT];
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    row[u] = (warp * RPT + u) * RPW + sub;
    ok[u] = row[u] < dv;
  }
  // float4 index of this lane's part of row r in a [dv][DK] matrix
  auto at = [&](int r) { return static_cast<size_t>(r) * (DK / 4) + c4; };
  auto ld4 = [&](const float* base, int u) {
    return ok[u] ? reinterpret_cast<const float4*>(base)[at(row[u])] : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto st4 = [&](float* base, int u, float4 x) {
    if (ok[u]) reinterpret_cast<float4*>(base)[at(row[u])] = x;
  };

  // Stages the chunk [t0, t0 + n) (k, v, eta always; q and dO for sweep 2)
  // and clears the per-token sums.
  auto stage = [&](int t0, int n, bool back) {
    for (int i = threadIdx.x; i < CK * (DK / 4); i += blockDim.x) {
      const int t = i / (DK / 4), c = i % (DK / 4);
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      reinterpret_cast<float4*>(ks)[i] = t < n ? load4(kg + static_cast<size_t>(t0 + t) * DK + 4 * c) : z;
      if (back) {
        reinterpret_cast<float4*>(qs)[i] = t < n ? load4(qg + static_cast<size_t>(t0 + t) * DK + 4 * c) : z;
        reinterpret_cast<float4*>(dqs)[i] = z;
        reinterpret_cast<float4*>(dks)[i] = z;
      }
    }
    for (int i = threadIdx.x; i < CK * dv; i += blockDim.x) {
      const int t = i / dv, r = i % dv;
      vs[i] = t < n ? to_f(vg[static_cast<size_t>(t0 + t) * dv + r]) : 0.f;
      if (back) dos[i] = t < n ? to_f(dog[static_cast<size_t>(t0 + t) * dv + r]) : 0.f;
    }
    if (threadIdx.x < CK) {
      es[threadIdx.x] = threadIdx.x < n ? (eg ? eg[t0 + threadIdx.x] : p.eta_const) : 0.f;
      des[threadIdx.x] = 0.f;
    }
  };
  // One forward token (index j of the staged chunk) on this thread's rows.
  auto step = [&](int j, float4 (&w)[RPT], float4 (&m)[RPT]) {
    const float4 kk = reinterpret_cast<const float4*>(ks + j * DK)[c4];
    const float eta = es[j];
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
      const float vv = ok[u] ? vs[j * dv + row[u]] : 0.f;
      if (MOM) {
        m[u] = f4_fma(-p.sigma * vv, kk, make_float4(p.beta * m[u].x, p.beta * m[u].y, p.beta * m[u].z,
                                                     p.beta * m[u].w));
        w[u] = f4_fma(-eta, m[u], w[u]);
      } else {
        w[u] = f4_fma(p.sigma * eta * vv, kk, w[u]);
      }
    }
  };

  float4 w[RPT], m[RPT];
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    w[u] = p.S_in ? ld4(p.S_in + static_cast<size_t>(bh) * DD, u) : make_float4(0.f, 0.f, 0.f, 0.f);
    m[u] = (MOM && p.M_in) ? ld4(p.M_in + static_cast<size_t>(bh) * DD, u) : make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // ---- sweep 1: checkpoints of (W, M) at every chunk start ----
  for (int c = 0; c < p.nck; ++c) {
    const int t0 = c * CK, n = min(CK, nT - t0);
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
      st4(ck + (static_cast<size_t>(c) * NS) * DD, u, w[u]);
      if (MOM) st4(ck + (static_cast<size_t>(c) * NS + 1) * DD, u, m[u]);
    }
    __syncthreads();
    stage(t0, n, false);
    __syncthreads();
    for (int j = 0; j < n; ++j) step(j, w, m);
  }

  // ---- sweep 2: chunks in reverse ----
  float4 g[RPT], h[RPT];
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    g[u] = p.dS ? ld4(p.dS + static_cast<size_t>(bh) * DD, u) : make_float4(0.f, 0.f, 0.f, 0.f);
    h[u] = (MOM && p.dM) ? ld4(p.dM + static_cast<size_t>(bh) * DD, u) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float hscale = 1.f;  // H_T starts from dL/dM_T itself; later tokens scale by beta
  T* dqg = static_cast<T*>(p.dq) + static_cast<size_t>(bh) * nT * DK;
  T* dkg = static_cast<T*>(p.dk_out) + static_cast<size_t>(bh) * nT * DK;
  T* dvg = static_cast<T*>(p.dv_out) + static_cast<size_t>(bh) * nT * dv;
  float* deg = p.deta ? p.deta + static_cast<size_t>(bh) * nT : nullptr;

  for (int c = p.nck - 1; c >= 0; --c) {
    const int t0 = c * CK, n = min(CK, nT - t0);
    __syncthreads();
    stage(t0, n, true);
    __syncthreads();
    // replay the chunk from its checkpoint into this thread's history rows
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
      w[u] = ld4(ck + (static_cast<size_t>(c) * NS) * DD, u);
      if (MOM) m[u] = ld4(ck + (static_cast<size_t>(c) * NS + 1) * DD, u);
    }
    for (int j = 0; j < n; ++j) {
      step(j, w, m);
#pragma unroll
      for (int u = 0; u < RPT; ++u) {
        st4(hs + (static_cast<size_t>(j) * NS) * DD, u, w[u]);
        if (MOM) st4(hs + (static_cast<size_t>(j) * NS + 1) * DD, u, m[u]);
      }
    }
    // walk it backwards
    for (int j = n - 1; j >= 0; --j) {
      const float4 qq = reinterpret_cast<const float4*>(qs + j * DK)[c4];
      const float4 kk = reinterpret_cast<const float4*>(ks + j * DK)[c4];
      const float eta = es[j];
      float4 aq = make_float4(0.f, 0.f, 0.f, 0.f), ak = aq;
      float ae = 0.f;
      float rdot[RPT];
#pragma unroll
      for (int u = 0; u < RPT; ++u) {
        const float dov = ok[u] ? dos[j * dv + row[u]] : 0.f;
        const float vv = ok[u] ? vs[j * dv + row[u]] : 0.f;
        const float4 wt = ld4(hs + (static_cast<size_t>(j) * NS) * DD, u);
        g[u] = f4_fma(dov, qq, g[u]);  // G_t = G_{t+1} + do_t q_t^T
        aq = f4_fma(dov, wt, aq);      // (W_t^T do_t), this thread's rows
        if (MOM) {
          const float4 mt = ld4(hs + (static_cast<size_t>(j) * NS + 1) * DD, u);
          h[u] = f4_fma(-eta, g[u], make_float4(hscale * h[u].x, hscale * h[u].y, hscale * h[u].z,
                                                 hscale * h[u].w));
          rdot[u] = f4_dot(h[u], kk);  // (H_t k_t)[row], partial over this lane's columns
          ak = f4_fma(vv, h[u], ak);   // (H_t^T v_t)
          ae += f4_dot(g[u], mt);      // <G_t, M_t>
        } else {
          rdot[u] = f4_dot(g[u], kk);  // (G_t k_t)[row], partial
          ak = f4_fma(vv, g[u], ak);   // (G_t^T v_t)
        }
      }
      hscale = p.beta;
      // complete the row dot products over the row's TPR lanes
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1)
#pragma unroll
        for (int u = 0; u < RPT; ++u) rdot[u] += __shfl_xor_sync(0xffffffffu, rdot[u], off);
#pragma unroll
      for (int u = 0; u < RPT; ++u) {
        if (!MOM && c4 == 0) ae += (ok[u] ? vs[j * dv + row[u]] : 0.f) * rdot[u];  // v_t^T G_t k_t
        if (c4 == 0 && ok[u]) {
          const float dvv = MOM ? -p.sigma * rdot[u] : p.sigma * eta * rdot[u];
          dvg[static_cast<size_t>(t0 + j) * dv + row[u]] = from_f<T>(dvv);
        }
      }
      // sums over rows: lanes with equal c4 first, then across warps
#pragma unroll
      for (int off = TPR; off < 32; off <<= 1) {
        aq.x += __shfl_xor_sync(0xffffffffu, aq.x, off);
        aq.y += __shfl_xor_sync(0xffffffffu, aq.y, off);
        aq.z += __shfl_xor_sync(0xffffffffu, aq.z, off);
        aq.w += __shfl_xor_sync(0xffffffffu, aq.w, off);
        ak.x += __shfl_xor_sync(0xffffffffu, ak.x, off);
        ak.y += __shfl_xor_sync(0xffffffffu, ak.y, off);
        ak.z += __shfl_xor_sync(0xffffffffu, ak.z, off);
        ak.w += __shfl_xor_sync(0xffffffffu, ak.w, off);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ae += __shfl_xor_sync(0xffffffffu, ae, off);
      if (sub == 0) {
        float* dq4 = dqs + j * DK + 4 * c4;
        float* dk4 = dks + j * DK + 4 * c4;
        atomicAdd(dq4 + 0, aq.x);
        atomicAdd(dq4 + 1, aq.y);
        atomicAdd(dq4 + 2, aq.z);
        atomicAdd(dq4 + 3, aq.w);
        atomicAdd(dk4 + 0, ak.x);
        atomicAdd(dk4 + 1, ak.y);
        atomicAdd(dk4 + 2, ak.z);
        atomicAdd(dk4 + 3, ak.w);
      }
      if (lane == 0) atomicAdd(des + j, ae);
    }
    __syncthreads();
    // the chunk's dq, dk, deta
    for (int i = threadIdx.x; i < n * DK; i += blockDim.x) {
      const int j = i / DK;
      const float sk = MOM ? -p.sigma : p.sigma * es[j];
      dqg[static_cast<size_t>(t0) * DK + i] = from_f<T>(dqs[i]);
      dkg[static_cast<size_t>(t0) * DK + i] = from_f<T>(sk * dks[i]);
    }
    if (deg && static_cast<int>(threadIdx.x) < n)
      deg[t0 + threadIdx.x] = MOM ? -des[threadIdx.x] : p.sigma * des[threadIdx.x];
  }

#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    if (p.dS_in) st4(p.dS_in + static_cast<size_t>(bh) * DD, u, g[u]);  // dW_0 = G_1
    if (MOM && p.dM_in)                                                  // dM_0 = beta H_1
      st4(p.dM_in + static_cast<size_t>(bh) * DD, u,
          make_float4(p.beta * h[u].x, p.beta * h[u].y, p.beta * h[u].z, p.beta * h[u].w));
  }
  if (!MOM && p.dM_in) {
#pragma unroll
    for (int u = 0; u < RPT; ++u) st4(p.dM_in + static_cast<size_t>(bh) * DD, u, make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

}  // namespace ttt
