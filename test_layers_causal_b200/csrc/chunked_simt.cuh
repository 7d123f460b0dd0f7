// chunked_simt.cuh -- chunk-parallel forward in fp32 FMA for fp32 inputs.
//
// The layer in its chunked form ("fully parallel formulations", abstract of
// "Test-Time Training with KV Binding Is Secretly Linear Attention"; the
// linear-attention regrouping of the kualia.ai explainer, section "The Linear
// Attention Equivalence").  For a chunk of n tokens with local indices i, j:
//   A_ij = c_ij (q_i . k_j) for j <= i, 0 otherwise
//   o_i  = sigma sum_j A_ij v_j + W q_i - g_i M q_i
//   W'   = W - g_{n-1} M + sigma sum_j c_{n-1,j} v_j k_j^T
//   M'   = beta^n M - sigma sum_j beta^(n-1-j) v_j k_j^T
// where c_ij = eta_j without momentum (g = 0, M unused) and, with momentum,
// c_ij = eta_j + beta c_{i,j+1}, c_ii = eta_i, g_i = beta c_{i,0}.
//
// fp32 inputs promise 1e-4 relative accuracy, which a single tf32 tensor-core
// pass cannot give, so this path is plain fp32 FMA: one block per (b, h)
// walks the chunks in order with Q, K, V, the score tile and the state in
// shared memory.  It serves small fp32 layers; bf16 layers use the tensor-core
// path.
#pragma once
#include "common.cuh"
#include "recurrent.cuh"  // SeqParams

namespace ttt {

struct SimtShape {
  int C, dk, dv;
  bool mom;
  __host__ __device__ int ldq() const { return dk + 1; }
  __host__ __device__ int ldv() const { return dv + 1; }
  __host__ __device__ int lda() const { return C + 1; }
  __host__ __device__ size_t floats() const {
    size_t f = static_cast<size_t>(C) * ldq() * 2 + static_cast<size_t>(C) * ldv() + static_cast<size_t>(C) * lda() +
               static_cast<size_t>(dv) * dk * (mom ? 2 : 1) + 4 * static_cast<size_t>(C) + 4;
    return f;
  }
  __host__ __device__ size_t bytes() const { return floats() * sizeof(float); }
};

template <bool MOM>
__global__ void __launch_bounds__(256) chunked_simt_f32_kernel(const SeqParams p, const SimtShape sh) {
  extern __shared__ __align__(16) float sm[];
  const int C = sh.C, dk = sh.dk, dv = sh.dv;
  const int ldq = sh.ldq(), ldv = sh.ldv(), lda = sh.lda();
  float* Qs = sm;
  float* Ks = Qs + C * ldq;
  float* Vs = Ks + C * ldq;
  float* As = Vs + C * ldv;
  float* Ws = As + C * lda;
  float* Ms = Ws + dv * dk;                 // momentum only
  float* es = Ms + (MOM ? dv * dk : 0);     // eta of the chunk
  float* cl = es + C;                       // c_{n-1, j}
  float* gs = cl + C;                       // g_i
  float* bp = gs + C;                       // beta^j, j = 0..C

  const int bh = blockIdx.x;
  const int tid = threadIdx.x, nt = blockDim.x;
  const float* qg = static_cast<const float*>(p.q) + static_cast<size_t>(bh) * p.T * dk;
  const float* kg = static_cast<const float*>(p.k) + static_cast<size_t>(bh) * p.T * dk;
  const float* vg = static_cast<const float*>(p.v) + static_cast<size_t>(bh) * p.T * dv;
  const float* eg = p.eta ? p.eta + static_cast<size_t>(bh) * p.T : nullptr;
  float* og = static_cast<float*>(p.o) + static_cast<size_t>(bh) * p.T * dv;
  const float sigma = p.sigma, beta = p.beta;

  for (int i = tid; i < dv * dk; i += nt) {
    Ws[i] = p.S_in ? p.S_in[static_cast<size_t>(bh) * dv * dk + i] : 0.f;
    if (MOM) Ms[i] = p.M_in ? p.M_in[static_cast<size_t>(bh) * dv * dk + i] : 0.f;
  }
  if (MOM && tid == 0) {
    float b = 1.f;
    for (int j = 0; j <= C; ++j) {
      bp[j] = b;
      b *= beta;
    }
  }

  for (int t0 = 0; t0 < p.T; t0 += C) {
    const int n = min(C, p.T - t0);
    __syncthreads();
    for (int i = tid; i < C * dk; i += nt) {
      const int r = i / dk, c = i % dk;
      const bool ok = r < n;
      Qs[r * ldq + c] = ok ? qg[static_cast<size_t>(t0 + r) * dk + c] : 0.f;
      Ks[r * ldq + c] = ok ? kg[static_cast<size_t>(t0 + r) * dk + c] : 0.f;
    }
    for (int i = tid; i < C * dv; i += nt) {
      const int r = i / dv, c = i % dv;
      Vs[r * ldv + c] = r < n ? vg[static_cast<size_t>(t0 + r) * dv + c] : 0.f;
    }
    for (int i = tid; i < C; i += nt) es[i] = i < n ? (eg ? eg[t0 + i] : p.eta_const) : 0.f;
    __syncthreads();

    // raw scores q_i . k_j for j <= i
    for (int e = tid; e < C * C; e += nt) {
      const int i = e / C, j = e % C;
      float acc = 0.f;
      if (j <= i && i < n) {
        for (int c = 0; c < dk; ++c) acc = fmaf(Qs[i * ldq + c], Ks[j * ldq + c], acc);
      }
      As[i * lda + j] = acc;
    }
    __syncthreads();
    // coefficients: one thread per query row
    for (int i = tid; i < C; i += nt) {
      if (!MOM) {
        for (int j = 0; j <= i && i < n; ++j) As[i * lda + j] *= sigma * es[j];
        if (i < n) cl[i] = es[i];
        gs[i] = 0.f;
      } else {
        float c = 0.f;
        if (i < n) {
          for (int j = i; j >= 0; --j) {
            c = es[j] + beta * c;
            As[i * lda + j] *= sigma * c;
            if (i == n - 1) cl[j] = c;
          }
        }
        gs[i] = beta * c;
      }
    }
    __syncthreads();
    // outputs
    for (int e = tid; e < n * dv; e += nt) {
      const int i = e / dv, col = e % dv;
      float acc = 0.f;
      for (int j = 0; j <= i; ++j) acc = fmaf(As[i * lda + j], Vs[j * ldv + col], acc);
      float sw = 0.f, sm2 = 0.f;
      for (int c = 0; c < dk; ++c) {
        sw = fmaf(Ws[col * dk + c], Qs[i * ldq + c], sw);
        if (MOM) sm2 = fmaf(Ms[col * dk + c], Qs[i * ldq + c], sm2);
      }
      og[static_cast<size_t>(t0 + i) * dv + col] = acc + sw - (MOM ? gs[i] * sm2 : 0.f);
    }
    __syncthreads();
    // carried state
    for (int e = tid; e < dv * dk; e += nt) {
      const int col = e / dk, c = e % dk;
      float dw = 0.f, dm = 0.f;
      for (int j = 0; j < n; ++j) {
        const float vk = Vs[j * ldv + col] * Ks[j * ldq + c];
        dw = fmaf(cl[j], vk, dw);
        if (MOM) dm = fmaf(bp[n - 1 - j], vk, dm);
      }
      if (MOM) {
        const float mo = Ms[e];
        Ws[e] = Ws[e] - gs[n - 1] * mo + sigma * dw;
        Ms[e] = bp[n] * mo - sigma * dm;
      } else {
        Ws[e] += sigma * dw;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < dv * dk; i += nt) {
    if (p.S_out) p.S_out[static_cast<size_t>(bh) * dv * dk + i] = Ws[i];
    if (MOM && p.M_out) p.M_out[static_cast<size_t>(bh) * dv * dk + i] = Ms[i];
  }
}

}  // namespace ttt
