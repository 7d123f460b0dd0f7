// host_pipeline.h -- the chunked forward with host buffers: the sequences are
// cut into pieces, and piece j's host-to-device copy, piece j-1's forward and
// piece j-2's device-to-host copy run at the same time on three streams
// (copy-in, the caller's stream, copy-out), through two sets of device
// staging buffers.  Included once, by ttt_la.cu (host code only).
#pragma once

namespace {

struct HostPipe {
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t fork = nullptr, join_in = nullptr, join_out = nullptr;
  cudaEvent_t in_ready[2] = {}, done[2] = {}, out_done[2] = {};
  std::mutex mu;  // one enqueue at a time per device (the events are shared)
};

// The device's pipe, created on first use and kept for the process.
HostPipe* host_pipe() {
  static std::mutex mu;
  static HostPipe* pipes[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (pipes[dev]) return pipes[dev];
  HostPipe* p = new HostPipe();
  bool ok = cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking) == cudaSuccess;
  cudaEvent_t* evs[] = {&p->fork, &p->join_in, &p->join_out, &p->in_ready[0], &p->in_ready[1],
                        &p->done[0], &p->done[1], &p->out_done[0], &p->out_done[1]};
  for (cudaEvent_t* e : evs) ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) return nullptr;  // leaks what was created; the call reports TTT_LA_ERR_CUDA
  pipes[dev] = p;
  return p;
}

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// Offsets of one staging set (all 256-byte aligned) for pieces of `per` sequences.
struct PieceLayout {
  int per = 0, pieces = 0;
  size_t q = 0, k = 0, v = 0, o = 0, eta = 0, s_in = 0, s_out = 0, m_in = 0, m_out = 0, ws = 0, ws_bytes = 0;
  size_t set_bytes = 0;
};

// Device-side arguments of a piece of `cnt` sequences at staging offset `base`
// (null base: placeholder pointers, for sizing only).
ttt_la_args piece_args(const ttt_la_args* a, const PieceLayout& L, int cnt, uint8_t* base) {
  ttt_la_args b = *a;
  b.B = 1;
  b.H = cnt;
  auto at = [&](size_t off, const void* host) -> void* {
    if (!host) return nullptr;
    return base ? static_cast<void*>(base + off) : reinterpret_cast<void*>(static_cast<uintptr_t>(256 + off));
  };
  b.q = at(L.q, a->q);
  b.k = at(L.k, a->k);
  b.v = at(L.v, a->v);
  b.o = at(L.o, a->o);
  b.eta = static_cast<const float*>(at(L.eta, a->eta));
  b.state_in = static_cast<const float*>(at(L.s_in, a->state_in));
  b.state_out = static_cast<float*>(at(L.s_out, a->state_out));
  b.mom_in = static_cast<const float*>(at(L.m_in, a->mom_in));
  b.mom_out = static_cast<float*>(at(L.m_out, a->mom_out));
  b.workspace = L.ws_bytes ? at(L.ws, a->q) : nullptr;
  b.workspace_bytes = L.ws_bytes;
  return b;
}

PieceLayout piece_layout(const ttt_la_args* a) {
  PieceLayout L;
  const int bh = a->B * a->H;
  const size_t es = a->dtype == TTT_LA_BF16 ? 2 : 4;
  // about 24 MB of inputs per piece, 2 to 8 pieces: more, smaller pieces hide
  // more of the copy-out but each costs a launch and a pipeline hand-off
  const size_t st_all = static_cast<size_t>(a->d_v) * a->d_k * sizeof(float) *
                        ((a->state_in ? 1 : 0) + (a->mom_in ? 1 : 0));
  const size_t in_bytes = static_cast<size_t>(bh) *
                          (static_cast<size_t>(a->T) * ((2 * a->d_k + a->d_v) * es + (a->eta ? 4 : 0)) + st_all);
  const int want = static_cast<int>(std::min<size_t>(8, std::max<size_t>(2, in_bytes / (24u << 20))));
  L.pieces = std::min(bh, want);
  L.per = (bh + L.pieces - 1) / L.pieces;
  L.pieces = (bh + L.per - 1) / L.per;
  const size_t tok = static_cast<size_t>(L.per) * a->T;
  const size_t st = static_cast<size_t>(L.per) * a->d_v * a->d_k * sizeof(float);
  size_t off = 0;
  auto take = [&](size_t bytes, bool present) {
    const size_t at = off;
    if (present) off += align256(bytes);
    return at;
  };
  L.q = take(tok * a->d_k * es, true);
  L.k = take(tok * a->d_k * es, true);
  L.v = take(tok * a->d_v * es, true);
  L.o = take(tok * a->d_v * es, true);
  L.eta = take(tok * sizeof(float), a->eta != nullptr);
  L.s_in = take(st, a->state_in != nullptr);
  L.s_out = take(st, a->state_out != nullptr);
  L.m_in = take(st, a->mom_in != nullptr);
  L.m_out = take(st, a->mom_out != nullptr);
  L.ws = off;
  const ttt_la_args probe = piece_args(a, L, L.per, nullptr);
  L.ws_bytes = workspace_for(&probe);
  off += align256(L.ws_bytes);
  L.set_bytes = off;
  return L;
}

}  // namespace
