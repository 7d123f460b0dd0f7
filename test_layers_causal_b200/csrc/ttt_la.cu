// ttt_la.cu -- C ABI of libttt_la: argument checks, kernel selection and
// launches for the causal TTT / linear-attention layer (see include/ttt_la.h).
//
// One translation unit holds every kernel so that the device status word is a
// single symbol.  Host code never computes any part of the layer: it checks
// arguments, builds TMA descriptors and launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/ttt_la.h"
#include "backward.cuh"
#include "backward_chunked.cuh"
#include "backward_mom_tc.cuh"
#include "chunked_simt.cuh"
#include "chunked_tc.cuh"
#include "chunked_tc_mom.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "feature_map.cuh"
#include "recurrent.cuh"
#include "seqshard.cuh"

namespace {

uint64_t g_limit_ns = 1000000000ull;

// NVTX range around each entry point, in the "ttt_la" domain: a profiler
// (nsys, ncu --nvtx) shows which call launched what.  NVTX v3 is header-only;
// with no tool attached each push and pop is a call through a no-op pointer.
nvtxDomainHandle_t nvtx_domain() {
  static const nvtxDomainHandle_t d = nvtxDomainCreateA("ttt_la");
  return d;
}
struct NvtxRange {
  explicit NvtxRange(const char* name) {
    nvtxEventAttributes_t e = {};
    e.version = NVTX_VERSION;
    e.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    e.messageType = NVTX_MESSAGE_TYPE_ASCII;
    e.message.ascii = name;
    nvtxDomainRangePushEx(nvtx_domain(), &e);
  }
  ~NvtxRange() { nvtxDomainRangePop(nvtx_domain()); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// Raises `fn`'s dynamic shared-memory limit to `bytes` on the current device.
// The attribute belongs to each device's context, so the grant is recorded
// per (kernel, device), under a lock: host threads may launch concurrently,
// and one process may drive several devices.
bool grant_smem(const void* fn, int bytes) {
  if (bytes <= 48 * 1024) return true;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  struct Grant {
    const void* fn;
    int dev, bytes;
  };
  static std::mutex mu;
  static std::vector<Grant> granted;
  std::lock_guard<std::mutex> lock(mu);
  for (const Grant& g : granted)
    if (g.fn == fn && g.dev == dev && g.bytes >= bytes) return true;
  // the largest shared-memory carveout, so that the occupancy calculator and
  // the launch both see the whole 228 KB of an SM
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess ||
      cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
          cudaSuccess)
    return false;
  for (Grant& g : granted)
    if (g.fn == fn && g.dev == dev) {
      g.bytes = bytes;
      return true;
    }
  granted.push_back({fn, dev, bytes});
  return true;
}

// Blocks of `fn` (threads, dynamic shared memory) that one SM holds at once on
// the current device, from the occupancy calculator, at most `cap` (tensor
// memory, which the calculator does not count, caps some kernels).  Without a
// device (size queries on a host with no GPU) the answer is `cap`.
int resident_per_sm(const void* fn, int threads, int smem, int cap) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return cap;
  }
  int n = 0;
  if (!grant_smem(fn, smem) || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    return cap;
  }
  return std::min(n, cap);
}

// Launches `kern` on `st`; `coop` makes it a cooperative launch, which
// guarantees that every block of the grid is resident at once (or fails to
// launch), as kernels whose blocks wait for one another need.
template <typename... P, typename... A>
ttt_la_status launch_kernel(void (*kern)(P...), int grid, int threads, int smem, cudaStream_t st, bool coop,
                            A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = coop ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return TTT_LA_ERR_CUDA;
  }
  return TTT_LA_OK;
}

// ------------------------------------------------------------ TMA maps ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [BH][T][d] bf16 tensor, boxes of `cols` elements x `rows` tokens.
bool make_map_box(CUtensorMap* m, const void* base, int BH, int T, int d, int cols, int rows,
                  CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(T) * d * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(cols), static_cast<cuuint32_t>(rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
// Boxes of 64 elements x `rows` tokens, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int BH, int T, int d, int rows) {
  return make_map_box(m, base, BH, T, d, 64, rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

// ------------------------------------------------------ argument checks ----
ttt_la_status check_seq(const ttt_la_args* a) {
  if (!a) return TTT_LA_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->T < 1 || a->d_k < 1 || a->d_v < 1) return TTT_LA_ERR_INVALID_ARG;
  if (a->dtype != TTT_LA_F32 && a->dtype != TTT_LA_BF16) return TTT_LA_ERR_INVALID_ARG;
  if (!a->q || !a->k || !a->v || !a->o) return TTT_LA_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o)) return TTT_LA_ERR_INVALID_ARG;
  if ((a->eta && !aligned16(a->eta)) || (a->state_in && !aligned16(a->state_in)) ||
      (a->state_out && !aligned16(a->state_out)) || (a->mom_in && !aligned16(a->mom_in)) ||
      (a->mom_out && !aligned16(a->mom_out)))
    return TTT_LA_ERR_INVALID_ARG;
  const long long bh = static_cast<long long>(a->B) * a->H;
  if (bh > (1 << 30) || static_cast<long long>(a->T) * std::max(a->d_k, a->d_v) * bh > (1ll << 40))
    return TTT_LA_ERR_INVALID_ARG;
  if (!(a->beta >= 0.f && a->beta < 1.f) && a->beta != 0.f) return TTT_LA_ERR_INVALID_ARG;
  if (a->o == a->q || a->o == a->k || a->o == a->v) return TTT_LA_ERR_INVALID_ARG;
  return TTT_LA_OK;
}

ttt::SeqParams seq_params(const ttt_la_args* a) {
  ttt::SeqParams p;
  p.B = a->B;
  p.H = a->H;
  p.T = a->T;
  p.dk = a->d_k;
  p.dv = a->d_v;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.eta = a->eta;
  p.eta_const = a->eta_const;
  p.beta = a->beta;
  p.sigma = a->ascent ? -1.f : 1.f;
  p.S_in = a->state_in;
  p.S_out = a->state_out;
  p.M_in = a->mom_in;
  p.M_out = a->mom_out;
  p.o = a->o;
  return p;
}

ttt_la_status launched() { return cudaGetLastError() == cudaSuccess ? TTT_LA_OK : TTT_LA_ERR_CUDA; }

// Two more streams per device, one at the device's greatest priority, with a
// fork and two join events, for chains of launches that run beside the call's
// own stream (the momentum backward: dL/dW_0 then deta, its critical path,
// whose blocks the priority puts on the SMs first; dv's reverse launch).
// The caller issues fork -> launches -> join under side_mutex(), so calls from
// several host threads never interleave on the shared events.  Created on
// first use outside stream capture; a call that finds none while its stream
// is capturing runs its launches on its own stream, one after the other.
struct SideStream {
  int dev;
  cudaStream_t s, s2;       // greatest priority; default priority
  cudaEvent_t fork, join, join2;
};
std::mutex& side_mutex() {
  static std::mutex mu;
  return mu;
}
bool side_stream(cudaStream_t st, SideStream* out) {  // side_mutex() held
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static std::vector<SideStream> made;
  for (const SideStream& x : made)
    if (x.dev == dev) {
      // a side stream that another host thread's capture has taken in (it
      // stays captured until that capture ends) is not used
      cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone, cap2 = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(x.s, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone ||
          cudaStreamIsCapturing(x.s2, &cap2) != cudaSuccess || cap2 != cudaStreamCaptureStatusNone) {
        cudaGetLastError();
        return false;
      }
      *out = x;
      return true;
    }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return false;
  }
  SideStream x{dev, nullptr, nullptr, nullptr, nullptr, nullptr};
  int least = 0, greatest = 0;
  if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
      cudaStreamCreateWithPriority(&x.s, cudaStreamNonBlocking, greatest) != cudaSuccess ||
      cudaStreamCreateWithFlags(&x.s2, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&x.join2, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  made.push_back(x);
  *out = x;
  return true;
}

// Zeroes the n words of one call's segment flags and counters.  A kernel
// rather than cudaMemsetAsync: between two kernels of a CUDA graph a memset
// node costs about 3 us more, a small kernel node about 1 us (B200).
__global__ void zero_words_kernel(unsigned* w, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) w[i] = 0u;
}
ttt_la_status zero_words(unsigned* w, size_t n, cudaStream_t st) {
  const int blocks = static_cast<int>(std::min<size_t>((n + 255) / 256, 64));
  zero_words_kernel<<<blocks, 256, 0, st>>>(w, static_cast<int>(n));
  return launched();
}

// ------------------------------------------------------------ recurrent ----
template <int DK, typename T, bool MOM>
ttt_la_status launch_recurrent(const ttt_la_args* a, cudaStream_t st) {
  using Sh = ttt::RecurrentShape<DK>;
  dim3 grid(a->B * a->H, (a->d_v + Sh::ROWS - 1) / Sh::ROWS);
  ttt::recurrent_kernel<DK, T, MOM><<<grid, 128, 0, st>>>(seq_params(a));
  return launched();
}
template <typename T, bool MOM>
ttt_la_status recurrent_dk(const ttt_la_args* a, cudaStream_t st) {
  switch (a->d_k) {
    case 32: return launch_recurrent<32, T, MOM>(a, st);
    case 64: return launch_recurrent<64, T, MOM>(a, st);
    case 128: return launch_recurrent<128, T, MOM>(a, st);
    default: return TTT_LA_ERR_UNSUPPORTED;
  }
}

// --------------------------------------------------------------- chunked ----
struct SegPlan {
  int nchunks, cps, nseg;
  int nwave = 1;      // waves of the cooperative schedule without momentum (1 otherwise)
  int keep = 0;       // phase-A chunks per run whose K and V are loaded evict-last
  int resident = 0;   // blocks of the selected kernel resident at once on the device
  bool coop = false;  // cooperative start states (the head's blocks wait for one another)
};

// Tokens each block handles per wave in the cooperative schedule without
// momentum.  More waves keep K and V in L2 for phase B (two waves live, about
// 150 KB per 512 tokens per block at d = 128), but every wave costs one
// in-place scan of the blocks' d x d totals and a meeting of the head's
// blocks; measured on the long-context layer (B1 H8 T65536 d128) the
// meetings cost more than the re-read saves at every length tried (256 to
// 1024 tokens), so by default the schedule is a single wave (phase A over a
// block's whole run, one scan, phase B).  TTT_LA_WAVE_TOKENS sets the length
// (tuning and tests).
// MB of phase-A K and V loaded evict-last (TTT_LA_L2_KEEP_MB, tuning).
int l2_keep_mb() {
  const char* e = std::getenv("TTT_LA_L2_KEEP_MB");
  const int v = e ? std::atoi(e) : -1;
  return v >= 0 ? v : 64;
}

int wave_tokens() {
  const char* e = std::getenv("TTT_LA_WAVE_TOKENS");
  const int v = e ? std::atoi(e) : 0;
  return v > 0 ? v : (1 << 30);
}

// Tokens per tensor-core tile: the requested chunk, except with momentum, whose
// kernel always runs 64-token tiles (a 128-token chunk is the same layer).
int tc_tile(const ttt_la_args* a) { return a->beta != 0.f ? 64 : a->chunk; }

// Resident blocks per SM of the tensor-core kernel that these arguments
// select (1 for every tile but 64 x 64, whose 256 tensor-memory columns let
// two blocks share an SM).
template <int C, int D>
int tc_per_sm() {
  using Cfg = ttt::TcCfg<C, D>;
  return resident_per_sm(reinterpret_cast<const void*>(ttt::chunked_tc_kernel<C, D>), 256, Cfg::SMEM, Cfg::MINB);
}
template <int D>
int tcm_per_sm() {
  using Cfg = ttt::TcMomCfg<D>;
  return resident_per_sm(reinterpret_cast<const void*>(ttt::chunked_tc_mom_kernel<D>), Cfg::THREADS, Cfg::SMEM, 1);
}
int tc_resident_per_sm(const ttt_la_args* a) {
  if (a->beta != 0.f) return a->d_k == 64 ? tcm_per_sm<64>() : tcm_per_sm<128>();
  if (a->d_k == 64) return a->chunk == 64 ? tc_per_sm<64, 64>() : tc_per_sm<128, 64>();
  return a->chunk == 64 ? tc_per_sm<64, 128>() : tc_per_sm<128, 128>();
}

// Set (on this host thread) while the momentum backward launches its dq pass
// beside other kernels: the start states then come from the decoupled
// look-back, which needs no co-residency of the grid (its blocks wait only
// for blocks that took their tiles earlier), instead of the cooperative prefix.
thread_local bool t_lookback_only = false;

SegPlan plan_segments(const ttt_la_args* a) {
  SegPlan s;
  const int C = tc_tile(a);
  s.nchunks = (a->T + C - 1) / C;
  const int bh = a->B * a->H;
  // Automatic: as many segments as the tile's design places on the SMs at
  // once (two 64 x 64 blocks per SM, one otherwise; never a partial second
  // wave), at least one per sequence.  Whether the grid is really resident as
  // a whole, which the cooperative schedules need, is the occupancy
  // calculator's answer (`resident`).
  s.resident = sm_count() * tc_resident_per_sm(a);
  const int design_per_sm = (a->beta == 0.f && C == 64 && a->d_k == 64) ? 2 : 1;
  int nseg = a->segments > 0 ? a->segments : std::max(1, sm_count() * design_per_sm / bh);
  nseg = std::max(1, std::min(nseg, s.nchunks));
  s.cps = (s.nchunks + nseg - 1) / nseg;
  s.nseg = (s.nchunks + s.cps - 1) / s.cps;
  // Cooperative start states (blocks of a head wait for one another, so the
  // grid must be one wave and is launched cooperatively): with momentum
  // whenever the grid is one wave; without, when a decoupled look-back would
  // also have the last segment read more than 192 KB of totals.
  const bool one_wave = s.nseg > 1 && static_cast<long long>(bh) * s.nseg <= s.resident;
  const size_t lookback_bytes = static_cast<size_t>(s.nseg - 1) * a->d_k * a->d_v * sizeof(float);
  // (the 64 x 64 tile without momentum runs the look-back only: see chunked_tc.cuh)
  const bool tile64 = a->beta == 0.f && C == 64 && a->d_k == 64;
  s.coop = !t_lookback_only && one_wave && (a->beta != 0.f || (lookback_bytes > 192 * 1024 && !tile64));
  if (s.coop && a->beta == 0.f) {
    // every run of every wave holds at least one chunk: nwave <= nchunks / nseg
    const int per_run = std::max(1, wave_tokens() / C);
    s.nwave = std::max(1, std::min(s.nchunks / (s.nseg * per_run), s.nchunks / s.nseg));
  }
  if (a->beta == 0.f && s.nseg > 1 && !tile64) {
    // K and V phase B reads first, kept in L2 from phase A: about l2_keep_mb
    // MB over the whole grid (beside the Q, O and scratch streams).  Measured
    // on the 128-wide tiles only: on 64 x 64 tiles, whose K and V of a whole
    // call already fit in L2 at the LLM shape, the hint was slower.
    const size_t chunk_kv = static_cast<size_t>(C) * (a->d_k + a->d_v) * 2;
    const size_t blocks = static_cast<size_t>(bh) * s.nseg;
    s.keep = static_cast<int>(std::min<size_t>(static_cast<size_t>(l2_keep_mb()) << 20, size_t(1) << 40) /
                              (blocks * chunk_kv));
  }
  return s;
}

bool tc_supported(const ttt_la_args* a) {
  return a->dtype == TTT_LA_BF16 && a->d_k == a->d_v && (a->d_k == 64 || a->d_k == 128) &&
         (a->chunk == 64 || a->chunk == 128);
}

bool simt_supported(const ttt_la_args* a, ttt::SimtShape* sh) {
  if (a->dtype != TTT_LA_F32) return false;
  if (!(a->chunk == 16 || a->chunk == 32 || a->chunk == 64)) return false;
  if (a->d_k > 128 || a->d_v > 128) return false;
  const bool mom = a->beta != 0.f;
  if (mom && (a->d_k > 64 || a->d_v > 64)) return false;
  sh->C = a->chunk;
  sh->dk = a->d_k;
  sh->dv = a->d_v;
  sh->mom = mom;
  return sh->bytes() <= 227 * 1024;
}

// Scratch layout of the chunked tensor-core path: fp32 [BH][nseg][2][d_v][d_k]
// (segment totals, segment start states), then nseg*BH publication flags, one
// tile counter and BH per-head counters (uint32), which every call clears
// before its launch.
// The wave schedule uses fp32 [BH][2][nseg][d_v][d_k] (run totals, scanned in
// place into start states, slot = wave parity) plus [BH][d_v][d_k] (state at
// the wave's end): (2 nseg + 1) matrices per head instead of 2 nseg.
size_t tc_ws_floats(int bh, int nseg, int D, bool waves = false) {
  return static_cast<size_t>(bh) * (2 * nseg + (waves ? 1 : 0)) * D * D;
}
size_t tc_flag_words(int bh, int nseg) { return static_cast<size_t>(bh) * nseg + 1 + bh; }
size_t tc_ws_bytes(int bh, int nseg, int D, bool waves = false) {
  const size_t b = tc_ws_floats(bh, nseg, D, waves) * sizeof(float) + tc_flag_words(bh, nseg) * sizeof(unsigned);
  return (b + 15) & ~static_cast<size_t>(15);
}

// BWD: one of the backward's reverse-time passes (see chunked_tc.cuh), with
// vdot/deta for the per-token learning-rate gradient.
template <int C, int D, bool BWD = false>
ttt_la_status launch_tc(const ttt_la_args* a, const SegPlan& sp, cudaStream_t st, const void* vdot = nullptr,
                        float* deta = nullptr) {
  using Cfg = ttt::TcCfg<C, D, BWD>;
  if (!grant_smem(reinterpret_cast<const void*>(ttt::chunked_tc_kernel<C, D, BWD>), Cfg::SMEM))
    return TTT_LA_ERR_CUDA;
  const int bh = a->B * a->H;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, a->q, bh, a->T, D, C) || !make_map(&mk, a->k, bh, a->T, D, C) ||
      !make_map(&mv, a->v, bh, a->T, D, C) || !make_map(&mo, a->o, bh, a->T, D, C))
    return TTT_LA_ERR_CUDA;
  ttt::TcParams p;
  p.BH = bh;
  p.T = a->T;
  p.nchunks = sp.nchunks;
  p.cps = sp.cps;
  p.nseg = sp.nseg;
  p.eta = a->eta;
  p.eta_const = a->eta_const;
  p.sigma = a->ascent ? -1.f : 1.f;
  p.S_in = a->state_in;
  p.ws = nullptr;
  p.flags = nullptr;
  p.coop = sp.coop ? 1 : 0;
  p.nwave = sp.coop ? sp.nwave : 1;
  p.keep = sp.keep;
  p.S_out = a->state_out;
  p.vdot = vdot;
  p.deta = deta;
  p.limit_ns = g_limit_ns;
  if (sp.nseg > 1) {
    p.ws = static_cast<float*>(a->workspace);
    p.flags = reinterpret_cast<unsigned*>(p.ws + tc_ws_floats(bh, sp.nseg, D, sp.coop));
    const ttt_la_status s = zero_words(p.flags, tc_flag_words(bh, sp.nseg), st);
    if (s != TTT_LA_OK) return s;
  }
  return launch_kernel(ttt::chunked_tc_kernel<C, D, BWD>, bh * sp.nseg, 256, Cfg::SMEM, st, sp.coop, mq, mk, mv, mo,
                       p);
}

// One of the backward's two reverse-time passes (bf16, no momentum): the
// chunked forward over the chunks last to first with the anti-causal mask,
// K unscaled, the state read out as bf16(W) + bf16(W - bf16(W)), and the
// epilogue writing o_t := sigma eta_t O_t in bf16 (dv or dk; a->eta,
// a->eta_const and a->ascent are the layer's) plus, when deta is given,
// deta_t = sigma vdot_t . O_t from O in fp32.  Tiles of 64 tokens: 64 x 64
// (not merged: the second bf16 copy of W needs its own buffer; two blocks per
// SM) at d = 64, 64 x 128 at d = 128.
size_t workspace_for(const ttt_la_args* a);
ttt_la_status backward_pass_tc(const ttt_la_args* a, const void* vdot, float* deta, cudaStream_t st) {
  if (!a || (deta && (!vdot || !aligned16(vdot)))) return TTT_LA_ERR_INVALID_ARG;
  const ttt_la_status s = check_seq(a);
  if (s != TTT_LA_OK) return s;
  if (a->dtype != TTT_LA_BF16 || a->beta != 0.f || a->d_k != a->d_v ||
      !((a->d_k == 64 && a->chunk == 64) || (a->d_k == 128 && a->chunk == 64)))
    return TTT_LA_ERR_UNSUPPORTED;
  const SegPlan sp = plan_segments(a);
  if (sp.nseg > 1) {
    const size_t need = workspace_for(a);
    if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace)) return TTT_LA_ERR_INVALID_ARG;
  }
  return a->d_k == 64 ? launch_tc<64, 64, true>(a, sp, st, vdot, deta)
                      : launch_tc<64, 128, true>(a, sp, st, vdot, deta);
}

template <bool MOM>
ttt_la_status launch_simt(const ttt_la_args* a, const ttt::SimtShape& sh, cudaStream_t st) {
  const size_t bytes = sh.bytes();
  if (!grant_smem(reinterpret_cast<const void*>(ttt::chunked_simt_f32_kernel<MOM>), static_cast<int>(bytes)))
    return TTT_LA_ERR_CUDA;
  ttt::chunked_simt_f32_kernel<MOM><<<a->B * a->H, 256, bytes, st>>>(seq_params(a), sh);
  return launched();
}

// Momentum scratch: fp32 [BH][nseg][4][d_v][d_k] (dW, dM, W_incl, M_incl),
// fp32 [BH][nseg][2] (G, B), then flags and the tile counter.
size_t tcm_ws_floats(int bh, int nseg, int D) { return static_cast<size_t>(bh) * nseg * (4 * D * D + 2); }
size_t tcm_ws_bytes(int bh, int nseg, int D) {
  const size_t b = tcm_ws_floats(bh, nseg, D) * sizeof(float) + tc_flag_words(bh, nseg) * sizeof(unsigned);
  return (b + 15) & ~static_cast<size_t>(15);
}

// Chunkwise momentum backward (backward_mom_tc.cuh): one block per (b, h)
// and 64 rows of the state.
// Reverse kernel: rows of `kr` (the K role) get the output rows `out`; qr,
// dr are the Q and dO roles; G_in/X_in the chunk-end states of the sequence
// (nullptr: zero); G_out/X_out its chunk-start states (nullptr: not written).
template <int D>
ttt_la_status launch_mom_rev(int BH, int T, const void* kr, const void* qr, const void* dr, void* out,
                             const float* eta, float eta_const, float sigma, float beta, const float* G_in,
                             const float* X_in, float* G_out, float* X_out, cudaStream_t st) {
  using Cfg = ttt::MomRevCfg<D>;
  if (!grant_smem(reinterpret_cast<const void*>(ttt::mom_bwd_rev_kernel<D>), Cfg::SMEM)) return TTT_LA_ERR_CUDA;
  CUtensorMap mk, mq, md, mo;
  if (!make_map(&mk, kr, BH, T, D, Cfg::C) || !make_map(&mq, qr, BH, T, D, Cfg::C) ||
      !make_map(&md, dr, BH, T, D, Cfg::C) || !make_map(&mo, out, BH, T, D, Cfg::C))
    return TTT_LA_ERR_CUDA;
  ttt::MomBwdParams p;
  std::memset(&p, 0, sizeof p);
  p.BH = BH;
  p.T = T;
  p.nchunks = (T + Cfg::C - 1) / Cfg::C;
  p.eta = eta;
  p.eta_const = eta_const;
  p.sigma = sigma;
  p.beta = beta;
  p.G_in = G_in;
  p.X_in = X_in;
  p.G_out = G_out;
  p.X_out = X_out;
  p.limit_ns = g_limit_ns;
  return launch_kernel(ttt::mom_bwd_rev_kernel<D>, BH * (D / Cfg::RS), Cfg::THREADS, Cfg::SMEM, st, false, mk, mq, md,
                       mo, p);
}

// deta kernel: G_in = dL/dW_0 (required), X_in = M_0 (nullptr: zero).
template <int D>
ttt_la_status launch_mom_deta(int BH, int T, const void* q, const void* k, const void* v, const void* dO,
                              float sigma, float beta, const float* G_in, const float* X_in, float* deta,
                              cudaStream_t st) {
  using Cfg = ttt::MomDetaCfg<D>;
  if (!grant_smem(reinterpret_cast<const void*>(ttt::mom_bwd_deta_kernel<D>), Cfg::SMEM)) return TTT_LA_ERR_CUDA;
  CUtensorMap mq, mk, mv, md;
  if (!make_map(&mq, q, BH, T, D, Cfg::C) || !make_map(&mk, k, BH, T, D, Cfg::C) ||
      !make_map(&mv, v, BH, T, D, Cfg::C) || !make_map(&md, dO, BH, T, D, Cfg::C))
    return TTT_LA_ERR_CUDA;
  ttt::MomBwdParams p;
  std::memset(&p, 0, sizeof p);
  p.BH = BH;
  p.T = T;
  p.nchunks = (T + Cfg::C - 1) / Cfg::C;
  p.sigma = sigma;
  p.beta = beta;
  p.G_in = G_in;
  p.X_in = X_in;
  p.deta = deta;
  p.limit_ns = g_limit_ns;
  // the blocks of a head add their rows' parts onto deta, which the caller
  // has zeroed (the state transposes at the start of the call do it)
  return launch_kernel(ttt::mom_bwd_deta_kernel<D>, BH * (D / Cfg::RS), Cfg::THREADS, Cfg::SMEM, st, false, mq, mk, mv,
                       md, p);
}

// dL/dW_0 = G_T + sum_t do_t q_t^T into g0 (fp32 [BH][d][d]; G_T may be
// nullptr): the tensor-core partials over `nsplit` token ranges into `part`,
// then their sum in a fixed order.
template <int D>
ttt_la_status launch_mom_g0(int BH, int T, int nsplit, const void* dO, const void* q, const float* G_T, float* part,
                            float* g0, cudaStream_t st) {
  using Cfg = ttt::MomG0Cfg<D>;
  if (!grant_smem(reinterpret_cast<const void*>(ttt::mom_g0_kernel<D>), Cfg::SMEM)) return TTT_LA_ERR_CUDA;
  CUtensorMap md, mq;
  if (!make_map(&md, dO, BH, T, D, Cfg::C) || !make_map(&mq, q, BH, T, D, Cfg::C)) return TTT_LA_ERR_CUDA;
  ttt::MomG0Params p;
  std::memset(&p, 0, sizeof p);
  p.BH = BH;
  p.T = T;
  p.nsplit = nsplit;
  const int tiles = (T + Cfg::C - 1) / Cfg::C;
  p.tiles_per_split = (tiles + nsplit - 1) / nsplit;
  p.part = part;
  p.limit_ns = g_limit_ns;
  ttt_la_status s = launch_kernel(ttt::mom_g0_kernel<D>, BH * nsplit, Cfg::THREADS, Cfg::SMEM, st, false, md, mq, p);
  if (s != TTT_LA_OK) return s;
  const long long n = static_cast<long long>(BH) * D * D;
  const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, static_cast<long long>(sm_count()) * 4));
  ttt::mom_g0_sum_kernel<<<blocks, 256, 0, st>>>(G_T, part, nsplit, n, g0);
  return launched();
}

size_t workspace_for(const ttt_la_args* a) {
  if (!tc_supported(a)) return 0;
  const SegPlan sp = plan_segments(a);
  if (sp.nseg <= 1) return 0;
  return a->beta != 0.f ? tcm_ws_bytes(a->B * a->H, sp.nseg, a->d_k)
                        : tc_ws_bytes(a->B * a->H, sp.nseg, a->d_k, sp.coop);
}

template <int D>
ttt_la_status launch_tc_mom(const ttt_la_args* a, const SegPlan& sp, cudaStream_t st) {
  using Cfg = ttt::TcMomCfg<D>;
  constexpr int C = Cfg::C;
  if (!grant_smem(reinterpret_cast<const void*>(ttt::chunked_tc_mom_kernel<D>), Cfg::SMEM)) return TTT_LA_ERR_CUDA;
  const int bh = a->B * a->H;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, a->q, bh, a->T, D, C) || !make_map(&mk, a->k, bh, a->T, D, C) ||
      !make_map(&mv, a->v, bh, a->T, D, C) || !make_map(&mo, a->o, bh, a->T, D, C))
    return TTT_LA_ERR_CUDA;
  ttt::TcMomParams p;
  p.BH = bh;
  p.T = a->T;
  p.nchunks = sp.nchunks;
  p.cps = sp.cps;
  p.nseg = sp.nseg;
  p.eta = a->eta;
  p.eta_const = a->eta_const;
  p.sigma = a->ascent ? -1.f : 1.f;
  p.beta = a->beta;
  p.S_in = a->state_in;
  p.M_in = a->mom_in;
  p.ws = nullptr;
  p.wsc = nullptr;
  p.flags = nullptr;
  p.S_out = a->state_out;
  p.M_out = a->mom_out;
  p.limit_ns = g_limit_ns;
  p.coop = sp.coop ? 1 : 0;
  if (sp.nseg > 1) {
    p.ws = static_cast<float*>(a->workspace);
    p.wsc = p.ws + static_cast<size_t>(bh) * sp.nseg * 4 * D * D;
    p.flags = reinterpret_cast<unsigned*>(p.ws + tcm_ws_floats(bh, sp.nseg, D));
    const ttt_la_status s = zero_words(p.flags, tc_flag_words(bh, sp.nseg), st);
    if (s != TTT_LA_OK) return s;
  }
  return launch_kernel(ttt::chunked_tc_mom_kernel<D>, bh * sp.nseg, Cfg::THREADS, Cfg::SMEM, st, sp.coop, mq, mk, mv,
                       mo, p);
}

// ---------------------------------------------------------------- decode ----
template <int DK, typename T, bool MOM>
ttt_la_status launch_decode(const ttt_la_decode_args* a, cudaStream_t st) {
  constexpr int U = 4;
  constexpr int RPW = 32 / (DK / 4);
  ttt::DecodeParams p;
  p.N = a->N;
  p.H = a->H;
  p.dk = a->d_k;
  p.dv = a->d_v;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.eta = a->eta;
  p.eta_const = a->eta_const;
  p.beta = a->beta;
  p.sigma = a->ascent ? -1.f : 1.f;
  p.S = a->state;
  p.M = a->mom;
  p.o = a->o;
  const long long rows = static_cast<long long>(a->N) * a->H * a->d_v;
  const long long warps = (rows + RPW * U - 1) / (RPW * U);
  const long long blocks_needed = (warps + 7) / 8;
  const int blocks = static_cast<int>(std::min<long long>(blocks_needed, static_cast<long long>(sm_count()) * 8));
  ttt::decode_step_kernel<DK, T, MOM, U><<<blocks, 256, 0, st>>>(p);
  return launched();
}
template <typename T, bool MOM>
ttt_la_status decode_dk(const ttt_la_decode_args* a, cudaStream_t st) {
  switch (a->d_k) {
    case 32: return launch_decode<32, T, MOM>(a, st);
    case 64: return launch_decode<64, T, MOM>(a, st);
    case 128: return launch_decode<128, T, MOM>(a, st);
    default: return TTT_LA_ERR_UNSUPPORTED;
  }
}

// ----------------------------------------------------------- feature map ----
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

ttt_la_status check_feature(const ttt_la_feature_args* a) {
  if (!a) return TTT_LA_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->T < 1 || a->d_in < 1 || a->d_out < 1) return TTT_LA_ERR_INVALID_ARG;
  if (a->n_inputs != 1 && a->n_inputs != 2) return TTT_LA_ERR_INVALID_ARG;
  if (!a->w1 || !a->w3 || !aligned16(a->w1) || !aligned16(a->w3)) return TTT_LA_ERR_INVALID_ARG;
  const long long bh = static_cast<long long>(a->B) * a->H;
  const long long ntile = (a->T + 127) / 128;
  if (bh > (1 << 30) || static_cast<long long>(a->T) * std::max(a->d_in, a->d_out) * bh > (1ll << 40) ||
      bh * ntile * a->n_inputs >= (1ll << 31))
    return TTT_LA_ERR_INVALID_ARG;
  const size_t xb = static_cast<size_t>(bh) * a->T * a->d_in * 2, yb = static_cast<size_t>(bh) * a->T * a->d_out * 2;
  const size_t wb = static_cast<size_t>(a->H) * a->d_out * a->d_in * 2;
  for (int i = 0; i < a->n_inputs; ++i) {
    if (!a->x[i] || !a->y[i] || !aligned16(a->x[i]) || !aligned16(a->y[i])) return TTT_LA_ERR_INVALID_ARG;
    if (overlaps(a->y[i], yb, a->w1, wb) || overlaps(a->y[i], yb, a->w3, wb)) return TTT_LA_ERR_INVALID_ARG;
    for (int j = 0; j < a->n_inputs; ++j)
      if (overlaps(a->y[i], yb, a->x[j], xb) || (j != i && overlaps(a->y[i], yb, a->y[j], yb)))
        return TTT_LA_ERR_INVALID_ARG;
  }
  if ((a->d_in != 64 && a->d_in != 128) || (a->d_out != 64 && a->d_out != 128)) return TTT_LA_ERR_UNSUPPORTED;
  return TTT_LA_OK;
}

template <int DIN, int DOUT>
ttt_la_status launch_feature(const ttt_la_feature_args* a, cudaStream_t st) {
  using Cfg = ttt::FmapCfg<DIN, DOUT>;
  if (!grant_smem(reinterpret_cast<const void*>(ttt::feature_map_kernel<DIN, DOUT>), Cfg::SMEM))
    return TTT_LA_ERR_CUDA;
  const int bh = a->B * a->H;
  CUtensorMap mx[2], my[2], m1, m3;
  for (int i = 0; i < 2; ++i) {
    const int j = i < a->n_inputs ? i : 0;  // a single input fills both slots
    if (!make_map(&mx[i], a->x[j], bh, a->T, DIN, Cfg::ROWS) || !make_map(&my[i], a->y[j], bh, a->T, DOUT, Cfg::ROWS))
      return TTT_LA_ERR_CUDA;
  }
  if (!make_map(&m1, a->w1, a->H, DOUT, DIN, DOUT) || !make_map(&m3, a->w3, a->H, DOUT, DIN, DOUT))
    return TTT_LA_ERR_CUDA;
  ttt::FmapParams p;
  p.H = a->H;
  p.B = a->B;
  p.T = a->T;
  p.ntile = (a->T + Cfg::ROWS - 1) / Cfg::ROWS;
  p.ninputs = a->n_inputs;
  p.total = a->H * a->n_inputs * a->B * p.ntile;
  p.limit_ns = g_limit_ns;
  const int grid = std::min(p.total, sm_count());
  ttt::feature_map_kernel<DIN, DOUT><<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(mx[0], mx[1], my[0], my[1], m1, m3, p);
  return launched();
}

// -------------------------------------------------------------- backward ----
int bwd_max_dv(int dk) { return dk == 32 ? 512 : dk == 64 ? 256 : 128; }  // 32 warps x rows per warp
int bwd_nck(int T) { return (T + ttt::BwdShape<32>::CK - 1) / ttt::BwdShape<32>::CK; }
size_t bwd_ws_bytes(const ttt_la_grad_args* a) {
  const size_t ns = a->beta != 0.f ? 2 : 1;
  const size_t per = (static_cast<size_t>(bwd_nck(a->T)) + ttt::BwdShape<32>::CK) * ns * a->d_v * a->d_k;
  return static_cast<size_t>(a->B) * a->H * per * sizeof(float);
}

// Checks shared by both backward forms: sizes, pointers, alignment, overlaps.
ttt_la_status check_grad_common(const ttt_la_grad_args* a) {
  if (!a) return TTT_LA_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->T < 1 || a->d_k < 1 || a->d_v < 1) return TTT_LA_ERR_INVALID_ARG;
  if (a->dtype != TTT_LA_F32 && a->dtype != TTT_LA_BF16) return TTT_LA_ERR_INVALID_ARG;
  if (!(a->beta >= 0.f && a->beta < 1.f)) return TTT_LA_ERR_INVALID_ARG;
  const void* need[] = {a->q, a->k, a->v, a->grad_o, a->grad_q, a->grad_k, a->grad_v};
  for (const void* x : need)
    if (!x || !aligned16(x)) return TTT_LA_ERR_INVALID_ARG;
  const void* opt[] = {a->eta, a->state_in, a->mom_in, a->grad_state, a->grad_mom, a->grad_eta,
                       a->grad_state_in, a->grad_mom_in, a->workspace};
  for (const void* x : opt)
    if (x && !aligned16(x)) return TTT_LA_ERR_INVALID_ARG;
  const long long bh = static_cast<long long>(a->B) * a->H;
  if (bh > (1 << 30) || static_cast<long long>(a->T) * std::max(a->d_k, a->d_v) * bh > (1ll << 40))
    return TTT_LA_ERR_INVALID_ARG;
  const size_t el = a->dtype == TTT_LA_F32 ? 4 : 2;
  const size_t nk = static_cast<size_t>(bh) * a->T * a->d_k * el, nv = static_cast<size_t>(bh) * a->T * a->d_v * el;
  const size_t ns = static_cast<size_t>(bh) * a->d_v * a->d_k * 4, ne = static_cast<size_t>(bh) * a->T * 4;
  const void* outs[] = {a->grad_q, a->grad_k, a->grad_v, a->grad_eta, a->grad_state_in, a->grad_mom_in};
  const size_t osz[] = {nk, nk, nv, ne, ns, ns};
  const void* ins[] = {a->q, a->k, a->v, a->grad_o, a->eta, a->state_in, a->mom_in, a->grad_state, a->grad_mom};
  const size_t isz[] = {nk, nk, nv, nv, ne, ns, ns, ns, ns};
  for (int i = 0; i < 6; ++i) {
    if (!outs[i]) continue;
    for (int j = 0; j < 9; ++j)
      if (ins[j] && overlaps(outs[i], osz[i], ins[j], isz[j])) return TTT_LA_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (outs[j] && overlaps(outs[i], osz[i], outs[j], osz[j])) return TTT_LA_ERR_INVALID_ARG;
  }
  return TTT_LA_OK;
}

ttt_la_status check_grad(const ttt_la_grad_args* a) {
  const ttt_la_status s = check_grad_common(a);
  if (s != TTT_LA_OK) return s;
  if (a->d_k != 32 && a->d_k != 64 && a->d_k != 128) return TTT_LA_ERR_UNSUPPORTED;
  if (a->d_v > bwd_max_dv(a->d_k)) return TTT_LA_ERR_UNSUPPORTED;
  if (!a->workspace || a->workspace_bytes < bwd_ws_bytes(a)) return TTT_LA_ERR_INVALID_ARG;
  return TTT_LA_OK;
}

template <int DK, typename T, bool MOM>
ttt_la_status launch_backward(const ttt_la_grad_args* a, cudaStream_t st) {
  using Sh = ttt::BwdShape<DK>;
  const size_t smem = ttt::bwd_smem_floats(DK, a->d_v, Sh::CK) * sizeof(float);
  if (!grant_smem(reinterpret_cast<const void*>(ttt::backward_recurrent_kernel<DK, T, MOM>), 232448))
    return TTT_LA_ERR_CUDA;
  ttt::BwdParams p;
  p.BH = a->B * a->H;
  p.T = a->T;
  p.dk = a->d_k;
  p.dv = a->d_v;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.eta = a->eta;
  p.eta_const = a->eta_const;
  p.beta = a->beta;
  p.sigma = a->ascent ? -1.f : 1.f;
  p.S_in = a->state_in;
  p.M_in = a->mom_in;
  p.dO = a->grad_o;
  p.dS = a->grad_state;
  p.dM = a->grad_mom;
  p.dq = a->grad_q;
  p.dk_out = a->grad_k;
  p.dv_out = a->grad_v;
  p.deta = a->grad_eta;
  p.dS_in = a->grad_state_in;
  p.dM_in = a->grad_mom_in;
  p.nck = bwd_nck(a->T);
  const size_t ns = MOM ? 2 : 1;
  p.ckpt = static_cast<float*>(a->workspace);
  p.hist = p.ckpt + static_cast<size_t>(p.BH) * p.nck * ns * a->d_v * a->d_k;
  const int warps = (a->d_v + Sh::ROWS_PER_WARP - 1) / Sh::ROWS_PER_WARP;
  ttt::backward_recurrent_kernel<DK, T, MOM><<<p.BH, 32 * warps, smem, st>>>(p);
  return launched();
}
template <typename T, bool MOM>
ttt_la_status backward_dk(const ttt_la_grad_args* a, cudaStream_t st) {
  switch (a->d_k) {
    case 32: return launch_backward<32, T, MOM>(a, st);
    case 64: return launch_backward<64, T, MOM>(a, st);
    default: return launch_backward<128, T, MOM>(a, st);
  }
}

// Scratch of ttt_la_forward_chunked_noalloc: one fixed array per device,
// shared by every call on that device (see include/ttt_la.h).
static __device__ __align__(256) unsigned char g_noalloc_scratch[TTT_LA_STATIC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code the
// symbol names a host-side stand-in, never the device array, so the address is
// looked up with cudaGetSymbolAddress once per device (that device current)
// and cached.  Returns nullptr when the lookup fails.
void* noalloc_scratch_ptr() {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* ptrs[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ttt::mbar_init(&bar, 1);
    ttt::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) ttt::mbar_wait(&bar, 0, limit_ns);  // nothing ever arrives
  __syncthreads();
}

}  // namespace

#include "host_pipeline.h"

extern "C" {

const char* ttt_la_status_string(ttt_la_status s) {
  switch (s) {
    case TTT_LA_OK: return "ok";
    case TTT_LA_ERR_INVALID_ARG: return "invalid argument";
    case TTT_LA_ERR_UNSUPPORTED: return "unsupported configuration";
    case TTT_LA_ERR_CUDA: return "CUDA error";
    case TTT_LA_ERR_TIMEOUT: return "in-kernel wait timed out";
    case TTT_LA_ERR_SCRATCH_LIMIT: return "scratch need exceeds the fixed no-alloc array";
    case TTT_LA_ERR_DEVICE_CHECK: return "device-side bounds check failed (debug build)";
  }
  return "unknown status";
}

const char* ttt_la_version(void) { return ttt::kDebugChecks ? "ttt_la 0.2 (sm_100a, debug checks)" : "ttt_la 0.2 (sm_100a)"; }

ttt_la_status ttt_la_set_wait_limit_ns(int64_t limit_ns) {
  if (limit_ns < 1000) return TTT_LA_ERR_INVALID_ARG;
  g_limit_ns = static_cast<uint64_t>(limit_ns);
  return TTT_LA_OK;
}

size_t ttt_la_workspace_size(const ttt_la_args* a) {
  if (check_seq(a) != TTT_LA_OK) return 0;
  return workspace_for(a);
}

ttt_la_status ttt_la_forward_chunked(const ttt_la_args* a, void* stream) {
  NvtxRange range("ttt_la_forward_chunked");
  ttt_la_status s = check_seq(a);
  if (s != TTT_LA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool mom = a->beta != 0.f;
  ttt::SimtShape sh;
  if (a->dtype == TTT_LA_F32) {
    if (!simt_supported(a, &sh)) return TTT_LA_ERR_UNSUPPORTED;
    return mom ? launch_simt<true>(a, sh, st) : launch_simt<false>(a, sh, st);
  }
  if (!tc_supported(a)) return TTT_LA_ERR_UNSUPPORTED;
  if (a->eta == nullptr && !(a->eta_const == a->eta_const)) return TTT_LA_ERR_INVALID_ARG;
  const SegPlan sp = plan_segments(a);
  if (sp.nseg > 1) {
    const size_t need = workspace_for(a);
    if (!a->workspace || a->workspace_bytes < need || !aligned16(a->workspace)) return TTT_LA_ERR_INVALID_ARG;
  }
  if (mom) return a->d_k == 64 ? launch_tc_mom<64>(a, sp, st) : launch_tc_mom<128>(a, sp, st);
  if (a->d_k == 64) return a->chunk == 64 ? launch_tc<64, 64>(a, sp, st) : launch_tc<128, 64>(a, sp, st);
  return a->chunk == 64 ? launch_tc<64, 128>(a, sp, st) : launch_tc<128, 128>(a, sp, st);
}

ttt_la_status ttt_la_chunked_plan(const ttt_la_args* a, ttt_la_plan* out) {
  if (!out) return TTT_LA_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof *out);
  const ttt_la_status s = check_seq(a);
  if (s != TTT_LA_OK) return s;
  if (a->dtype == TTT_LA_F32) {
    ttt::SimtShape sh;
    if (!simt_supported(a, &sh)) return TTT_LA_ERR_UNSUPPORTED;
    out->path = 2;
    out->tile = a->chunk;
    out->segments = 1;
    out->chunks_per_segment = (a->T + a->chunk - 1) / a->chunk;
    out->blocks = a->B * a->H;
    out->resident = out->blocks;
    return TTT_LA_OK;
  }
  if (!tc_supported(a)) return TTT_LA_ERR_UNSUPPORTED;
  const SegPlan sp = plan_segments(a);
  out->path = a->beta != 0.f ? 1 : 0;
  out->tile = tc_tile(a);
  out->segments = sp.nseg;
  out->chunks_per_segment = sp.cps;
  out->cooperative = sp.coop ? 1 : 0;
  out->waves = sp.nwave;
  out->blocks = a->B * a->H * sp.nseg;
  out->resident = sp.resident;
  out->workspace_bytes = workspace_for(a);
  return TTT_LA_OK;
}

ttt_la_status ttt_la_forward_chunked_noalloc(const ttt_la_args* a, void* stream) {
  NvtxRange range("ttt_la_forward_chunked_noalloc");
  ttt_la_status s = check_seq(a);
  if (s != TTT_LA_OK) return s;
  const size_t need = workspace_for(a);
  if (need > TTT_LA_STATIC_SCRATCH_BYTES) return TTT_LA_ERR_SCRATCH_LIMIT;
  ttt_la_args b = *a;
  b.workspace = nullptr;
  b.workspace_bytes = 0;
  if (need > 0) {
    void* p = noalloc_scratch_ptr();
    if (!p) return TTT_LA_ERR_CUDA;
    b.workspace = p;
    b.workspace_bytes = TTT_LA_STATIC_SCRATCH_BYTES;
  }
  return ttt_la_forward_chunked(&b, stream);
}

size_t ttt_la_host_staging_size(const ttt_la_args* a) {
  if (check_seq(a) != TTT_LA_OK) return 0;
  return 2 * piece_layout(a).set_bytes;
}

ttt_la_status ttt_la_forward_chunked_host(const ttt_la_args* a, void* device_buf, size_t device_bytes,
                                          void* stream) {
  NvtxRange range("ttt_la_forward_chunked_host");
  ttt_la_status s = check_seq(a);
  if (s != TTT_LA_OK) return s;
  if (a->dtype == TTT_LA_F32) {
    ttt::SimtShape sh;
    if (!simt_supported(a, &sh)) return TTT_LA_ERR_UNSUPPORTED;
  } else if (!tc_supported(a)) {
    return TTT_LA_ERR_UNSUPPORTED;
  }
  const PieceLayout L = piece_layout(a);
  if (!device_buf || !aligned16(device_buf) || device_bytes < 2 * L.set_bytes) return TTT_LA_ERR_INVALID_ARG;
  HostPipe* hp = host_pipe();
  if (!hp) return TTT_LA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(hp->mu);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t es = a->dtype == TTT_LA_BF16 ? 2 : 4;
  const int bh = a->B * a->H;
  const size_t qrow = static_cast<size_t>(a->T) * a->d_k * es, vrow = static_cast<size_t>(a->T) * a->d_v * es;
  const size_t erow = static_cast<size_t>(a->T) * sizeof(float);
  const size_t srow = static_cast<size_t>(a->d_v) * a->d_k * sizeof(float);
  auto h2d = [&](size_t dst, const void* src, size_t row, int first, int cnt, uint8_t* base) {
    if (!src) return true;
    return cudaMemcpyAsync(base + dst, static_cast<const uint8_t*>(src) + row * first, row * cnt,
                           cudaMemcpyHostToDevice, hp->s_in) == cudaSuccess;
  };
  auto d2h = [&](void* dst, size_t src, size_t row, int first, int cnt, uint8_t* base) {
    if (!dst) return true;
    return cudaMemcpyAsync(static_cast<uint8_t*>(dst) + row * first, base + src, row * cnt, cudaMemcpyDeviceToHost,
                           hp->s_out) == cudaSuccess;
  };
  // fork: copies out start after the caller's earlier work.  Copies in need
  // only their staging set to be free (the last forward that read it, of
  // this call or an earlier one), so a call's first copies overlap the end
  // of the previous call.
  if (cudaEventRecord(hp->fork, st) != cudaSuccess || cudaStreamWaitEvent(hp->s_out, hp->fork, 0) != cudaSuccess)
    return TTT_LA_ERR_CUDA;
  for (int j = 0; j < L.pieces; ++j) {
    const int b = j & 1, first = j * L.per, cnt = std::min(L.per, bh - first);
    uint8_t* base = static_cast<uint8_t*>(device_buf) + b * L.set_bytes;
    // copy in, once the last forward that read this set has finished
    if (cudaStreamWaitEvent(hp->s_in, hp->done[b], 0) != cudaSuccess) return TTT_LA_ERR_CUDA;
    if (!h2d(L.q, a->q, qrow, first, cnt, base) || !h2d(L.k, a->k, qrow, first, cnt, base) ||
        !h2d(L.v, a->v, vrow, first, cnt, base) || !h2d(L.eta, a->eta, erow, first, cnt, base) ||
        !h2d(L.s_in, a->state_in, srow, first, cnt, base) || !h2d(L.m_in, a->mom_in, srow, first, cnt, base) ||
        cudaEventRecord(hp->in_ready[b], hp->s_in) != cudaSuccess)
      return TTT_LA_ERR_CUDA;
    // forward on the caller's stream, once the inputs are in and piece j-2's
    // outputs have left this set
    if (cudaStreamWaitEvent(st, hp->in_ready[b], 0) != cudaSuccess) return TTT_LA_ERR_CUDA;
    if (cudaStreamWaitEvent(st, hp->out_done[b], 0) != cudaSuccess) return TTT_LA_ERR_CUDA;
    const ttt_la_args pa = piece_args(a, L, cnt, base);
    s = ttt_la_forward_chunked(&pa, st);
    if (s != TTT_LA_OK) return s;
    if (cudaEventRecord(hp->done[b], st) != cudaSuccess) return TTT_LA_ERR_CUDA;
    // copy out
    if (cudaStreamWaitEvent(hp->s_out, hp->done[b], 0) != cudaSuccess) return TTT_LA_ERR_CUDA;
    if (!d2h(a->o, L.o, vrow, first, cnt, base) || !d2h(a->state_out, L.s_out, srow, first, cnt, base) ||
        !d2h(a->mom_out, L.m_out, srow, first, cnt, base) ||
        cudaEventRecord(hp->out_done[b], hp->s_out) != cudaSuccess)
      return TTT_LA_ERR_CUDA;
  }
  // join: the caller's stream continues once every copy has completed
  if (cudaEventRecord(hp->join_in, hp->s_in) != cudaSuccess ||
      cudaEventRecord(hp->join_out, hp->s_out) != cudaSuccess ||
      cudaStreamWaitEvent(st, hp->join_in, 0) != cudaSuccess || cudaStreamWaitEvent(st, hp->join_out, 0) != cudaSuccess)
    return TTT_LA_ERR_CUDA;
  return TTT_LA_OK;
}

ttt_la_status ttt_la_segment_map(const ttt_la_args* a, float* dW, float* dM, float* GB, void* stream) {
  NvtxRange range("ttt_la_segment_map");
  ttt_la_status s = check_seq(a);
  if (s != TTT_LA_OK) return s;
  const bool mom = a->beta != 0.f;
  if (!dW || (mom && (!dM || !GB)) || !aligned16(dW) || (dM && !aligned16(dM))) return TTT_LA_ERR_INVALID_ARG;
  // The map's state part is the forward's final state from W = M = 0.
  ttt_la_args b = *a;
  b.state_in = nullptr;
  b.mom_in = nullptr;
  b.state_out = dW;
  b.mom_out = mom ? dM : nullptr;
  s = ttt_la_forward_chunked(&b, stream);
  if (s != TTT_LA_OK || !mom) return s;
  ttt::MapScalarParams p;
  p.BH = a->B * a->H;
  p.T = a->T;
  p.eta = a->eta;
  p.eta_const = a->eta_const;
  p.beta = a->beta;
  p.GB = GB;
  const int blocks = (p.BH * 32 + 255) / 256;
  ttt::segment_scalars_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launched();
}

ttt_la_status ttt_la_compose_maps(int32_t nmaps, int32_t BH, int32_t d_v, int32_t d_k, const float* dW,
                                  const float* dM, const float* GB, const float* W0, const float* M0, float* W_out,
                                  float* M_out, void* stream) {
  NvtxRange range("ttt_la_compose_maps");
  if (nmaps < 0 || BH < 1 || d_v < 1 || d_k < 1 || !W_out || (nmaps > 0 && !dW)) return TTT_LA_ERR_INVALID_ARG;
  if ((dM == nullptr) != (GB == nullptr)) return TTT_LA_ERR_INVALID_ARG;
  if (static_cast<long long>(BH) * d_v * d_k >= (1ll << 40)) return TTT_LA_ERR_INVALID_ARG;
  ttt::ComposeParams p;
  p.nmaps = nmaps;
  p.DD = d_v * d_k;
  p.n = static_cast<long long>(BH) * p.DD;
  p.dW = dW;
  p.dM = dM;
  p.GB = GB;
  p.W0 = W0;
  p.M0 = M0;
  p.W_out = W_out;
  p.M_out = M_out;
  const long long want = (p.n + 255) / 256;
  const int blocks = static_cast<int>(std::min<long long>(want, static_cast<long long>(sm_count()) * 8));
  ttt::compose_maps_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launched();
}

ttt_la_status ttt_la_feature_map(const ttt_la_feature_args* a, void* stream) {
  NvtxRange range("ttt_la_feature_map");
  const ttt_la_status s = check_feature(a);
  if (s != TTT_LA_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a->d_in == 64) return a->d_out == 64 ? launch_feature<64, 64>(a, st) : launch_feature<64, 128>(a, st);
  return a->d_out == 64 ? launch_feature<128, 64>(a, st) : launch_feature<128, 128>(a, st);
}

size_t ttt_la_backward_workspace_size(const ttt_la_grad_args* a) {
  if (!a || a->B < 1 || a->H < 1 || a->T < 1 || a->d_k < 1 || a->d_v < 1) return 0;
  return bwd_ws_bytes(a);
}

ttt_la_status ttt_la_backward_recurrent(const ttt_la_grad_args* a, void* stream) {
  NvtxRange range("ttt_la_backward_recurrent");
  const ttt_la_status s = check_grad(a);
  if (s != TTT_LA_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool mom = a->beta != 0.f;
  if (a->dtype == TTT_LA_F32) return mom ? backward_dk<float, true>(a, st) : backward_dk<float, false>(a, st);
  return mom ? backward_dk<__nv_bfloat16, true>(a, st) : backward_dk<__nv_bfloat16, false>(a, st);
}

ttt_la_status ttt_la_forward_recurrent(const ttt_la_args* a, void* stream) {
  NvtxRange range("ttt_la_forward_recurrent");
  ttt_la_status s = check_seq(a);
  if (s != TTT_LA_OK) return s;
  if (a->d_v > 1024) return TTT_LA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool mom = a->beta != 0.f;
  if (a->dtype == TTT_LA_F32)
    return mom ? recurrent_dk<float, true>(a, st) : recurrent_dk<float, false>(a, st);
  return mom ? recurrent_dk<__nv_bfloat16, true>(a, st) : recurrent_dk<__nv_bfloat16, false>(a, st);
}

ttt_la_status ttt_la_decode_step(const ttt_la_decode_args* a, void* stream) {
  NvtxRange range("ttt_la_decode_step");
  if (!a) return TTT_LA_ERR_INVALID_ARG;
  if (a->N < 1 || a->H < 1 || a->d_k < 1 || a->d_v < 1) return TTT_LA_ERR_INVALID_ARG;
  if (a->dtype != TTT_LA_F32 && a->dtype != TTT_LA_BF16) return TTT_LA_ERR_INVALID_ARG;
  if (!a->q || !a->k || !a->v || !a->o || !a->state) return TTT_LA_ERR_INVALID_ARG;
  const bool mom = a->beta != 0.f;
  if (mom && !a->mom) return TTT_LA_ERR_INVALID_ARG;
  if (!(a->beta >= 0.f && a->beta < 1.f)) return TTT_LA_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o) || !aligned16(a->state) ||
      (a->mom && !aligned16(a->mom)) || (a->eta && !aligned16(a->eta)))
    return TTT_LA_ERR_INVALID_ARG;
  if (static_cast<long long>(a->N) * a->H * a->d_v >= (1ll << 31)) return TTT_LA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a->dtype == TTT_LA_F32) return mom ? decode_dk<float, true>(a, st) : decode_dk<float, false>(a, st);
  return mom ? decode_dk<__nv_bfloat16, true>(a, st) : decode_dk<__nv_bfloat16, false>(a, st);
}

ttt_la_status ttt_la_get_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TTT_LA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, ttt::g_status, sizeof(int)) != cudaSuccess) return TTT_LA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(ttt::g_status, &zero, sizeof(int)) != cudaSuccess) return TTT_LA_ERR_CUDA;
  if (v == 0) return TTT_LA_OK;
  return v == ttt::kStatusDeviceCheck ? TTT_LA_ERR_DEVICE_CHECK : TTT_LA_ERR_TIMEOUT;
}

int32_t ttt_la_debug_check_line(void* stream) {
  if (!ttt::kDebugChecks) return -1;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return -2;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, ttt::g_check_line, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(ttt::g_check_line, &zero, sizeof(int)) != cudaSuccess)
    return -2;
  return v;
}

ttt_la_status ttt_la_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return TTT_LA_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_ns));
  return launched();
}

}  // extern "C"

// Chunk-parallel backward without momentum: three runs of the chunked forward
// (see backward_chunked.cuh) over scratch carved from the caller's workspace.
// bf16: the two reverse-time passes run on the tensor cores in reverse chunk
// order and write dv (with deta) and dk themselves; fp32: they run on copies
// of the inputs reversed along T and a finishing kernel forms dv, dk, deta.
namespace {
struct BwdChunkedLayout {
  size_t rev[4], u, r, w0t, dwt, m0t, dmt, dw0, g0part, g0, fwd, total, fwd_bytes;
};

// Token splits of the momentum backward's dL/dW_0 kernel (64-token tiles).
int mom_g0_splits(int T) { return std::max(1, std::min(4, (T + 63) / 64)); }

bool bwdc_fused(const ttt_la_grad_args* a) { return a->dtype == TTT_LA_BF16; }
bool bwdc_mom(const ttt_la_grad_args* a) { return a->beta != 0.f; }

// Momentum: the dq pass, the momentum forward on (q, k, v) := (do, v, k)
// from W_0^T and M_0^T (64-token tiles).
ttt_la_args bwdc_mom_dq(const ttt_la_grad_args* a, const float* w0t, const float* m0t) {
  ttt_la_args f;
  std::memset(&f, 0, sizeof f);
  f.B = a->B;
  f.H = a->H;
  f.T = a->T;
  f.d_k = a->d_v;
  f.d_v = a->d_k;
  f.dtype = a->dtype;
  f.chunk = 64;
  f.beta = a->beta;
  f.q = a->grad_o;
  f.k = a->v;
  f.v = a->k;
  f.eta = a->eta;
  f.eta_const = a->eta_const;
  f.ascent = a->ascent;
  f.state_in = w0t;
  f.mom_in = m0t;
  f.o = a->grad_q;
  return f;
}

// The reverse passes' tiles: 64 tokens (bf16: 64 x 64, two blocks per SM, at
// d = 64; 64 x 128 at d = 128); fp32: the fp32 chunked path's 64.
int bwdc_chunk(const ttt_la_grad_args*) { return 64; }

// Arguments of forward pass p: 0 gives dq, 1 gives u = G k (bf16: dv) and
// dL/dW_0, 2 gives r = G^T v (bf16: dk).  fp32: rev[] are q, k, v, dO
// reversed along T, and u, r come out in reversed order.
ttt_la_args bwdc_pass(const ttt_la_grad_args* a, int p, void* const* rev, void* u, void* r, const float* w0t,
                      const float* dwt) {
  ttt_la_args f;
  std::memset(&f, 0, sizeof f);
  f.B = a->B;
  f.H = a->H;
  f.T = a->T;
  f.dtype = a->dtype;
  f.chunk = bwdc_chunk(a);
  f.beta = 0.f;
  const bool fused = bwdc_fused(a);
  // the reverse passes: the layer's eta and sigma for the fused epilogue, or
  // eta = 1, sigma = +1 for a plain run on reversed copies
  if (p > 0) {
    f.eta = fused ? a->eta : nullptr;
    f.eta_const = fused ? a->eta_const : 1.f;
    f.ascent = fused ? a->ascent : 0;
  }
  if (p == 0) {  // W_t^T do_t: keys v, values k, from W_0^T, the layer's eta and sigma
    // (a plain forward: bf16 takes the forward's own best tile, 64 tokens at d = 64, 128 at d = 128)
    if (a->dtype == TTT_LA_BF16) f.chunk = a->d_k == 64 ? 64 : 128;
    f.d_k = a->d_v;
    f.d_v = a->d_k;
    f.q = a->grad_o;
    f.k = a->v;
    f.v = a->k;
    f.eta = a->eta;
    f.eta_const = a->eta_const;
    f.ascent = a->ascent;
    f.state_in = w0t;
    f.o = a->grad_q;
  } else if (p == 1) {  // G_t k_t: reverse time, (q, k, v) := (k, q, dO), from dL/dW_T
    f.d_k = a->d_k;
    f.d_v = a->d_v;
    f.q = fused ? a->k : rev[1];
    f.k = fused ? a->q : rev[0];
    f.v = fused ? a->grad_o : rev[3];
    f.state_in = a->grad_state;
    f.state_out = a->grad_state_in;
    f.o = fused ? a->grad_v : u;
  } else {  // G_t^T v_t: reverse time, (q, k, v) := (v, dO, q), from (dL/dW_T)^T
    f.d_k = a->d_v;
    f.d_v = a->d_k;
    f.q = fused ? a->v : rev[2];
    f.k = fused ? a->grad_o : rev[3];
    f.v = fused ? a->q : rev[0];
    f.state_in = dwt;
    f.o = fused ? a->grad_k : r;
  }
  return f;
}

BwdChunkedLayout bwdc_layout(const ttt_la_grad_args* a) {
  BwdChunkedLayout L;
  std::memset(&L, 0, sizeof L);
  const size_t el = a->dtype == TTT_LA_F32 ? 4 : 2, bh = static_cast<size_t>(a->B) * a->H;
  const size_t ns = align256(bh * a->d_k * a->d_v * 4);
  size_t off = 0;
  if (!bwdc_fused(a)) {
    // q, k, v, dO reversed, then u and r (fp32)
    const size_t nk = align256(bh * a->T * a->d_k * el), nv = align256(bh * a->T * a->d_v * el);
    const size_t sizes[4] = {nk, nk, nv, nv};
    for (int i = 0; i < 4; ++i) {
      L.rev[i] = off;
      off += sizes[i];
    }
    L.u = off;
    off += align256(bh * a->T * a->d_v * 4);
    L.r = off;
    off += align256(bh * a->T * a->d_k * 4);
  }
  L.w0t = off;
  off += a->state_in ? ns : 0;
  L.dwt = off;
  off += a->grad_state ? ns : 0;
  const bool mom = bwdc_mom(a);
  L.m0t = off;  // momentum: M_0^T, (dL/dM_T)^T, and dL/dW_0 when the caller does not take it
  off += (mom && a->mom_in) ? ns : 0;
  L.dmt = off;
  off += (mom && a->grad_mom) ? ns : 0;
  L.dw0 = off;
  off += (mom && !a->grad_state_in) ? ns : 0;
  L.g0part = off;  // momentum: the dL/dW_0 kernel's partials, then their sum
  off += mom ? static_cast<size_t>(mom_g0_splits(a->T)) * ns : 0;
  L.g0 = off;
  off += mom ? ns : 0;
  L.fwd = off;
  L.fwd_bytes = 0;
  if (mom) {
    ttt_la_args f = bwdc_mom_dq(a, nullptr, nullptr);
    L.fwd_bytes = ttt_la_workspace_size(&f);
  } else {
    void* none[4] = {nullptr, nullptr, nullptr, nullptr};
    for (int p = 0; p < 3; ++p) {
      ttt_la_args f = bwdc_pass(a, p, none, nullptr, nullptr, nullptr, nullptr);
      L.fwd_bytes = std::max(L.fwd_bytes, ttt_la_workspace_size(&f));
    }
  }
  L.total = off + align256(L.fwd_bytes);
  return L;
}

ttt_la_status check_grad_chunked(const ttt_la_grad_args* a) {
  const ttt_la_status s = check_grad_common(a);
  if (s != TTT_LA_OK) return s;
  if (a->beta == 0.f && (a->mom_in || a->grad_mom)) return TTT_LA_ERR_UNSUPPORTED;
  if (a->beta != 0.f && a->dtype != TTT_LA_BF16) return TTT_LA_ERR_UNSUPPORTED;  // momentum: bf16 tensor cores
  if (a->dtype == TTT_LA_BF16 && !(a->d_k == a->d_v && (a->d_k == 64 || a->d_k == 128)))
    return TTT_LA_ERR_UNSUPPORTED;
  if (a->dtype == TTT_LA_F32 && (a->d_k % 4 || a->d_v % 4 || a->d_k > 128 || a->d_v > 128))
    return TTT_LA_ERR_UNSUPPORTED;
  if (!a->workspace || a->workspace_bytes < bwdc_layout(a).total) return TTT_LA_ERR_INVALID_ARG;
  return TTT_LA_OK;
}

// Momentum (bf16): transposes of W_0, M_0, dL/dW_T, dL/dM_T; dq from the
// momentum forward; dv, dL/dW_0, dL/dM_0 from the reverse kernel on (k, q,
// do); dk from it on (v, do, q) with the transposed states; deta from the
// forward-order kernel (backward_mom_tc.cuh).
template <int D>
ttt_la_status backward_chunked_mom(const ttt_la_grad_args* a, const BwdChunkedLayout& L, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  auto at = [&](bool present, size_t off) { return present ? reinterpret_cast<float*>(ws + off) : nullptr; };
  float* w0t = at(a->state_in != nullptr, L.w0t);
  float* dwt = at(a->grad_state != nullptr, L.dwt);
  float* m0t = at(a->mom_in != nullptr, L.m0t);
  float* dmt = at(a->grad_mom != nullptr, L.dmt);
  float* dw0 = a->grad_state_in ? a->grad_state_in : reinterpret_cast<float*>(ws + L.dw0);
  const int BH = a->B * a->H;
  ttt_la_status s;
  ttt::TransposeParams tp;
  std::memset(&tp, 0, sizeof tp);
  tp.BH = BH;
  tp.R = D;
  tp.C = D;
  const float* src[4] = {a->state_in, a->mom_in, a->grad_state, a->grad_mom};
  float* dst[4] = {w0t, m0t, dwt, dmt};
  for (int i = 0; i < 4; ++i)
    if (src[i]) {
      tp.src[tp.n] = src[i];
      tp.dst[tp.n++] = dst[i];
    }
  // deta is accumulated by the deta kernel's row blocks: zeroed here, which
  // saves a memset node ahead of that kernel
  tp.zero = a->grad_eta;
  tp.zero_n = static_cast<long long>(BH) * a->T;
  if (tp.n > 0 || tp.zero) {
    ttt::transpose_states_kernel<<<sm_count() * 4, 256, 0, st>>>(tp);
    if ((s = launched()) != TTT_LA_OK) return s;
  }
  ttt_la_args f = bwdc_mom_dq(a, w0t, m0t);
  f.workspace = L.fwd_bytes ? ws + L.fwd : nullptr;
  f.workspace_bytes = L.fwd_bytes;
  const float sigma = a->ascent ? -1.f : 1.f;
  {
    // After the transposes the launches form three independent chains:
    // dL/dW_0 then deta (the longest, the call's critical path) on a side
    // stream at the device's greatest priority, dv's reverse launch on a
    // second side stream, and dk's reverse launch then dq on the call's
    // stream, which waits for both side streams at the end.  deta starts
    // from its own dL/dW_0 (a short tensor-core reduction), not from the
    // reverse launch that also carries it.  dq fills the SMs the others
    // leave, so it runs with the look-back start states.  Without the side
    // streams the launches run one after the other on the call's stream, and
    // deta takes dL/dW_0 from the reverse launch.
    std::lock_guard<std::mutex> lock(side_mutex());
    SideStream side;
    const bool two = side_stream(st, &side);
    if (two) {
      float* part = reinterpret_cast<float*>(ws + L.g0part);
      float* g0 = reinterpret_cast<float*>(ws + L.g0);
      if (cudaEventRecord(side.fork, st) != cudaSuccess || cudaStreamWaitEvent(side.s, side.fork, 0) != cudaSuccess ||
          cudaStreamWaitEvent(side.s2, side.fork, 0) != cudaSuccess)
        return TTT_LA_ERR_CUDA;
      ttt_la_status s1 = TTT_LA_OK;
      if (a->grad_eta) {
        s1 = launch_mom_g0<D>(BH, a->T, mom_g0_splits(a->T), a->grad_o, a->q, a->grad_state, part, g0, side.s);
        if (s1 == TTT_LA_OK)
          s1 = launch_mom_deta<D>(BH, a->T, a->q, a->k, a->v, a->grad_o, sigma, a->beta, g0, a->mom_in, a->grad_eta,
                                  side.s);
      }
      if (cudaEventRecord(side.join, side.s) != cudaSuccess) s1 = TTT_LA_ERR_CUDA;
      ttt_la_status s2 = launch_mom_rev<D>(BH, a->T, a->k, a->q, a->grad_o, a->grad_v, a->eta, a->eta_const, sigma,
                                           a->beta, a->grad_state, a->grad_mom, dw0, a->grad_mom_in, side.s2);
      if (cudaEventRecord(side.join2, side.s2) != cudaSuccess) s2 = TTT_LA_ERR_CUDA;
      s = launch_mom_rev<D>(BH, a->T, a->v, a->grad_o, a->q, a->grad_k, a->eta, a->eta_const, sigma, a->beta, dwt,
                            dmt, nullptr, nullptr, st);
      if (s == TTT_LA_OK) {
        t_lookback_only = true;
        s = ttt_la_forward_chunked(&f, st);
        t_lookback_only = false;
      }
      if (cudaStreamWaitEvent(st, side.join, 0) != cudaSuccess || cudaStreamWaitEvent(st, side.join2, 0) != cudaSuccess)
        return TTT_LA_ERR_CUDA;
      return s1 != TTT_LA_OK ? s1 : s2 != TTT_LA_OK ? s2 : s;
    }
    s = launch_mom_rev<D>(BH, a->T, a->k, a->q, a->grad_o, a->grad_v, a->eta, a->eta_const, sigma, a->beta,
                          a->grad_state, a->grad_mom, dw0, a->grad_mom_in, st);
    if (s == TTT_LA_OK && a->grad_eta)
      s = launch_mom_deta<D>(BH, a->T, a->q, a->k, a->v, a->grad_o, sigma, a->beta, dw0, a->mom_in, a->grad_eta, st);
    if (s == TTT_LA_OK)
      s = launch_mom_rev<D>(BH, a->T, a->v, a->grad_o, a->q, a->grad_k, a->eta, a->eta_const, sigma, a->beta, dwt,
                            dmt, nullptr, nullptr, st);
    if (s == TTT_LA_OK) s = ttt_la_forward_chunked(&f, st);
    return s;
  }
}
}  // namespace

extern "C" {

size_t ttt_la_backward_chunked_workspace_size(const ttt_la_grad_args* a) {
  if (!a || a->B < 1 || a->H < 1 || a->T < 1 || a->d_k < 1 || a->d_v < 1) return 0;
  return bwdc_layout(a).total;
}

ttt_la_status ttt_la_backward_chunked(const ttt_la_grad_args* a, void* stream) {
  NvtxRange range("ttt_la_backward_chunked");
  ttt_la_status s = check_grad_chunked(a);
  if (s != TTT_LA_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const BwdChunkedLayout L = bwdc_layout(a);
  if (bwdc_mom(a))
    return a->d_k == 64 ? backward_chunked_mom<64>(a, L, st) : backward_chunked_mom<128>(a, L, st);
  const bool fused = bwdc_fused(a);
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  void* rev[4] = {ws + L.rev[0], ws + L.rev[1], ws + L.rev[2], ws + L.rev[3]};
  float* w0t = a->state_in ? reinterpret_cast<float*>(ws + L.w0t) : nullptr;
  float* dwt = a->grad_state ? reinterpret_cast<float*>(ws + L.dwt) : nullptr;
  const int BH = a->B * a->H, el = a->dtype == TTT_LA_F32 ? 4 : 2;
  const int grid = sm_count() * 4;

  // fp32: q, k (rows of d_k) and v, dO (rows of d_v) reversed along T
  for (int g = 0; g < 2 && !fused; ++g) {
    ttt::ReverseParams rp;
    std::memset(&rp, 0, sizeof rp);
    rp.n = 2;
    rp.BH = BH;
    rp.T = a->T;
    rp.units = ((g == 0 ? a->d_k : a->d_v) * el) / 16;
    rp.src[0] = static_cast<const uint4*>(g == 0 ? a->q : a->v);
    rp.src[1] = static_cast<const uint4*>(g == 0 ? a->k : a->grad_o);
    rp.dst[0] = static_cast<uint4*>(rev[2 * g]);
    rp.dst[1] = static_cast<uint4*>(rev[2 * g + 1]);
    ttt::reverse_tokens_kernel<<<grid, 256, 0, st>>>(rp);
    if ((s = launched()) != TTT_LA_OK) return s;
  }
  // W_0^T and (dL/dW_T)^T
  ttt::TransposeParams tp;
  std::memset(&tp, 0, sizeof tp);
  tp.BH = BH;
  tp.R = a->d_v;
  tp.C = a->d_k;
  if (a->state_in) {
    tp.src[tp.n] = a->state_in;
    tp.dst[tp.n++] = w0t;
  }
  if (a->grad_state) {
    tp.src[tp.n] = a->grad_state;
    tp.dst[tp.n++] = dwt;
  }
  if (tp.n > 0) {
    ttt::transpose_states_kernel<<<grid, 256, 0, st>>>(tp);
    if ((s = launched()) != TTT_LA_OK) return s;
  }
  // the three forward passes
  void* u = ws + L.u;
  void* r = ws + L.r;
  for (int p = 0; p < 3; ++p) {
    ttt_la_args f = bwdc_pass(a, p, rev, u, r, w0t, dwt);
    f.workspace = L.fwd_bytes ? ws + L.fwd : nullptr;
    f.workspace_bytes = L.fwd_bytes;
    if (p > 0 && fused)  // dv with deta (the layer's v dotted with u), then dk
      s = backward_pass_tc(&f, p == 1 ? a->v : nullptr, p == 1 ? a->grad_eta : nullptr, st);
    else
      s = ttt_la_forward_chunked(&f, stream);
    if (s != TTT_LA_OK) return s;
  }
  if (!fused) {
    // dv, dk, deta
    ttt::FinishParams fp;
    fp.BH = BH;
    fp.T = a->T;
    fp.dk = a->d_k;
    fp.dv = a->d_v;
    fp.u_rev = static_cast<const float*>(u);
    fp.r_rev = static_cast<const float*>(r);
    fp.v = static_cast<const float*>(a->v);
    fp.eta = a->eta;
    fp.eta_const = a->eta_const;
    fp.sigma = a->ascent ? -1.f : 1.f;
    fp.dk_out = static_cast<float*>(a->grad_k);
    fp.dv_out = static_cast<float*>(a->grad_v);
    fp.deta = a->grad_eta;
    const long long warps = static_cast<long long>(BH) * a->T;
    const unsigned blocks = static_cast<unsigned>((warps * 32 + 255) / 256);
    ttt::backward_finish_kernel<<<blocks, 256, 0, st>>>(fp);
    if ((s = launched()) != TTT_LA_OK) return s;
  }
  if (a->grad_mom_in &&
      cudaMemsetAsync(a->grad_mom_in, 0, static_cast<size_t>(BH) * a->d_v * a->d_k * sizeof(float), st) !=
          cudaSuccess)
    return TTT_LA_ERR_CUDA;
  return TTT_LA_OK;
}

}  // extern "C"

