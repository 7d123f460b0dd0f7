"""ctypes binding of libttt_la.so (include/ttt_la.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module only
fills the C structs with tensor pointers and sizes, allocates outputs and
scratch through PyTorch, and turns status codes into exceptions.  There is no
CPU path: if the shared library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libttt_la.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libttt_la_debug.so")  # built with -DTTT_LA_DEBUG (device-side bounds checks)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_SCRATCH_LIMIT, ERR_DEVICE_CHECK = 0, 1, 2, 3, 4, 5, 6
STATIC_SCRATCH_BYTES = 8 << 20  # TTT_LA_STATIC_SCRATCH_BYTES
F32, BF16 = 0, 1

_c_i32, _c_f32, _c_vp, _c_sz = ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class TttArgs(ctypes.Structure):
    """Mirror of ``ttt_la_args``."""
    _fields_ = [
        ("B", _c_i32), ("H", _c_i32), ("T", _c_i32), ("d_k", _c_i32), ("d_v", _c_i32), ("dtype", _c_i32),
        ("q", _c_vp), ("k", _c_vp), ("v", _c_vp), ("eta", _c_vp),
        ("eta_const", _c_f32), ("beta", _c_f32), ("ascent", _c_i32), ("chunk", _c_i32), ("segments", _c_i32),
        ("state_in", _c_vp), ("state_out", _c_vp), ("mom_in", _c_vp), ("mom_out", _c_vp),
        ("o", _c_vp), ("workspace", _c_vp), ("workspace_bytes", _c_sz),
    ]


class TttDecodeArgs(ctypes.Structure):
    """Mirror of ``ttt_la_decode_args``."""
    _fields_ = [
        ("N", _c_i32), ("H", _c_i32), ("d_k", _c_i32), ("d_v", _c_i32), ("dtype", _c_i32),
        ("q", _c_vp), ("k", _c_vp), ("v", _c_vp), ("eta", _c_vp),
        ("eta_const", _c_f32), ("beta", _c_f32), ("ascent", _c_i32),
        ("state", _c_vp), ("mom", _c_vp), ("o", _c_vp),
    ]


class TttFeatureArgs(ctypes.Structure):
    """Mirror of ``ttt_la_feature_args``."""
    _fields_ = [
        ("B", _c_i32), ("H", _c_i32), ("T", _c_i32), ("d_in", _c_i32), ("d_out", _c_i32), ("n_inputs", _c_i32),
        ("x", _c_vp * 2), ("y", _c_vp * 2), ("w1", _c_vp), ("w3", _c_vp),
    ]


class TttGradArgs(ctypes.Structure):
    """Mirror of ``ttt_la_grad_args``."""
    _fields_ = [
        ("B", _c_i32), ("H", _c_i32), ("T", _c_i32), ("d_k", _c_i32), ("d_v", _c_i32), ("dtype", _c_i32),
        ("q", _c_vp), ("k", _c_vp), ("v", _c_vp), ("eta", _c_vp),
        ("eta_const", _c_f32), ("beta", _c_f32), ("ascent", _c_i32),
        ("state_in", _c_vp), ("mom_in", _c_vp),
        ("grad_o", _c_vp), ("grad_state", _c_vp), ("grad_mom", _c_vp),
        ("grad_q", _c_vp), ("grad_k", _c_vp), ("grad_v", _c_vp),
        ("grad_eta", _c_vp), ("grad_state_in", _c_vp), ("grad_mom_in", _c_vp),
        ("workspace", _c_vp), ("workspace_bytes", _c_sz),
    ]


class TttPlan(ctypes.Structure):
    """Mirror of ``ttt_la_plan``."""
    _fields_ = [
        ("path", _c_i32), ("tile", _c_i32), ("segments", _c_i32), ("chunks_per_segment", _c_i32),
        ("cooperative", _c_i32), ("blocks", _c_i32), ("resident", _c_i32), ("waves", _c_i32),
        ("workspace_bytes", _c_sz),
    ]


# (name, restype, argtypes) for every symbol of include/ttt_la.h
SIGNATURES = [
    ("ttt_la_workspace_size", _c_sz, [ctypes.POINTER(TttArgs)]),
    ("ttt_la_forward_chunked", ctypes.c_int, [ctypes.POINTER(TttArgs), _c_vp]),
    ("ttt_la_chunked_plan", ctypes.c_int, [ctypes.POINTER(TttArgs), ctypes.POINTER(TttPlan)]),
    ("ttt_la_forward_chunked_noalloc", ctypes.c_int, [ctypes.POINTER(TttArgs), _c_vp]),
    ("ttt_la_host_staging_size", _c_sz, [ctypes.POINTER(TttArgs)]),
    ("ttt_la_forward_chunked_host", ctypes.c_int, [ctypes.POINTER(TttArgs), _c_vp, _c_sz, _c_vp]),
    ("ttt_la_forward_recurrent", ctypes.c_int, [ctypes.POINTER(TttArgs), _c_vp]),
    ("ttt_la_segment_map", ctypes.c_int, [ctypes.POINTER(TttArgs), _c_vp, _c_vp, _c_vp, _c_vp]),
    ("ttt_la_compose_maps", ctypes.c_int, [ctypes.c_int32] * 4 + [_c_vp] * 8),
    ("ttt_la_decode_step", ctypes.c_int, [ctypes.POINTER(TttDecodeArgs), _c_vp]),
    ("ttt_la_feature_map", ctypes.c_int, [ctypes.POINTER(TttFeatureArgs), _c_vp]),
    ("ttt_la_backward_workspace_size", _c_sz, [ctypes.POINTER(TttGradArgs)]),
    ("ttt_la_backward_recurrent", ctypes.c_int, [ctypes.POINTER(TttGradArgs), _c_vp]),
    ("ttt_la_backward_chunked_workspace_size", _c_sz, [ctypes.POINTER(TttGradArgs)]),
    ("ttt_la_backward_chunked", ctypes.c_int, [ctypes.POINTER(TttGradArgs), _c_vp]),
    ("ttt_la_get_last_device_status", ctypes.c_int, [_c_vp]),
    ("ttt_la_debug_check_line", _c_i32, [_c_vp]),
    ("ttt_la_set_wait_limit_ns", ctypes.c_int, [ctypes.c_int64]),
    ("ttt_la_selftest_wait_timeout", ctypes.c_int, [ctypes.c_int64, _c_vp]),
    ("ttt_la_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("ttt_la_version", ctypes.c_char_p, []),
]

_lib = None


class TttError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        msg = status_string(code) if _lib is not None else str(code)
        super().__init__(f"{fn} failed: {msg} (status {code})")


def _load(path):
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m test_layers_causal_b200.build`")
    L = ctypes.CDLL(path)
    for name, res, args in SIGNATURES:
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def lib():
    """Loads the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


_debug_lib = None


def debug_lib():
    """The debug build of the library (device-side bounds checks), loaded once
    beside the release one; the binding's functions keep using lib()."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = _load(DEBUG_LIB_PATH)
    return _debug_lib


def status_string(code: int) -> str:
    return lib().ttt_la_status_string(int(code)).decode()


def version() -> str:
    return lib().ttt_la_version().decode()


def _check(fn, code):
    if code != OK:
        raise TttError(fn, code)


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("inputs must be contiguous CUDA tensors")


def _seq_args(q, k, v, eta, eta_const, beta, ascent, chunk, segments, state_in, mom_in, o, S_out, M_out):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    a = TttArgs()
    a.B, a.H, a.T, a.d_k, a.d_v, a.dtype = B, H, T, dk, dv, _dtype_code(q)
    a.q, a.k, a.v, a.eta = q.data_ptr(), k.data_ptr(), v.data_ptr(), (eta.data_ptr() if eta is not None else None)
    a.eta_const = float(1.0 / math.sqrt(dk) if eta_const is None else eta_const)
    a.beta, a.ascent, a.chunk, a.segments = float(beta), int(bool(ascent)), int(chunk), int(segments)
    a.state_in = state_in.data_ptr() if state_in is not None else None
    a.mom_in = mom_in.data_ptr() if mom_in is not None else None
    a.state_out = S_out.data_ptr() if S_out is not None else None
    a.mom_out = M_out.data_ptr() if M_out is not None else None
    a.o = o.data_ptr()
    return a


def _check_shapes(q, k, v, eta, state_in, mom_in):
    if q.dim() != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k: [B,H,T,d_k]; v: [B,H,T,d_v]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share a dtype")
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if eta is not None and (eta.shape != (B, H, T) or eta.dtype != torch.float32):
        raise ValueError("eta must be fp32 [B,H,T]")
    for s in (state_in, mom_in):
        if s is not None and (s.shape != (B, H, dv, dk) or s.dtype != torch.float32):
            raise ValueError("state_in / mom_in must be fp32 [B,H,d_v,d_k]")
    _need_cuda(q, k, v, eta, state_in, mom_in)


def _check_buf(t, shape, dtype, name):
    """A caller-supplied buffer must have exactly the shape and dtype the
    library will write: a smaller one would be written past its end."""
    if t is not None and (tuple(t.shape) != tuple(shape) or t.dtype != dtype):
        raise ValueError(f"{name}: expected {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _alloc_outputs(q, v, beta, return_state, out, state_out=None, mom_out=None):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _check_buf(out, v.shape, v.dtype, "out")
    _check_buf(state_out, (B, H, dv, dk), torch.float32, "state_out")
    _check_buf(mom_out, (B, H, dv, dk), torch.float32, "mom_out")
    o = torch.empty_like(v) if out is None else out
    S = M = None
    if return_state:
        S = torch.empty(B, H, dv, dk, device=q.device, dtype=torch.float32) if state_out is None else state_out
        if beta != 0:
            M = torch.empty(B, H, dv, dk, device=q.device, dtype=torch.float32) if mom_out is None else mom_out
    return o, S, M


def forward_chunked(q, k, v, eta=None, eta_const=None, beta=0.0, ascent=False, chunk=64, segments=0,
                    state_in=None, mom_in=None, return_state=True, out=None, workspace=None, stream=None,
                    state_out=None, mom_out=None):
    """Chunk-parallel forward (ttt_la_forward_chunked).  Returns (o, W_T, M_T);
    W_T / M_T are None when not requested / without momentum.  `out`,
    `state_out`, `mom_out` and `workspace` may be preallocated buffers."""
    _check_shapes(q, k, v, eta, state_in, mom_in)
    o, S, M = _alloc_outputs(q, v, beta, return_state, out, state_out, mom_out)
    _need_cuda(o, S, M, workspace)
    a = _seq_args(q, k, v, eta, eta_const, beta, ascent, chunk, segments, state_in, mom_in, o, S, M)
    L = lib()
    need = L.ttt_la_workspace_size(ctypes.byref(a))
    if need:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("ttt_la_forward_chunked", L.ttt_la_forward_chunked(ctypes.byref(a), _stream_handle(stream)))
    return o, S, M


def forward_chunked_host(q, k, v, eta=None, eta_const=None, beta=0.0, ascent=False, chunk=64, segments=0,
                         state_in=None, mom_in=None, out=None, state_out=None, mom_out=None, staging=None,
                         stream=None):
    """Chunked forward on host tensors (ttt_la_forward_chunked_host): q, k, v,
    eta, state_in, mom_in are read from, and out / state_out / mom_out written
    to, contiguous CPU tensors (pinned ones let the copies overlap).  `staging`
    is a uint8 CUDA tensor of at least host_staging_bytes(...) bytes, allocated
    on the current device when missing or short.  Returns (o, staging); the
    outputs are complete once `stream` (default: the current one) is."""
    if q.dim() != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k: [B,H,T,d_k]; v: [B,H,T,d_v]")
    for t in (q, k, v, eta, state_in, mom_in, out, state_out, mom_out):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("forward_chunked_host takes contiguous host tensors")
    B, H, T, dk = q.shape
    _check_buf(out, v.shape, v.dtype, "out")
    for t, name in ((state_in, "state_in"), (mom_in, "mom_in"), (state_out, "state_out"), (mom_out, "mom_out")):
        _check_buf(t, (B, H, v.shape[-1], dk), torch.float32, name)
    _check_buf(eta, (B, H, T), torch.float32, "eta")
    o = torch.empty(v.shape, dtype=v.dtype, pin_memory=True) if out is None else out
    a = _seq_args(q, k, v, eta, eta_const, beta, ascent, chunk, segments, state_in, mom_in, o, state_out, mom_out)
    L = lib()
    need = int(L.ttt_la_host_staging_size(ctypes.byref(a)))
    if need == 0:
        raise ValueError("invalid arguments for ttt_la_forward_chunked_host")
    if staging is None or staging.numel() * staging.element_size() < need:
        staging = torch.empty(need, dtype=torch.uint8, device="cuda")
    _check("ttt_la_forward_chunked_host",
           L.ttt_la_forward_chunked_host(ctypes.byref(a), ctypes.c_void_p(staging.data_ptr()),
                                         staging.numel() * staging.element_size(), _stream_handle(stream)))
    return o, staging


def segment_map(q, k, v, eta=None, eta_const=None, beta=0.0, ascent=False, chunk=64, segments=0, scratch=None,
                workspace=None, stream=None):
    """Affine map of this run of tokens on the carried state
    (ttt_la_segment_map): returns (dW, dM, GB) with dW, dM [B,H,d_v,d_k] and
    GB [B,H,2] = (G, B); dM and GB are None without momentum.  `scratch`
    ([B,H,T,d_v] like v) receives throwaway outputs."""
    _check_shapes(q, k, v, eta, None, None)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _check_buf(scratch, v.shape, v.dtype, "scratch")
    _need_cuda(scratch, workspace)
    o = torch.empty_like(v) if scratch is None else scratch
    dW = torch.empty(B, H, dv, dk, device=q.device, dtype=torch.float32)
    dM = GB = None
    if beta != 0:
        dM = torch.empty_like(dW)
        GB = torch.empty(B, H, 2, device=q.device, dtype=torch.float32)
    a = _seq_args(q, k, v, eta, eta_const, beta, ascent, chunk, segments, None, None, o, None, None)
    L = lib()
    need = L.ttt_la_workspace_size(ctypes.byref(a))
    if need:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("ttt_la_segment_map", L.ttt_la_segment_map(ctypes.byref(a), _ptr(dW), _ptr(dM), _ptr(GB),
                                                      _stream_handle(stream)))
    return dW, dM, GB


def compose_maps(dW, dM=None, GB=None, W0=None, M0=None, stream=None):
    """Applies maps 0..n-1 in order to (W0, M0) (ttt_la_compose_maps): dW, dM
    [n,B,H,d_v,d_k], GB [n,B,H,2] (dM, GB None: no momentum); W0, M0
    [B,H,d_v,d_k] or None (zeros).  Returns (W, M); M is None when neither
    dM nor M0 is given."""
    if dW.dim() != 5:
        raise ValueError("dW must be [n,B,H,d_v,d_k]")
    n = dW.shape[0]
    B, H, dv, dk = dW.shape[1:]
    if (dM is None) != (GB is None):
        raise ValueError("dM and GB come together (maps with momentum) or not at all")
    for t, shape in ((dM, dW.shape), (GB, (n, B, H, 2)), (W0, (B, H, dv, dk)), (M0, (B, H, dv, dk))):
        if t is not None and (tuple(t.shape) != tuple(shape) or t.dtype != torch.float32):
            raise ValueError(f"compose_maps: expected fp32 {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")
    if dW.dtype != torch.float32:
        raise ValueError("dW must be fp32")
    _need_cuda(dW, dM, GB, W0, M0)
    W = torch.empty(B, H, dv, dk, device=dW.device, dtype=torch.float32)
    M = torch.empty_like(W) if (dM is not None or M0 is not None) else None
    _check("ttt_la_compose_maps", lib().ttt_la_compose_maps(
        n, B * H, dv, dk, _ptr(dW), _ptr(dM), _ptr(GB), _ptr(W0), _ptr(M0), _ptr(W), _ptr(M),
        _stream_handle(stream)))
    return W, M


def feature_map(xs, W1, W3, out=None, stream=None):
    """phi(x) = silu(W1 x) * (W3 x) of one or two bf16 inputs in one launch
    (ttt_la_feature_map).  xs: a tensor or a sequence of one or two tensors
    [B,H,T,d_in]; W1, W3: bf16 [H,d_out,d_in].  Returns a list of bf16
    [B,H,T,d_out] tensors (written into `out` when given)."""
    xs = [xs] if torch.is_tensor(xs) else list(xs)
    if not 1 <= len(xs) <= 2:
        raise ValueError("one or two inputs")
    x0 = xs[0]
    if x0.dim() != 4 or any(x.shape != x0.shape for x in xs):
        raise ValueError("inputs must share one [B,H,T,d_in] shape")
    B, H, T, d_in = x0.shape
    if W1.dim() != 3 or W1.shape != W3.shape or W1.shape[0] != H or W1.shape[2] != d_in:
        raise ValueError("W1, W3 must be [H,d_out,d_in]")
    if any(t.dtype != torch.bfloat16 for t in (*xs, W1, W3)):
        raise TypeError("the feature map takes bf16 inputs and weights")
    if not all(t.is_contiguous() for t in (*xs, W1, W3)):
        raise ValueError("inputs and weights must be contiguous")
    _need_cuda(*xs, W1, W3, *(out or []))
    d_out = W1.shape[1]
    ys = list(out) if out is not None else [torch.empty(B, H, T, d_out, device=x0.device, dtype=torch.bfloat16)
                                            for _ in xs]
    if len(ys) != len(xs) or any(y.shape != (B, H, T, d_out) or y.dtype != torch.bfloat16 or not y.is_contiguous()
                                 for y in ys):
        raise ValueError("out: one contiguous bf16 [B,H,T,d_out] tensor per input")
    a = TttFeatureArgs()
    a.B, a.H, a.T, a.d_in, a.d_out, a.n_inputs = B, H, T, d_in, d_out, len(xs)
    for i, (x, y) in enumerate(zip(xs, ys)):
        a.x[i] = x.data_ptr()
        a.y[i] = y.data_ptr()
    a.w1, a.w3 = W1.data_ptr(), W3.data_ptr()
    _check("ttt_la_feature_map", lib().ttt_la_feature_map(ctypes.byref(a), _stream_handle(stream)))
    return ys


def forward_chunked_phi(q, k, v, W1, W3, eta=None, **kw):
    """The layer whose fast weight is the last layer of a frozen gated MLP:
    phi(q), phi(k) by ttt_la_feature_map (one launch for both), then the
    chunked forward on (phi(q), phi(k), v) with d_k = d_out.  Keyword
    arguments as forward_chunked.  Returns forward_chunked's (o, S, M)."""
    fq, fk = feature_map([q, k], W1, W3, stream=kw.get("stream"))
    return forward_chunked(fq, fk, v, eta, **kw)


def backward_recurrent(q, k, v, grad_o, eta=None, eta_const=None, beta=0.0, ascent=False, state_in=None,
                       mom_in=None, grad_state=None, grad_mom=None, workspace=None, stream=None):
    """Gradients of the layer (ttt_la_backward_recurrent): returns a dict with
    dq, dk, dv (dtype of q), deta [B,H,T] fp32 (per token), dW0 and dM0
    [B,H,d_v,d_k] fp32 (dM0 None without momentum)."""
    _check_shapes(q, k, v, eta, state_in, mom_in)
    if grad_o.shape != v.shape or grad_o.dtype != v.dtype or not grad_o.is_contiguous():
        raise ValueError("grad_o must match v")
    state_shape = (q.shape[0], q.shape[1], v.shape[-1], q.shape[-1])
    for t in (grad_state, grad_mom):
        if t is not None and (t.shape != state_shape or t.dtype != torch.float32):
            raise ValueError("grad_state / grad_mom must be fp32 [B,H,d_v,d_k]")
    _need_cuda(q, k, v, grad_o, eta, state_in, mom_in, grad_state, grad_mom)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               deta=torch.empty(B, H, T, device=q.device, dtype=torch.float32),
               dW0=torch.empty(B, H, dv, dk, device=q.device, dtype=torch.float32),
               dM0=torch.empty(B, H, dv, dk, device=q.device, dtype=torch.float32) if beta else None)
    a = TttGradArgs()
    a.B, a.H, a.T, a.d_k, a.d_v, a.dtype = B, H, T, dk, dv, _dtype_code(q)
    a.q, a.k, a.v, a.eta = q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(eta)
    a.eta_const = (1.0 / math.sqrt(dk)) if eta_const is None else float(eta_const)
    a.beta, a.ascent = float(beta), int(bool(ascent))
    a.state_in, a.mom_in = _ptr(state_in), _ptr(mom_in)
    a.grad_o, a.grad_state, a.grad_mom = grad_o.data_ptr(), _ptr(grad_state), _ptr(grad_mom)
    a.grad_q, a.grad_k, a.grad_v = out["dq"].data_ptr(), out["dk"].data_ptr(), out["dv"].data_ptr()
    a.grad_eta, a.grad_state_in, a.grad_mom_in = _ptr(out["deta"]), _ptr(out["dW0"]), _ptr(out["dM0"])
    L = lib()
    need = L.ttt_la_backward_workspace_size(ctypes.byref(a))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("ttt_la_backward_recurrent", L.ttt_la_backward_recurrent(ctypes.byref(a), _stream_handle(stream)))
    return out


def _chunked_grad_args(q, k, v, grad_o, eta, eta_const, ascent, state_in, grad_state, beta=0.0, mom_in=None,
                       grad_mom=None):
    """The TttGradArgs of ttt_la_backward_chunked and the output tensors it
    points at (no workspace yet)."""
    _check_shapes(q, k, v, eta, state_in, mom_in)
    if grad_o.shape != v.shape or grad_o.dtype != v.dtype:
        raise ValueError("grad_o must match v")
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    for t in (grad_state, grad_mom):
        if t is not None and (t.shape != (B, H, dv, dk) or t.dtype != torch.float32):
            raise ValueError("grad_state / grad_mom must be fp32 [B,H,d_v,d_k]")
    _need_cuda(q, k, v, grad_o, eta, state_in, grad_state, mom_in, grad_mom)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               deta=torch.empty(B, H, T, device=q.device, dtype=torch.float32),
               dW0=torch.empty(B, H, dv, dk, device=q.device, dtype=torch.float32),
               dM0=torch.empty(B, H, dv, dk, device=q.device, dtype=torch.float32) if beta else None)
    a = TttGradArgs()
    a.B, a.H, a.T, a.d_k, a.d_v, a.dtype = B, H, T, dk, dv, _dtype_code(q)
    a.q, a.k, a.v, a.eta = q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(eta)
    a.eta_const = (1.0 / math.sqrt(dk)) if eta_const is None else float(eta_const)
    a.beta, a.ascent = float(beta), int(bool(ascent))
    a.state_in, a.grad_o, a.grad_state = _ptr(state_in), grad_o.data_ptr(), _ptr(grad_state)
    a.mom_in, a.grad_mom = _ptr(mom_in), _ptr(grad_mom)
    a.grad_q, a.grad_k, a.grad_v = out["dq"].data_ptr(), out["dk"].data_ptr(), out["dv"].data_ptr()
    a.grad_eta, a.grad_state_in = out["deta"].data_ptr(), out["dW0"].data_ptr()
    a.grad_mom_in = _ptr(out["dM0"])
    return a, out


def backward_chunked(q, k, v, grad_o, eta=None, eta_const=None, ascent=False, state_in=None, grad_state=None,
                     workspace=None, stream=None, beta=0.0, mom_in=None, grad_mom=None):
    """Gradients of the layer from its chunk-parallel form
    (ttt_la_backward_chunked): returns a dict with dq, dk, dv (dtype of q),
    deta [B,H,T] fp32 (per token), dW0 [B,H,d_v,d_k] fp32 and, with momentum
    (beta != 0: bf16, d_k == d_v in {64, 128}), dM0 (else None)."""
    _need_cuda(workspace)
    a, out = _chunked_grad_args(q, k, v, grad_o, eta, eta_const, ascent, state_in, grad_state, beta, mom_in,
                                grad_mom)
    L = lib()
    need = L.ttt_la_backward_chunked_workspace_size(ctypes.byref(a))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("ttt_la_backward_chunked", L.ttt_la_backward_chunked(ctypes.byref(a), _stream_handle(stream)))
    return out


def workspace_bytes(q, v, chunk=64, beta=0.0, segments=0):
    """Scratch bytes ttt_la_forward_chunked needs for these shapes."""
    B, H, T, dk = q.shape
    a = TttArgs()
    a.B, a.H, a.T, a.d_k, a.d_v, a.dtype = B, H, T, dk, v.shape[-1], _dtype_code(q)
    a.q, a.k, a.v, a.o = 16, 32, 48, 64  # never dereferenced by the size query
    a.beta, a.chunk, a.segments = float(beta), int(chunk), int(segments)
    return int(lib().ttt_la_workspace_size(ctypes.byref(a)))


def chunked_plan(B, H, T, d_k, d_v, dtype="bf16", chunk=64, beta=0.0, segments=0, eta=False):
    """How ttt_la_forward_chunked would run these shapes on the current device
    (ttt_la_chunked_plan; no launch, no tensors): a dict of the plan's fields."""
    a = TttArgs()
    a.B, a.H, a.T, a.d_k, a.d_v = B, H, T, d_k, d_v
    a.dtype = BF16 if dtype == "bf16" else F32
    a.q, a.k, a.v, a.o = 16, 32, 48, 64  # never dereferenced by the query
    a.eta = 80 if eta else None
    a.eta_const = 1.0 / math.sqrt(d_k)
    a.beta, a.chunk, a.segments = float(beta), int(chunk), int(segments)
    p = TttPlan()
    _check("ttt_la_chunked_plan", lib().ttt_la_chunked_plan(ctypes.byref(a), ctypes.byref(p)))
    return {name: getattr(p, name) for name, _ in TttPlan._fields_}


def forward_recurrent(q, k, v, eta=None, eta_const=None, beta=0.0, ascent=False, state_in=None, mom_in=None,
                      return_state=True, out=None, stream=None):
    """Token-by-token forward (ttt_la_forward_recurrent).  Returns (o, W_T, M_T)."""
    _check_shapes(q, k, v, eta, state_in, mom_in)
    o, S, M = _alloc_outputs(q, v, beta, return_state, out)
    _need_cuda(o)
    a = _seq_args(q, k, v, eta, eta_const, beta, ascent, 0, 0, state_in, mom_in, o, S, M)
    _check("ttt_la_forward_recurrent", lib().ttt_la_forward_recurrent(ctypes.byref(a), _stream_handle(stream)))
    return o, S, M


def decode_step(q, k, v, state, mom=None, eta=None, eta_const=None, beta=0.0, ascent=False, out=None,
                stream=None):
    """One decode step (ttt_la_decode_step): q, k [N,H,d_k], v [N,H,d_v];
    state (and mom with momentum) [N,H,d_v,d_k] fp32 updated in place.
    Returns o [N,H,d_v]."""
    if q.dim() != 3 or k.shape != q.shape or v.shape[:2] != q.shape[:2]:
        raise ValueError("q, k: [N,H,d_k]; v: [N,H,d_v]")
    N, H, dk = q.shape
    dv = v.shape[-1]
    if state.shape != (N, H, dv, dk) or state.dtype != torch.float32:
        raise ValueError("state must be fp32 [N,H,d_v,d_k]")
    if eta is not None and (eta.shape != (N, H) or eta.dtype != torch.float32):
        raise ValueError("eta must be fp32 [N,H]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share a dtype")
    _check_buf(mom, (N, H, dv, dk), torch.float32, "mom")
    _check_buf(out, v.shape, v.dtype, "out")
    _need_cuda(q, k, v, state, mom, eta, out)
    o = torch.empty_like(v) if out is None else out
    a = TttDecodeArgs()
    a.N, a.H, a.d_k, a.d_v, a.dtype = N, H, dk, dv, _dtype_code(q)
    a.q, a.k, a.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    a.eta = eta.data_ptr() if eta is not None else None
    a.eta_const = float(1.0 / math.sqrt(dk) if eta_const is None else eta_const)
    a.beta, a.ascent = float(beta), int(bool(ascent))
    a.state, a.mom, a.o = state.data_ptr(), (mom.data_ptr() if mom is not None else None), o.data_ptr()
    _check("ttt_la_decode_step", lib().ttt_la_decode_step(ctypes.byref(a), _stream_handle(stream)))
    return o


def device_status(stream=None) -> int:
    """Synchronises and returns (then clears) the device status word."""
    return int(lib().ttt_la_get_last_device_status(_stream_handle(stream)))


def set_wait_limit_ns(ns: int):
    _check("ttt_la_set_wait_limit_ns", lib().ttt_la_set_wait_limit_ns(int(ns)))


def selftest_wait_timeout(ns: int, stream=None):
    _check("ttt_la_selftest_wait_timeout", lib().ttt_la_selftest_wait_timeout(int(ns), _stream_handle(stream)))
