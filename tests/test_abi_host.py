"""Host-side checks of the C ABI (no GPU needed, nothing is launched):
the library loads, exports every symbol include/ttt_la.h declares, the ctypes
structs match the C layout, and bad arguments are rejected before launch."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "include", "ttt_la.h")


@pytest.fixture(scope="module")
def abi():
    from test_layers_causal_b200 import _abi
    from test_layers_causal_b200.build import build
    build()
    _abi.lib()
    return _abi


def declared_functions():
    src = open(HDR).read()
    return re.findall(r"TTT_LA_API\s+[\w\s\*]+?\b(ttt_la_\w+)\s*\(", src)


def test_header_declares_entry_points():
    names = set(declared_functions())
    for n in ("ttt_la_forward_chunked", "ttt_la_forward_recurrent", "ttt_la_decode_step",
              "ttt_la_workspace_size", "ttt_la_get_last_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(abi):
    L = abi.lib()
    for n in declared_functions():
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (ttt_la_\w+)", out))
    assert set(declared_functions()) <= exported
    assert {name for name, _, _ in abi.SIGNATURES} == set(declared_functions())


def test_struct_layout_matches_c(abi):
    """Compile a probe against the header with gcc and compare sizeof/offsetof."""
    probe = r"""
#include <stdio.h>
#include <stddef.h>
#include "ttt_la.h"
#define P(T, f) printf(#T "." #f " %zu\n", offsetof(T, f))
int main(void) {
  printf("ttt_la_args %zu\n", sizeof(ttt_la_args));
  printf("ttt_la_decode_args %zu\n", sizeof(ttt_la_decode_args));
  P(ttt_la_args, q); P(ttt_la_args, eta); P(ttt_la_args, eta_const); P(ttt_la_args, segments);
  P(ttt_la_args, state_in); P(ttt_la_args, o); P(ttt_la_args, workspace_bytes);
  P(ttt_la_decode_args, q); P(ttt_la_decode_args, eta_const); P(ttt_la_decode_args, state);
  P(ttt_la_decode_args, o);
  printf("ttt_la_feature_args %zu\n", sizeof(ttt_la_feature_args));
  P(ttt_la_feature_args, n_inputs); P(ttt_la_feature_args, x); P(ttt_la_feature_args, y);
  P(ttt_la_feature_args, w1); P(ttt_la_feature_args, w3);
  printf("ttt_la_grad_args %zu\n", sizeof(ttt_la_grad_args));
  P(ttt_la_grad_args, q); P(ttt_la_grad_args, eta_const); P(ttt_la_grad_args, state_in);
  P(ttt_la_grad_args, grad_o); P(ttt_la_grad_args, grad_q); P(ttt_la_grad_args, grad_eta);
  P(ttt_la_grad_args, grad_mom_in); P(ttt_la_grad_args, workspace_bytes);
  printf("ttt_la_plan %zu\n", sizeof(ttt_la_plan));
  P(ttt_la_plan, cooperative); P(ttt_la_plan, resident); P(ttt_la_plan, workspace_bytes);
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "probe.c")
        exe = os.path.join(d, "probe")
        open(c, "w").write(probe)
        subprocess.run(["gcc", "-I" + os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    vals = dict(l.split() for l in lines if l.strip())
    assert int(vals["ttt_la_args"]) == ctypes.sizeof(abi.TttArgs)
    assert int(vals["ttt_la_decode_args"]) == ctypes.sizeof(abi.TttDecodeArgs)
    assert int(vals["ttt_la_feature_args"]) == ctypes.sizeof(abi.TttFeatureArgs)
    assert int(vals["ttt_la_grad_args"]) == ctypes.sizeof(abi.TttGradArgs)
    assert int(vals["ttt_la_plan"]) == ctypes.sizeof(abi.TttPlan)
    classes = {"ttt_la_args": abi.TttArgs, "ttt_la_decode_args": abi.TttDecodeArgs,
               "ttt_la_feature_args": abi.TttFeatureArgs, "ttt_la_grad_args": abi.TttGradArgs,
               "ttt_la_plan": abi.TttPlan}
    for key, v in vals.items():
        if "." in key:
            struct, field = key.split(".")
            cls = classes[struct]
            assert getattr(cls, field).offset == int(v), key


def test_status_strings(abi):
    L = abi.lib()
    assert L.ttt_la_status_string(0) == b"ok"
    assert b"timed out" in L.ttt_la_status_string(4)
    assert b"sm_100a" in L.ttt_la_version()


def _args(abi, **kw):
    a = abi.TttArgs()
    a.B, a.H, a.T, a.d_k, a.d_v, a.dtype = 1, 2, 100, 64, 64, abi.BF16
    a.q, a.k, a.v, a.o = 0x10000, 0x20000, 0x30000, 0x40000  # never dereferenced on these paths
    a.chunk, a.eta_const = 64, 0.125
    for n, x in kw.items():
        setattr(a, n, x)
    return a


@pytest.mark.parametrize("bad", [
    dict(B=0), dict(T=0), dict(d_k=0), dict(dtype=7), dict(q=None), dict(o=None),
    dict(q=0x10004), dict(eta=0x1008), dict(state_in=0x2004), dict(o=0x10000),
    dict(beta=1.5), dict(beta=-0.5),
])
def test_invalid_arguments_rejected_before_launch(abi, bad):
    L = abi.lib()
    a = _args(abi, **bad)
    assert L.ttt_la_forward_chunked(ctypes.byref(a), None) == abi.ERR_INVALID_ARG
    assert L.ttt_la_forward_recurrent(ctypes.byref(a), None) == abi.ERR_INVALID_ARG
    assert L.ttt_la_workspace_size(ctypes.byref(a)) == 0
    assert L.ttt_la_host_staging_size(ctypes.byref(a)) == 0
    assert L.ttt_la_forward_chunked_host(ctypes.byref(a), ctypes.c_void_p(0x100000), 1 << 30, None) == \
        abi.ERR_INVALID_ARG


@pytest.mark.parametrize("cfg", [
    dict(d_k=96, d_v=96), dict(d_k=64, d_v=128), dict(chunk=32), dict(chunk=256),
    dict(dtype=0, chunk=128), dict(dtype=0, d_k=256, d_v=256, chunk=64),
    dict(dtype=0, d_k=128, d_v=128, beta=0.9, chunk=64), dict(beta=0.9, chunk=32),
])
def test_unsupported_combinations(abi, cfg):
    L = abi.lib()
    a = _args(abi, **cfg)
    assert L.ttt_la_forward_chunked(ctypes.byref(a), None) == abi.ERR_UNSUPPORTED


def test_recurrent_unsupported_head_dim(abi):
    a = _args(abi, d_k=48, d_v=48)
    assert abi.lib().ttt_la_forward_recurrent(ctypes.byref(a), None) == abi.ERR_UNSUPPORTED


def test_decode_validation(abi):
    L = abi.lib()
    d = abi.TttDecodeArgs()
    d.N, d.H, d.d_k, d.d_v, d.dtype = 4, 2, 128, 128, abi.BF16
    d.q, d.k, d.v, d.o, d.state = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    d.beta = 0.9  # momentum without a buffer
    assert L.ttt_la_decode_step(ctypes.byref(d), None) == abi.ERR_INVALID_ARG
    d.beta, d.state = 0.0, 0x50008  # misaligned state
    assert L.ttt_la_decode_step(ctypes.byref(d), None) == abi.ERR_INVALID_ARG
    d.state, d.N = 0x50000, 0
    assert L.ttt_la_decode_step(ctypes.byref(d), None) == abi.ERR_INVALID_ARG
    assert L.ttt_la_decode_step(None, None) == abi.ERR_INVALID_ARG


def _feature_args(abi, B=2, H=4, T=300, d_in=64, d_out=64, n=2):
    f = abi.TttFeatureArgs()
    f.B, f.H, f.T, f.d_in, f.d_out, f.n_inputs = B, H, T, d_in, d_out, n
    # fake, disjoint, 16-byte aligned device addresses: nothing is launched
    # because every case below fails a host-side check
    f.x[0], f.x[1], f.y[0], f.y[1] = 0x1000000, 0x2000000, 0x3000000, 0x4000000
    f.w1, f.w3 = 0x5000000, 0x5100000
    return f


def test_feature_map_validation(abi):
    L = abi.lib()
    call = lambda f: L.ttt_la_feature_map(ctypes.byref(f), None)  # noqa: E731
    assert L.ttt_la_feature_map(None, None) == abi.ERR_INVALID_ARG
    for field, val in [("B", 0), ("T", 0), ("H", -1), ("n_inputs", 0), ("n_inputs", 3)]:
        f = _feature_args(abi)
        setattr(f, field, val)
        assert call(f) == abi.ERR_INVALID_ARG, field
    f = _feature_args(abi)
    f.x[1] = 0x2000008  # misaligned input
    assert call(f) == abi.ERR_INVALID_ARG
    f = _feature_args(abi)
    f.w3 = 0  # missing weight
    assert call(f) == abi.ERR_INVALID_ARG
    f = _feature_args(abi)
    f.y[0] = f.x[1] + 4096  # output overlaps an input
    assert call(f) == abi.ERR_INVALID_ARG
    f = _feature_args(abi)
    f.y[1] = f.y[0] + 4096  # the two outputs overlap
    assert call(f) == abi.ERR_INVALID_ARG
    f = _feature_args(abi)
    f.y[0] = f.w1 - 16  # output runs into the weights
    assert call(f) == abi.ERR_INVALID_ARG
    for d_in, d_out in [(32, 64), (64, 96), (256, 128)]:
        assert call(_feature_args(abi, d_in=d_in, d_out=d_out)) == abi.ERR_UNSUPPORTED
    # a single input leaves the second slots unused: junk there is ignored
    f = _feature_args(abi, n=1, d_in=32)
    f.x[1], f.y[1] = 0x7, 0x3000000
    assert call(f) == abi.ERR_UNSUPPORTED


def _grad_args(abi, B=2, H=2, T=100, dk=64, dv=64, beta=0.0):
    g = abi.TttGradArgs()
    g.B, g.H, g.T, g.d_k, g.d_v, g.dtype, g.beta = B, H, T, dk, dv, abi.BF16, beta
    # fake, disjoint, 16-byte aligned addresses: every case below fails a host check
    g.q, g.k, g.v, g.grad_o = 0x1000000, 0x2000000, 0x3000000, 0x4000000
    g.grad_q, g.grad_k, g.grad_v = 0x5000000, 0x6000000, 0x7000000
    g.workspace = 0x10000000
    g.workspace_bytes = abi.lib().ttt_la_backward_workspace_size(ctypes.byref(g))
    return g


def test_backward_workspace_and_validation(abi):
    L = abi.lib()
    call = lambda g: L.ttt_la_backward_recurrent(ctypes.byref(g), None)  # noqa: E731
    size = lambda g: L.ttt_la_backward_workspace_size(ctypes.byref(g))  # noqa: E731
    # checkpoints every 32 tokens plus one chunk of history, W (and M) per head
    g = _grad_args(abi, T=100)
    assert size(g) == 2 * 2 * (4 + 32) * 1 * 64 * 64 * 4
    assert size(_grad_args(abi, T=100, beta=0.9)) == 2 * 2 * (4 + 32) * 2 * 64 * 64 * 4
    assert L.ttt_la_backward_workspace_size(None) == 0
    assert L.ttt_la_backward_recurrent(None, None) == abi.ERR_INVALID_ARG
    for field, val in [("T", 0), ("B", 0), ("beta", 1.0), ("beta", -0.1), ("grad_o", 0), ("grad_v", 0x7000008),
                       ("workspace_bytes", 16)]:
        g = _grad_args(abi)
        setattr(g, field, val)
        assert call(g) == abi.ERR_INVALID_ARG, field
    g = _grad_args(abi)
    g.grad_q = g.q + 64  # output overlaps an input
    assert call(g) == abi.ERR_INVALID_ARG
    g = _grad_args(abi)
    g.grad_eta = g.grad_k + 256  # two outputs overlap
    assert call(g) == abi.ERR_INVALID_ARG
    for dk, dv in [(48, 64), (128, 256), (64, 512)]:
        assert call(_grad_args(abi, dk=dk, dv=dv)) == abi.ERR_UNSUPPORTED


def test_workspace_query(abi):
    L = abi.lib()
    def expected(bh, nseg, d):  # fp32 [bh][nseg][2][d][d], bh*nseg flags, tile counter, bh head counters
        b = bh * nseg * 2 * d * d * 4 + (bh * nseg + 1 + bh) * 4
        return (b + 15) // 16 * 16

    one_seq_long = _args(abi, B=1, H=1, T=65536, chunk=128)
    ws = L.ttt_la_workspace_size(ctypes.byref(one_seq_long))
    assert ws > 0 and ws % 16 == 0
    many = _args(abi, B=64, H=16, T=256, chunk=64)  # enough sequences: no split
    assert L.ttt_la_workspace_size(ctypes.byref(many)) == 0
    fixed = _args(abi, B=1, H=1, T=64 * 10, chunk=64, segments=3)  # 10 chunks -> 4+4+2
    assert L.ttt_la_workspace_size(ctypes.byref(fixed)) == expected(1, 3, 64)
    fixed4 = _args(abi, B=2, H=3, T=64 * 10, chunk=64, segments=4)  # 10 chunks -> 3+3+3+1
    assert L.ttt_la_workspace_size(ctypes.byref(fixed4)) == expected(6, 4, 64)
    # a request beyond one wave of resident blocks is honoured (64 chunks / 40 -> 32 segments of 2)
    wide = _args(abi, B=4, H=16, T=64 * 64, chunk=64, segments=40)
    assert L.ttt_la_workspace_size(ctypes.byref(wide)) == expected(64, 32, 64)
    # short workspace is refused on the host
    fixed.workspace, fixed.workspace_bytes = 0x60000, 100
    assert L.ttt_la_forward_chunked(ctypes.byref(fixed), None) == abi.ERR_INVALID_ARG
    assert L.ttt_la_set_wait_limit_ns(10) == abi.ERR_INVALID_ARG
    assert L.ttt_la_selftest_wait_timeout(10, None) == abi.ERR_INVALID_ARG


def test_chunked_plan_launch_modes(abi, monkeypatch):
    """Blocks of a head that wait for one another (cooperative start states)
    are launched cooperatively, which guarantees they are resident together;
    the plan the launch uses is the one the query reports.  Without a GPU the
    plan is that of a 148-SM B200 (one 128-wide tile per SM, two 64 x 64)."""
    long_ctx = abi.chunked_plan(1, 8, 65536, 128, 128, chunk=128)
    assert long_ctx["path"] == 0 and long_ctx["cooperative"] == 1
    assert long_ctx["segments"] == 18 and long_ctx["blocks"] == 144 <= long_ctx["resident"] == 148
    # by default a single wave; runs of about 512 tokens: 512 chunks / (18 x 4) -> 7 waves
    assert long_ctx["waves"] == 1
    monkeypatch.setenv("TTT_LA_WAVE_TOKENS", "512")
    assert abi.chunked_plan(1, 8, 65536, 128, 128, chunk=128)["waves"] == 7
    long64 = abi.chunked_plan(1, 8, 65536, 128, 128, chunk=64)
    assert long64["cooperative"] == 1 and long64["waves"] == 1024 // (18 * 8)
    monkeypatch.delenv("TTT_LA_WAVE_TOKENS")
    # the merged 64 x 64 tile keeps the decoupled look-back even for one long sequence
    d64 = abi.chunked_plan(1, 1, 64 * 400, 64, 64, chunk=64)
    assert d64["cooperative"] == 0 and d64["waves"] == 1
    mom = abi.chunked_plan(2, 16, 8192, 128, 128, chunk=128, beta=0.9, eta=True)
    assert mom["path"] == 1 and mom["tile"] == 64 and mom["cooperative"] == 1 and mom["blocks"] <= mom["resident"]
    assert mom["waves"] == 1
    llm = abi.chunked_plan(4, 16, 4096, 64, 64, chunk=64, eta=True)  # short look-back: no waiting on peers
    assert llm["path"] == 0 and llm["cooperative"] == 0 and llm["segments"] == 4 and llm["resident"] == 296
    # a grid beyond one wave never waits on peers
    wide = abi.chunked_plan(1, 8, 65536, 128, 128, chunk=128, segments=40)
    assert wide["cooperative"] == 0 and wide["blocks"] == 320
    # one segment per sequence: no scratch, nothing to wait for
    many = abi.chunked_plan(64, 16, 256, 64, 64, chunk=64)
    assert many["segments"] == 1 and many["cooperative"] == 0 and many["workspace_bytes"] == 0
    f32 = abi.chunked_plan(1, 2, 256, 32, 32, dtype="f32", chunk=64)
    assert f32["path"] == 2 and f32["blocks"] == 2
    with pytest.raises(abi.TttError):
        abi.chunked_plan(1, 8, 1024, 96, 96, chunk=64)


def test_debug_build_exports_the_same_abi(abi):
    """The debug build (-DTTT_LA_DEBUG) exports every declared symbol and says
    it checks; the release build compiles the checks away (line query -1)."""
    from test_layers_causal_b200.build import DEBUG_OUT, build
    build(out=DEBUG_OUT, debug=True)
    D = abi.debug_lib()
    for n in declared_functions():
        assert hasattr(D, n), n
    assert b"debug checks" in D.ttt_la_version() and b"debug" not in abi.lib().ttt_la_version()
    assert abi.lib().ttt_la_debug_check_line(None) == -1
    assert D.ttt_la_status_string(abi.ERR_DEVICE_CHECK) == abi.lib().ttt_la_status_string(6)
    assert b"bounds check" in D.ttt_la_status_string(6)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from test_layers_causal_b200 import _abi
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _abi.lib()


def test_host_staging_size_and_checks(abi):
    """Two staging sets of up to 8 pieces: q, k, v, o (+ eta, states) per
    piece at 256-byte alignment, plus the piece's scratch; a missing, short or
    misaligned staging buffer is refused before anything is queued."""
    L = abi.lib()
    # 9 small sequences -> the minimum of 2 pieces, of 5 sequences; bf16 T=100 d=64:
    # 4 tensors of 5*100*64*2 = 64000 B (a multiple of 256) each, eta 5*100*4 = 2000 -> 2048
    a = _args(abi, B=3, H=3, T=100, eta=0x50000)
    per_set = 4 * 64000 + 2048
    ws = L.ttt_la_workspace_size(ctypes.byref(_args(abi, B=1, H=5, T=100)))
    assert L.ttt_la_host_staging_size(ctypes.byref(a)) == 2 * (per_set + (ws + 255) // 256 * 256)
    need = L.ttt_la_host_staging_size(ctypes.byref(a))
    assert L.ttt_la_forward_chunked_host(ctypes.byref(a), None, need, None) == abi.ERR_INVALID_ARG
    assert L.ttt_la_forward_chunked_host(ctypes.byref(a), ctypes.c_void_p(0x100000), need - 1, None) == \
        abi.ERR_INVALID_ARG
    assert L.ttt_la_forward_chunked_host(ctypes.byref(a), ctypes.c_void_p(0x100008), need, None) == \
        abi.ERR_INVALID_ARG
    unsupported = _args(abi, d_k=96, d_v=96)
    assert L.ttt_la_forward_chunked_host(ctypes.byref(unsupported), ctypes.c_void_p(0x100000), 1 << 30, None) == \
        abi.ERR_UNSUPPORTED


def test_binding_rejects_wrongly_shaped_buffers(abi):
    """Caller buffers the library would write past the end of are refused in
    the binding (checked here where no GPU is needed: host-buffer forward and
    decode step argument checks run before any CUDA requirement)."""
    import torch
    q = torch.zeros(1, 2, 8, 32)
    for kw in (dict(out=torch.zeros(1, 2, 8, 16)), dict(state_out=torch.zeros(1, 2, 32, 16)),
               dict(mom_out=torch.zeros(1, 2, 32, 32, dtype=torch.float64)), dict(eta=torch.zeros(1, 2, 7))):
        with pytest.raises(ValueError):
            abi.forward_chunked_host(q, q, q, **kw)
    x = torch.zeros(1, 2, 32)
    S = torch.zeros(1, 2, 32, 32)
    with pytest.raises(ValueError):
        abi.decode_step(x, x, x, S, mom=torch.zeros(1, 2, 32, 16))
    with pytest.raises(ValueError):
        abi.decode_step(x, x, x, S, out=torch.zeros(1, 2, 16))
    with pytest.raises(TypeError):
        abi.decode_step(x, x.bfloat16(), x, S)


def test_backward_chunked_workspace_and_validation(abi):
    L = abi.lib()
    call = lambda g: L.ttt_la_backward_chunked(ctypes.byref(g), None)  # noqa: E731
    size = lambda g: L.ttt_la_backward_chunked_workspace_size(ctypes.byref(g))  # noqa: E731
    # bf16: the reverse passes read the inputs in place and write dv, dk
    # themselves; the scratch holds the two transposed states (and whatever
    # the chunked forward's own plan needs)
    g = _grad_args(abi, T=100)
    g.state_in, g.grad_state = 0x8000000, 0x9000000
    states = 2 * 2 * 2 * 64 * 64 * 4
    q = torch.empty(2, 2, 100, 64, dtype=torch.bfloat16)  # shapes only: the size query reads no memory
    fwd = max(abi.workspace_bytes(q, q, chunk=64), abi.workspace_bytes(q, q, chunk=128))  # dq pass, reverse passes
    assert size(g) == states + (fwd + 255) // 256 * 256
    # fp32: plus four inputs reversed along T and the passes' fp32 outputs
    f = _grad_args(abi, T=100)
    f.dtype = abi.F32
    assert size(f) >= 6 * (2 * 2 * 100 * 64 * 4)
    assert L.ttt_la_backward_chunked_workspace_size(None) == 0
    assert L.ttt_la_backward_chunked(None, None) == abi.ERR_INVALID_ARG
    # momentum states without momentum, and momentum in fp32 (the recurrent form's)
    for field, val in [("mom_in", 0xA000000), ("grad_mom", 0xB000000)]:
        g = _grad_args(abi)
        setattr(g, field, val)
        g.workspace_bytes = 1 << 40
        assert call(g) == abi.ERR_UNSUPPORTED, field
    g = _grad_args(abi, beta=0.9)
    g.dtype = abi.F32
    g.workspace_bytes = 1 << 40
    assert call(g) == abi.ERR_UNSUPPORTED
    g = _grad_args(abi, dk=64, dv=128, beta=0.9)
    g.workspace_bytes = 1 << 40
    assert call(g) == abi.ERR_UNSUPPORTED
    # momentum scratch: the four transposed states, and dL/dW_0 when the caller does not take it
    g = _grad_args(abi, T=100, beta=0.9)
    base = size(g)
    g.state_in, g.mom_in, g.grad_state, g.grad_mom = 0x8000000, 0xA000000, 0x9000000, 0xB000000
    assert size(g) == base + 4 * 2 * 2 * 64 * 64 * 4
    g.grad_state_in = 0xC000000
    assert size(g) == base + 3 * 2 * 2 * 64 * 64 * 4
    g = _grad_args(abi, dk=64, dv=128)  # the bf16 tensor-core forward wants d_k == d_v
    g.workspace_bytes = 1 << 40
    assert call(g) == abi.ERR_UNSUPPORTED
    g = _grad_args(abi)
    g.state_in, g.grad_state = 0x8000000, 0x9000000
    g.workspace_bytes = size(g) - 256
    assert call(g) == abi.ERR_INVALID_ARG
