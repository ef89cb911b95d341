"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import linear_recurrent_sequence_scale_b200 as ret

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "retention.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"RET_API\s+[\w\s\*]*?\b(ret_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(ret.LIB_PATH):
        from linear_recurrent_sequence_scale_b200 import build
        build.build()
    return ret.load_library()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("ret_parallel", "ret_chunkwise", "ret_chunkwise_workspace", "ret_step",
              "ret_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(ret.LIB_PATH)
    for name in _declared():
        assert hasattr(raw, name), name
    assert set(_declared()) <= set(ret.SIGNATURES)


def test_status_strings(lib):
    assert lib.ret_status_string(0) == b"ok"
    assert lib.ret_status_string(-1) == b"invalid argument"
    assert lib.ret_status_string(-2) == b"unsupported configuration"
    assert lib.ret_status_string(-3) == b"CUDA runtime error"
    assert lib.ret_status_string(-4) == b"workspace too small"
    assert b"sm_100a" in lib.ret_version()


P = ctypes.c_void_p
A = P(0x10000)         # a 16-byte aligned fake address: never dereferenced,
M = P(0x10008)         # every call below is rejected before any launch


def test_parallel_rejects_bad_arguments(lib):
    f = lib.ret_parallel
    ok = dict(B=1, H=2, N=16, dk=64, dv=64, dt=1, eps=-1.0)

    def call(q=A, k=A, v=A, g=A, o=A, **kw):
        a = {**ok, **kw}
        return f(q, k, v, g, o, a["B"], a["H"], a["N"], a["dk"], a["dv"], a["dt"], a["eps"], None)

    assert call(q=None) == ret.RET_EINVAL
    assert call(g=None) == ret.RET_EINVAL
    assert call(o=M) == ret.RET_EINVAL            # misaligned
    assert call(B=0) == ret.RET_EINVAL
    assert call(dk=60) == ret.RET_EINVAL          # not a multiple of 8
    assert call(dv=0) == ret.RET_EINVAL
    assert call(dt=7) == ret.RET_EINVAL
    assert call(eps=float("nan")) == ret.RET_EINVAL
    assert call(dk=1024) == ret.RET_EUNSUPPORTED
    assert call(B=1000, H=1000) == ret.RET_EUNSUPPORTED
    # an empty sequence is valid and writes nothing
    assert call(N=0, q=None, k=None, v=None, o=None) == ret.RET_OK


def test_chunkwise_rejects_bad_arguments(lib):
    f = lib.ret_chunkwise
    need = lib.ret_chunkwise_workspace(1, 2, 300, 64, 64, 64, 0)
    assert need > 0
    assert lib.ret_chunkwise_workspace(1, 2, 300, 64, 64, 0, 0) == 0   # invalid chunk

    def call(q=A, k=A, v=A, g=A, chunk=64, si=None, so=None, o=A, N=300, dt=0, ws=A,
             wsb=None, eps=-1.0):
        wsb = need if wsb is None else wsb
        return f(q, k, v, g, chunk, si, so, o, 1, 2, N, 64, 64, dt, eps, ws, wsb, None)

    assert call(chunk=0) == ret.RET_EINVAL
    assert call(g=None) == ret.RET_EINVAL
    assert call(si=M) == ret.RET_EINVAL
    assert call(v=None) == ret.RET_EINVAL
    assert call(ws=None) == ret.RET_EWORKSPACE
    assert call(wsb=need - 1) == ret.RET_EWORKSPACE
    assert call(ws=M) == ret.RET_EINVAL
    assert call(N=-1) == ret.RET_EINVAL
    # no tokens, no state requested: nothing to do
    assert call(N=0, q=None, k=None, v=None, o=None, ws=None, wsb=0) == ret.RET_OK


def test_step_rejects_bad_arguments(lib):
    f = lib.ret_step

    def call(q=A, k=A, v=A, g=A, s=A, o=A, B=2, H=2, dk=64, dv=64, dt=1, eps=-1.0):
        return f(q, k, v, g, s, o, B, H, dk, dv, dt, eps, None)

    assert call(s=None) == ret.RET_EINVAL
    assert call(s=M) == ret.RET_EINVAL
    assert call(dk=12) == ret.RET_EINVAL
    assert call(dv=2048) == ret.RET_EUNSUPPORTED
    assert call(dt=-1) == ret.RET_EINVAL
    assert call(eps=float("nan")) == ret.RET_EINVAL


def test_chunkwise_phases_reject_bad_arguments(lib):
    need = lib.ret_chunkwise_workspace(1, 2, 300, 64, 64, 64, 0)

    def states(k=A, v=A, g=A, chunk=64, si=None, so=None, N=300, dt=0, ws=A, wsb=None):
        wsb = need if wsb is None else wsb
        return lib.ret_chunkwise_states(k, v, g, chunk, si, so, 1, 2, N, 64, 64, dt, ws, wsb,
                                        None)

    def output(q=A, k=A, v=A, g=A, chunk=64, hs=0, o=A, N=300, dt=0, eps=-1.0, ws=A, wsb=None):
        wsb = need if wsb is None else wsb
        return lib.ret_chunkwise_output(q, k, v, g, chunk, hs, o, 1, 2, N, 64, 64, dt, eps, ws,
                                        wsb, None)

    assert states(chunk=0) == ret.RET_EINVAL
    assert states(g=None) == ret.RET_EINVAL
    assert states(k=None) == ret.RET_EINVAL
    assert states(so=M) == ret.RET_EINVAL
    assert states(ws=None) == ret.RET_EWORKSPACE
    assert states(wsb=need - 1) == ret.RET_EWORKSPACE
    assert states(dt=3) == ret.RET_EINVAL
    assert output(q=None) == ret.RET_EINVAL
    assert output(o=M) == ret.RET_EINVAL
    assert output(eps=float("nan")) == ret.RET_EINVAL
    assert output(ws=None) == ret.RET_EWORKSPACE
    assert output(ws=M) == ret.RET_EINVAL
    # no tokens: the output phase writes nothing and the states phase has no
    # state to copy
    assert output(N=0, q=None, k=None, v=None, o=None, ws=None, wsb=0) == ret.RET_OK
    assert states(N=0, k=None, v=None, ws=None, wsb=0) == ret.RET_OK


def test_gated_entry_points_reject_bad_arguments(lib):
    """The gate is checked like the other operands (16-byte alignment); a
    NULL gate is the ungated call, so the ungated argument errors still show."""
    need = lib.ret_chunkwise_workspace(1, 2, 300, 64, 64, 64, 0)
    par = lambda g=A, o=A, N=16, eps=-1.0: lib.ret_parallel_gated(
        A, A, A, A, g, o, 1, 2, N, 64, 64, 1, eps, None)
    chk = lambda g=A, ws=A, N=300: lib.ret_chunkwise_gated(
        A, A, A, A, 64, None, None, g, A, 1, 2, N, 64, 64, 0, -1.0, ws, need, None)
    out = lambda g=A, eps=-1.0: lib.ret_chunkwise_output_gated(
        A, A, A, A, 64, 0, g, A, 1, 2, 300, 64, 64, 0, eps, A, need, None)
    stp = lambda g=A, s=A: lib.ret_step_gated(A, A, A, A, s, g, A, 2, 2, 64, 64, 1, -1.0, None)
    assert par(g=M) == ret.RET_EINVAL
    assert par(o=None) == ret.RET_EINVAL
    assert par(eps=float("nan")) == ret.RET_EINVAL
    assert par(N=0, g=None, o=None) == ret.RET_OK
    assert chk(g=M) == ret.RET_EINVAL
    assert chk(ws=None) == ret.RET_EWORKSPACE
    assert chk(N=0, g=None) == ret.RET_OK
    assert out(g=M) == ret.RET_EINVAL
    assert out(eps=float("nan")) == ret.RET_EINVAL
    assert stp(g=M) == ret.RET_EINVAL
    assert stp(s=None) == ret.RET_EINVAL


def test_state_combine_rejects_bad_arguments(lib):
    spans = (ctypes.c_int * 3)(5, 7, 9)
    bad = (ctypes.c_int * 3)(5, -1, 9)
    f = lambda loc=A, sp=spans, r=3, g=A, s0=None, out=A, dk=64: lib.ret_state_combine(
        loc, sp, r, g, s0, out, 1, 2, dk, 64, None)
    assert f(r=-1) == ret.RET_EINVAL
    assert f(loc=None) == ret.RET_EINVAL
    assert f(sp=None) == ret.RET_EINVAL
    assert f(sp=bad) == ret.RET_EINVAL
    assert f(out=None) == ret.RET_EINVAL
    assert f(out=M) == ret.RET_EINVAL
    assert f(s0=M) == ret.RET_EINVAL
    assert f(dk=12) == ret.RET_EINVAL
    assert f(r=65) == ret.RET_EUNSUPPORTED


def test_bf16_chunk_64_takes_the_tensor_core_layout(lib):
    """bf16 chunk 64 runs on the tensor-core kernels as 128-token chunks: its
    workspace is the 128-chunk one (2 bytes per state element, one state per
    128 tokens), while float32 chunk 64, and bf16 shapes the tensor cores do
    not tile, keep the CUDA-core layout."""
    for B, H, N, dk, dv in ((1, 2, 300, 64, 64), (2, 3, 1000, 256, 512), (1, 1, 128, 128, 256)):
        tc128 = lib.ret_chunkwise_workspace(B, H, N, dk, dv, 128, 1)
        assert tc128 == 2 * B * H * -(-N // 128) * dk * dv
        assert lib.ret_chunkwise_workspace(B, H, N, dk, dv, 64, 1) == tc128
        assert lib.ret_chunkwise_workspace(B, H, N, dk, dv, 64, 0) != tc128
    # d_k 32 is outside the tensor-core tiles: chunk 64 stays on the CUDA cores
    assert lib.ret_chunkwise_workspace(1, 2, 300, 32, 64, 64, 1) == \
        lib.ret_chunkwise_workspace(1, 2, 300, 32, 64, 64, 0)


def test_backward_rejects_bad_arguments(lib):
    need = lib.ret_chunkwise_backward_workspace(1, 2, 300, 64, 64, 64, 0)
    assert need > 0 and lib.ret_chunkwise_backward_workspace(1, 2, 300, 64, 64, 0, 0) == 0
    # CUDA-core backward (float32, and bf16 with chunks the tensor cores do not
    # tile): float32 forward and gradient states plus two [c][c] score blocks
    # per chunk of c = min(chunk, 128) tokens
    for dt, chunk, c in ((0, 64, 64), (0, 37, 37), (0, 512, 128), (1, 37, 37), (1, 100, 100)):
        nc = -(-300 // c)
        assert lib.ret_chunkwise_backward_workspace(1, 2, 300, 64, 96, chunk, dt) == \
            2 * 4 * 2 * nc * (64 * 96 + c * c)
    # bf16 with a tensor-core chunk: reversed copies of q, k, v and dO, four
    # float32 states, then the workspace of the forward calls (the larger of
    # the two mapped shapes), each region rounded up to 256 bytes
    al = lambda x: -(-x // 256) * 256
    for chunk in (64, 128, 512):
        fws = max(lib.ret_chunkwise_workspace(1, 2, 300, 96, 64, chunk, 1),
                  lib.ret_chunkwise_workspace(1, 2, 300, 64, 96, chunk, 1))
        want = (2 * al(2 * 300 * 64 * 2) + 2 * al(2 * 300 * 96 * 2) + 4 * al(2 * 64 * 96 * 4)
                + al(fws))
        assert lib.ret_chunkwise_backward_workspace(1, 2, 300, 64, 96, chunk, 1) == want

    def call(q=A, dO=A, gq=A, ds=A, si=None, dso=None, ws=A, wsb=None, N=300, chunk=64, dt=0):
        wsb = need if wsb is None else wsb
        return lib.ret_chunkwise_backward(q, A, A, A, chunk, si, dO, dso, gq, A, A, ds,
                                          1, 2, N, 64, 64, dt, ws, wsb, None)

    assert call(q=None) == ret.RET_EINVAL
    assert call(dO=None) == ret.RET_EINVAL
    assert call(gq=M) == ret.RET_EINVAL
    assert call(si=M) == ret.RET_EINVAL
    assert call(ds=M) == ret.RET_EINVAL
    assert call(chunk=0) == ret.RET_EINVAL
    assert call(dt=5) == ret.RET_EINVAL
    assert call(ws=None) == ret.RET_EWORKSPACE
    assert call(wsb=need - 1) == ret.RET_EWORKSPACE
    assert call(N=0, q=None, dO=None, gq=None, ds=None, ws=None, wsb=0) == ret.RET_OK
    # bf16 on the tensor cores: a sequence past the forward kernels' chunk-count
    # limit is refused before the row reversals launch (a failing status means
    # nothing ran; this process has no GPU, so a launch would fail otherwise)
    n_big = 128 * 65535 + 1
    big = lib.ret_chunkwise_backward_workspace(1, 2, n_big, 64, 64, 128, 1)
    assert big > 0
    assert call(N=n_big, chunk=128, dt=1, wsb=big) == ret.RET_EUNSUPPORTED


def test_selftest_rejects_bad_limits(lib):
    assert lib.ret_selftest_bounded_wait(0, None) == ret.RET_EINVAL
    assert lib.ret_selftest_bounded_wait(20000, None) == ret.RET_EINVAL


def test_rotate_rejects_bad_arguments(lib):
    def call(x=A, y=A, th=A, pos0=0, B=1, H=2, N=300, d=64, dt=0):
        return lib.ret_rotate(x, y, th, pos0, B, H, N, d, dt, None)

    assert call(x=None) == ret.RET_EINVAL
    assert call(y=None) == ret.RET_EINVAL
    assert call(th=None) == ret.RET_EINVAL
    assert call(x=M) == ret.RET_EINVAL
    assert call(y=M) == ret.RET_EINVAL
    assert call(d=63) == ret.RET_EINVAL
    assert call(d=0) == ret.RET_EINVAL
    assert call(N=-1) == ret.RET_EINVAL
    assert call(B=0) == ret.RET_EINVAL
    assert call(dt=5) == ret.RET_EINVAL
    assert call(pos0=-1) == ret.RET_EINVAL
    assert call(pos0=(1 << 53) - 299) == ret.RET_EINVAL
    assert call(y=P(0x10000 + 64)) == ret.RET_EINVAL  # overlaps x without equalling it
    assert call(N=0) == ret.RET_OK                   # nothing to launch
    assert call(N=0, x=None, y=None, th=None) == ret.RET_OK
