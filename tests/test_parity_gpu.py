"""CUDA path against the CPU oracle, element by element on the same inputs.

Tolerances (rel-Frobenius): 1e-5 for float32 inputs, 2e-2 for bf16 inputs
with float32 accumulation, 1e-4 for every float32 state returned.  Each holds
for the whole output and also for every (batch, head) slice and every
128-row tile of it, so that an error confined to one tile, ring slot or chunk
boundary is not diluted by the rest of the output.  bf16 inputs are rounded once by the input generator and the oracle
consumes exactly those rounded values in float64.
"""
import numpy as np
import pytest

import oracle
from linear_recurrent_sequence_scale_b200 import workloads as wl
from parity_check import worst_rel

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}
STATE_TOL = 1e-4


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.fixture(scope="module")
def ret(torch_cuda):
    import linear_recurrent_sequence_scale_b200 as ret
    ret.load_library()
    return ret


@pytest.fixture(autouse=True)
def no_device_error(ret):
    """Every test must end without a timed-out wait inside a kernel."""
    yield
    assert ret.device_error() == 0


def _dev(t):
    return wl.to_torch(t, "cuda")


def _gam(torch, g):
    return torch.from_numpy(np.asarray(g, dtype=np.float32)).cuda()


def _rel(x, ref):
    """The worst rel-Frobenius error over the whole output, each (batch, head)
    and each 128-row tile (see parity_check)."""
    return worst_rel(wl.from_torch(x) if not isinstance(x, np.ndarray) else x, ref)


def _ref_chunkwise(inp, chunk, gn, with_state_in):
    s0 = inp["state"].exact if with_state_in else None
    o, s = oracle.chunkwise(inp["q"].exact, inp["k"].exact, inp["v"].exact, inp["gammas"],
                            chunk, s0)
    if gn is not None:
        o = oracle.group_norm(o, gn)
    return o, s


# --- the tiny float32 workload: all three forms ---------------------------------

def test_tiny_f32_all_three_forms(torch_cuda, ret):
    torch = torch_cuda
    w = wl.WORKLOADS["tiny_f32"]
    inp = wl.make_inputs(w.B, w.H, w.N, w.dk, w.dv, "f32", seed=w.seed)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    o_ref, s_ref = oracle.recurrent(inp["q"].exact, inp["k"].exact, inp["v"].exact, inp["gammas"])

    o_par = ret.parallel(q, k, v, g)
    o_chk, s_chk = ret.chunkwise(q, k, v, g, w.chunk, return_state=True)
    state = torch.zeros((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    o_rec = torch.empty_like(v)
    for n in range(w.N):
        o_rec[:, :, n] = ret.step(q[:, :, n].contiguous(), k[:, :, n].contiguous(),
                                  v[:, :, n].contiguous(), g, state)
    torch.cuda.synchronize()
    assert _rel(o_par, o_ref) <= TOL["f32"]
    assert _rel(o_chk, o_ref) <= TOL["f32"]
    assert _rel(o_rec, o_ref) <= TOL["f32"]
    assert _rel(s_chk, s_ref) <= STATE_TOL
    assert _rel(state, s_ref) <= STATE_TOL


# --- chunkwise: several tiles, ragged tails, GroupNorm, carried state ------------

CHUNK_CASES = [
    # dtype, B, H, N, dk, dv, chunk, gn_eps, state_in
    ("bf16", 1, 3, 1000, 256, 512, 512, 1e-5, True),
    ("bf16", 2, 2, 700, 256, 256, 128, None, False),
    ("bf16", 1, 4, 333, 64, 64, 128, None, True),
    ("bf16", 2, 2, 640, 128, 128, 256, 1e-5, False),
    ("bf16", 1, 2, 1100, 128, 512, 256, None, True),
    ("bf16", 2, 3, 600, 64, 256, 128, None, True),     # d_k 64: state boxes past d_k skipped
    ("bf16", 1, 3, 300, 256, 512, 64, 1e-5, True),     # chunk 64: tensor cores, 128-token tiles
    ("bf16", 2, 2, 333, 128, 128, 64, None, False),
    ("bf16", 10, 4, 600, 256, 512, 256, 1e-5, False),  # 160 column tiles: both d_k halves per CTA
    ("f32", 1, 3, 301, 128, 64, 37, None, True),
    ("f32", 2, 2, 200, 64, 96, 64, 1e-5, False),
    ("f32", 1, 2, 130, 32, 40, 1, None, True),
]


@pytest.mark.parametrize("case", CHUNK_CASES, ids=lambda c: "-".join(map(str, c)))
def test_chunkwise_parity(torch_cuda, ret, case):
    torch = torch_cuda
    dt, B, H, N, dk, dv, chunk, gn, with_s0 = case
    inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=100 + N, with_state=with_s0)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    s0 = _dev(inp["state"]) if with_s0 else None
    o, s = ret.chunkwise(q, k, v, g, chunk, state_in=s0, return_state=True, gn_eps=gn)
    torch.cuda.synchronize()
    o_ref, s_ref = _ref_chunkwise(inp, chunk, gn, with_s0)
    assert _rel(o, o_ref) <= TOL[dt]
    assert _rel(s, s_ref) <= STATE_TOL


def _random_chunk_cases(n, seed):
    """Seeded random tensor-core shapes: ragged lengths, every supported
    d_k, d_v and chunk, GroupNorm, incoming and returned states mixed."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        dk = int(rng.choice([64, 128, 256]))
        dv = int(rng.choice([64, 128, 256, 512]))
        chunk = int(rng.choice([64, 128, 256, 512]))
        N = int(rng.integers(1, 1600))
        B, H = int(rng.integers(1, 3)), int(rng.integers(1, 4))
        gn = 1e-5 if rng.random() < 0.5 else None
        out.append((B, H, N, dk, dv, chunk, gn, bool(rng.random() < 0.5), bool(rng.random() < 0.5)))
    return out


@pytest.mark.parametrize("case", _random_chunk_cases(16, 2024), ids=lambda c: "-".join(map(str, c)))
def test_chunkwise_random_tensor_core_shapes(torch_cuda, ret, case):
    torch = torch_cuda
    B, H, N, dk, dv, chunk, gn, with_s0, want_s = case
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=300 + N, with_state=with_s0)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    s0 = _dev(inp["state"]) if with_s0 else None
    if want_s:
        o, s = ret.chunkwise(q, k, v, g, chunk, state_in=s0, return_state=True, gn_eps=gn)
    else:
        o, s = ret.chunkwise(q, k, v, g, chunk, state_in=s0, gn_eps=gn), None
    torch.cuda.synchronize()
    o_ref, s_ref = _ref_chunkwise(inp, chunk, gn, with_s0)
    assert _rel(o, o_ref) <= TOL["bf16"]
    if want_s:
        assert _rel(s, s_ref) <= STATE_TOL


@pytest.mark.parametrize("case", [c for c in CHUNK_CASES if c[0] == "bf16"],
                         ids=lambda c: "-".join(map(str, c)))
def test_chunkwise_parity_without_final_state(torch_cuda, ret, case):
    """The same calls without the final state: the state scan then runs its
    other variant (no hi/lo split, a deeper ring), whose bf16 chunk states
    the output kernel reads."""
    torch = torch_cuda
    dt, B, H, N, dk, dv, chunk, gn, with_s0 = case
    inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=200 + N, with_state=with_s0)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    s0 = _dev(inp["state"]) if with_s0 else None
    o = ret.chunkwise(q, k, v, g, chunk, state_in=s0, gn_eps=gn)
    torch.cuda.synchronize()
    o_ref, _ = _ref_chunkwise(inp, chunk, gn, with_s0)
    assert _rel(o, o_ref) <= TOL[dt]


# bf16 shapes outside the tensor-core tiling (chunk not in {64, 128, 256, 512}, or
# d_k / d_v not a power of two in [64, 256] / [64, 512]) run the float32
# CUDA-core kernels on the bf16 inputs; their only rounding is the bf16
# output, so they are held to a tolerance well inside the bf16 one.
OFF_TC_CASES = [
    # B, H, N, dk, dv, chunk, gn_eps, state_in
    (1, 3, 300, 256, 512, 32, 1e-5, True),    # chunk 32
    (2, 2, 333, 128, 128, 100, None, False),  # chunk not a power of two
    (1, 2, 200, 32, 64, 128, None, True),     # d_k below the tensor-core tiles
    (1, 2, 150, 512, 128, 128, None, False),  # d_k above them
]


@pytest.mark.parametrize("case", OFF_TC_CASES, ids=lambda c: "-".join(map(str, c)))
def test_bf16_outside_tensor_core_tiling_runs_float32_path(torch_cuda, ret, case):
    torch = torch_cuda
    B, H, N, dk, dv, chunk, gn, with_s0 = case
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=1200 + N, with_state=with_s0)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    s0 = _dev(inp["state"]) if with_s0 else None
    o, s = ret.chunkwise(q, k, v, g, chunk, state_in=s0, return_state=True, gn_eps=gn)
    torch.cuda.synchronize()
    o_ref, s_ref = _ref_chunkwise(inp, chunk, gn, with_s0)
    assert _rel(o, o_ref) <= 5e-3            # the bf16 rounding of o alone
    assert _rel(s, s_ref) <= STATE_TOL


def test_chunkwise_without_state_out_and_in_place(torch_cuda, ret):
    torch = torch_cuda
    B, H, N, dk, dv, C = 1, 2, 520, 128, 128, 128
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=7, with_state=True)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    o_ref, s_ref = _ref_chunkwise(inp, C, None, True)
    o1 = ret.chunkwise(q, k, v, g, C, state_in=_dev(inp["state"]))
    s = _dev(inp["state"])
    o2, s2 = ret.chunkwise(q, k, v, g, C, state_in=s, state_out=s)   # in place
    torch.cuda.synchronize()
    assert s2.data_ptr() == s.data_ptr()
    assert _rel(o1, o_ref) <= TOL["bf16"]
    assert _rel(o2, o_ref) <= TOL["bf16"]
    assert _rel(s, s_ref) <= STATE_TOL


@pytest.mark.parametrize("N", [1, 200, 512])
def test_single_chunk_state_out_read_right_after_the_call(torch_cuda, ret, N):
    """One chunk and no incoming state: no output tile reads a chunk state,
    so nothing inside the output kernel waits for the state scan.  The call
    must still complete only after the scan: the final state is consumed by
    the next operation on the same stream, with no synchronisation between."""
    torch = torch_cuda
    B, H, dk, dv, C = 2, 3, 256, 512, 512
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=900 + N)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    o_ref, s_ref = _ref_chunkwise(inp, C, 1e-5, False)
    for _ in range(3):
        s = torch.full((B, H, dk, dv), float("nan"), dtype=torch.float32, device="cuda")
        o, _ = ret.chunkwise(q, k, v, g, C, state_out=s, gn_eps=1e-5)
        s_next = s * 1.0   # the next stream operation reads the state at once
        torch.cuda.synchronize()
        assert _rel(o, o_ref) <= TOL["bf16"]
        assert _rel(s_next, s_ref) <= STATE_TOL


@pytest.mark.parametrize("dt,chunk,gn", [("bf16", 256, 1e-5), ("f32", 100, None)])
def test_chunkwise_in_two_phases(torch_cuda, ret, dt, chunk, gn):
    """ret_chunkwise_states then ret_chunkwise_output: the oracle's result, and
    bit for bit what the one-call form returns."""
    torch = torch_cuda
    B, H, N, dk, dv = 1, 2, 900, 128, 256
    inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=31, with_state=True)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    s0 = _dev(inp["state"])
    ws = torch.empty(ret.chunkwise_workspace_bytes(B, H, N, dk, dv, chunk, q.dtype),
                     dtype=torch.uint8, device="cuda")
    s = torch.empty_like(s0)
    ret.chunkwise_states(k, v, g, chunk, ws, state_in=s0, state_out=s)
    o = ret.chunkwise_output(q, k, v, g, chunk, ws, has_state_in=True, gn_eps=gn)
    o1, s1 = ret.chunkwise(q, k, v, g, chunk, state_in=s0, return_state=True, gn_eps=gn)
    torch.cuda.synchronize()
    o_ref, s_ref = _ref_chunkwise(inp, chunk, gn, True)
    assert _rel(o, o_ref) <= TOL[dt]
    assert _rel(s, s_ref) <= STATE_TOL
    assert torch.equal(o, o1) and torch.equal(s, s1)


@pytest.mark.parametrize("gn", [None, 1e-5])
def test_chunkwise_strong_and_weak_decays(torch_cuda, ret, gn):
    """Weak and strong decays with a state entering: gamma^256 runs from
    0.77 (0.999) down to 0.5^256 (below float32's range, so xi and the mask
    flush to zero) and 0 (where 0^0 = 1 keeps the diagonal).  The kernel
    scales each Q row by xi in place for every decay; all must match the
    oracle."""
    torch = torch_cuda
    B, H, N, dk, dv, C = 1, 4, 700, 128, 256, 256
    gam = [0.5, 0.9, 0.999, 0.0]
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=43, with_state=True, gammas=gam)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    o, s = ret.chunkwise(q, k, v, g, C, state_in=_dev(inp["state"]), return_state=True, gn_eps=gn)
    torch.cuda.synchronize()
    o_ref, s_ref = _ref_chunkwise(inp, C, gn, True)
    assert _rel(o, o_ref) <= TOL["bf16"]
    assert _rel(s, s_ref) <= STATE_TOL


def _offset_v(inp, dv, offset):
    """v with every fourth 32-column group spread 30x and a common offset:
    the retention output rows then carry a mean far from zero."""
    col = np.where((np.arange(dv) // 32) % 4 == 0, 30.0, 1.0)
    return wl.from_values(inp["v"].exact * col + offset, "bf16")


def test_groupnorm_far_from_zero_mean(torch_cuda, ret):
    """GroupNorm where every output row carries a large common offset (row
    means about 20x the spread) and the 32-column groups differ in spread by
    30x: the normalised deviations must still come out to bf16 accuracy in
    every tile (parallel form, one 256-column slice)."""
    torch = torch_cuda
    B, H, N, dk, dv = 1, 2, 600, 128, 256
    inp = wl.make_inputs(B, H, N, dk, 512, "bf16", seed=41)
    v = _offset_v(inp, 512, 40.0)
    q, k, vd = _dev(inp["q"]), _dev(inp["k"]), _dev(v)
    g = _gam(torch, inp["gammas"])
    vs = vd[..., :dv].contiguous()
    op = ret.parallel(q, k, vs, g, gn_eps=1e-5)
    p_ref, _ = oracle.parallel(inp["q"].exact, inp["k"].exact, v.exact[..., :dv], inp["gammas"])
    p_ref = oracle.group_norm(p_ref, 1e-5)
    torch.cuda.synchronize()
    assert _rel(op, p_ref) <= TOL["bf16"]


@pytest.mark.parametrize("offset", [8.0, 40.0])
def test_chunkwise_groupnorm_far_from_zero_mean(torch_cuda, ret, offset):
    """The same stress for the chunkwise form (two d_v slices, three chunks).
    Its cross-chunk term reads the chunk state as bf16, and that rounding
    (relative 2^-9 of every state element) is not removed by the GroupNorm's
    mean subtraction: after normalisation its error grows with the ratio of
    the row means to the row spread, about 1.4e-3 per unit of that ratio
    (float64 emulation of the rounding).  At offset 8 (ratio 4) every tile
    meets the bf16 tolerance; at offset 40 (ratio 20) the whole output does,
    and every tile stays within the bound that ratio gives (5e-2)."""
    torch = torch_cuda
    B, H, N, dk, dv, C = 1, 2, 600, 128, 512, 256
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=41)
    v = _offset_v(inp, dv, offset)
    q, k, vd = _dev(inp["q"]), _dev(inp["k"]), _dev(v)
    g = _gam(torch, inp["gammas"])
    o = ret.chunkwise(q, k, vd, g, C, gn_eps=1e-5)
    o_ref, _ = oracle.chunkwise(inp["q"].exact, inp["k"].exact, v.exact, inp["gammas"], C)
    o_ref = oracle.group_norm(o_ref, 1e-5)
    torch.cuda.synchronize()
    if offset <= 8.0:
        assert _rel(o, o_ref) <= TOL["bf16"]
    else:
        assert oracle.rel_frobenius(wl.from_torch(o), o_ref) <= TOL["bf16"]
        assert _rel(o, o_ref) <= 5e-2


# --- gated output: swish(G) (.) Y -----------------------------------------------

GATED_CASES = [
    # form, dtype, B, H, N, dk, dv, chunk, gn_eps
    ("chunkwise", "bf16", 1, 2, 1000, 256, 512, 512, 1e-5),   # tensor cores, 2 d_v slices
    ("chunkwise", "bf16", 2, 2, 333, 128, 128, 128, None),    # tensor cores, ragged tail
    ("chunkwise", "bf16", 1, 2, 300, 64, 64, 128, 1e-5),      # one 64-column box per slice
    ("parallel", "bf16", 1, 3, 300, 64, 256, None, 1e-5),
    ("chunkwise", "f32", 1, 2, 200, 64, 96, 64, 1e-5),        # SIMT path
    ("parallel", "f32", 1, 2, 130, 32, 40, None, None),
]


@pytest.mark.parametrize("case", GATED_CASES, ids=lambda c: "-".join(map(str, c)))
def test_gated_output_parity(torch_cuda, ret, case):
    torch = torch_cuda
    form, dt, B, H, N, dk, dv, chunk, gn = case
    inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=51 + N, with_state=True)
    rng = np.random.default_rng(52 + N)
    gate = wl.from_values(rng.standard_normal((B, H, N, dv)) * 2.0, dt)
    q, k, v, gd = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(gate)
    g = _gam(torch, inp["gammas"])
    if form == "chunkwise":
        o, s = ret.chunkwise(q, k, v, g, chunk, state_in=_dev(inp["state"]), return_state=True,
                             gn_eps=gn, gate=gd)
        y_ref, s_ref = _ref_chunkwise(inp, chunk, gn, True)
    else:
        o = ret.parallel(q, k, v, g, gn_eps=gn, gate=gd)
        y_ref, _ = oracle.parallel(inp["q"].exact, inp["k"].exact, inp["v"].exact, inp["gammas"])
        if gn is not None:
            y_ref = oracle.group_norm(y_ref, gn)
    torch.cuda.synchronize()
    assert _rel(o, oracle.gated(y_ref, gate.exact)) <= TOL[dt]
    if form == "chunkwise":
        assert _rel(s, s_ref) <= STATE_TOL


@pytest.mark.parametrize("gn", [None, 1e-5])
def test_gated_step_parity(torch_cuda, ret, gn):
    torch = torch_cuda
    B, H, dk, dv = 2, 3, 64, 256
    inp = wl.make_inputs(B, H, 1, dk, dv, "bf16", seed=61, with_state=True)
    gate = wl.from_values(np.random.default_rng(62).standard_normal((B, H, dv)), "bf16")
    state = _dev(inp["state"])
    o = ret.step(_dev(inp["q"])[:, :, 0].contiguous(), _dev(inp["k"])[:, :, 0].contiguous(),
                 _dev(inp["v"])[:, :, 0].contiguous(), _gam(torch, inp["gammas"]), state,
                 gn_eps=gn, gate=_dev(gate))
    torch.cuda.synchronize()
    y_ref, s_ref = oracle.step(inp["q"].exact[:, :, 0], inp["k"].exact[:, :, 0],
                               inp["v"].exact[:, :, 0], inp["gammas"], inp["state"].exact)
    if gn is not None:
        y_ref = oracle.group_norm(y_ref, gn)
    assert _rel(o, oracle.gated(y_ref, gate.exact)) <= TOL["bf16"]
    assert _rel(state, s_ref) <= STATE_TOL


def test_gated_output_phase(torch_cuda, ret):
    """The gate through the two-phase form (ret_chunkwise_output_gated)."""
    torch = torch_cuda
    B, H, N, dk, dv, C = 1, 2, 600, 128, 256, 256
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=73, with_state=True)
    gate = wl.from_values(np.random.default_rng(74).standard_normal((B, H, N, dv)), "bf16")
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    ws = torch.empty(ret.chunkwise_workspace_bytes(B, H, N, dk, dv, C, q.dtype),
                     dtype=torch.uint8, device="cuda")
    ret.chunkwise_states(k, v, g, C, ws, state_in=_dev(inp["state"]))
    o = ret.chunkwise_output(q, k, v, g, C, ws, has_state_in=True, gn_eps=1e-5, gate=_dev(gate))
    torch.cuda.synchronize()
    y_ref, _ = _ref_chunkwise(inp, C, 1e-5, True)
    assert _rel(o, oracle.gated(y_ref, gate.exact)) <= TOL["bf16"]


def test_gated_tensor_cores_across_the_gate_range(torch_cuda, ret):
    """The tensor-core epilogue takes sigmoid through the hardware tanh; gates
    spread over [-12, 12] (saturated tails on both sides, where 1 + tanh
    cancels) stay within the bf16 tolerance per 128-row tile, and the
    elementwise error of the gate factor stays below 2^-8 of |g| + 1."""
    torch = torch_cuda
    B, H, N, dk, dv, C = 1, 2, 1024, 256, 512, 512
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=75)
    gate = wl.from_values(np.random.default_rng(76).uniform(-12.0, 12.0, (B, H, N, dv)), "bf16")
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    o0 = ret.chunkwise(q, k, v, g, C, gn_eps=1e-5)
    o1 = ret.chunkwise(q, k, v, g, C, gn_eps=1e-5, gate=_dev(gate))
    torch.cuda.synchronize()
    y_ref, _ = _ref_chunkwise(inp, C, 1e-5, False)
    assert _rel(o1, oracle.gated(y_ref, gate.exact)) <= TOL["bf16"]
    # the gate factor itself, against the ungated output of the same kernel
    y = wl.from_torch(o0).astype(np.float64)
    want = oracle.gated(y, gate.exact)
    got = wl.from_torch(o1).astype(np.float64)
    err = np.abs(got - want) - 2.0 ** -8 * np.abs(want)   # beyond the bf16 rounding
    assert np.max(err / (np.abs(y) * (np.abs(gate.exact) + 1.0) + 1e-30)) <= 2.0 ** -8


def test_gate_none_is_the_ungated_call(torch_cuda, ret):
    """gate=None runs the ungated entry point; a gate of +40 (swish(40) = 40
    in bf16 arithmetic) scales the ungated result by 40."""
    torch = torch_cuda
    B, H, N, dk, dv, C = 1, 2, 300, 128, 256, 128
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=71)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    o0 = ret.chunkwise(q, k, v, g, C, gn_eps=1e-5)
    o1 = ret.chunkwise(q, k, v, g, C, gn_eps=1e-5,
                       gate=torch.full_like(o0, 40.0))
    torch.cuda.synchronize()
    assert _rel(o1, 40.0 * wl.from_torch(o0)) <= 1e-2


# --- sequence parallelism: spans of one sequence, emulated on one GPU -------------

def test_state_combine_matches_the_span_recurrence(torch_cuda, ret):
    torch = torch_cuda
    rng = np.random.default_rng(91)
    R, B, H, dk, dv = 4, 2, 3, 64, 128
    loc = rng.standard_normal((R, B, H, dk, dv)).astype(np.float32)
    s0 = rng.standard_normal((B, H, dk, dv)).astype(np.float32)
    gam = np.array([0.9, 0.999, 0.5], dtype=np.float32)
    spans = [100, 0, 37, 512]
    for r in range(R + 1):
        ref = s0.astype(np.float64)
        for i in range(r):
            ref = gam.astype(np.float64)[None, :, None, None] ** spans[i] * ref + loc[i]
        got = ret.state_combine(torch.from_numpy(loc).cuda(), spans, r,
                                torch.from_numpy(gam).cuda(), torch.from_numpy(s0).cuda())
        torch.cuda.synchronize()
        assert _rel(got, ref) <= 1e-6


def test_sequence_parallel_spans_on_one_gpu(torch_cuda, ret):
    """Three ranks' spans run one after another on this GPU with the real
    kernels (the all-gather replaced by stacking): each span's output and the
    sequence's end state against the oracle over the unsplit sequence."""
    from linear_recurrent_sequence_scale_b200 import seqpar
    torch = torch_cuda
    B, H, N, dk, dv, C = 1, 2, 1500, 128, 256, 256
    spans = [700, 300, 500]
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=92, with_state=True)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    s0 = _dev(inp["state"])
    cut = np.cumsum([0] + spans)
    part = lambda x, r: x[:, :, cut[r]:cut[r + 1]].contiguous()
    locs = torch.stack([seqpar.local_end_state(part(q, r), part(k, r), part(v, r), g, C)
                        for r in range(3)])
    outs = []
    for r in range(3):
        o, s = seqpar.span_output(part(q, r), part(k, r), part(v, r), g, C, locs, spans, r,
                                  state0=s0, gn_eps=1e-5, return_state=True)
        outs.append(o)
    torch.cuda.synchronize()
    o_ref, s_ref = _ref_chunkwise(inp, C, 1e-5, True)
    assert _rel(torch.cat(outs, dim=2), o_ref) <= TOL["bf16"]
    assert _rel(s, s_ref) <= STATE_TOL


# --- backward ----------------------------------------------------------------------

BWD_CASES = [
    # dtype, B, H, N, dk, dv, chunk, state_in, d_state_out
    ("f32", 1, 2, 200, 64, 96, 64, True, True),
    ("f32", 2, 1, 130, 32, 40, 37, False, True),
    ("f32", 1, 3, 257, 128, 128, 128, True, False),
    ("bf16", 1, 2, 700, 128, 256, 256, True, True),
    ("bf16", 1, 2, 333, 256, 512, 512, False, False),
    ("bf16", 1, 2, 300, 128, 256, 64, True, True),     # chunk 64: forward calls on 128-token tiles
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "-".join(map(str, c)))
def test_chunkwise_backward_parity(torch_cuda, ret, case):
    torch = torch_cuda
    dt, B, H, N, dk, dv, chunk, with_s0, with_ds = case
    inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=101 + N, with_state=True)
    rng = np.random.default_rng(102 + N)
    d_o = wl.from_values(rng.standard_normal((B, H, N, dv)) * 0.1, dt)
    d_s = rng.standard_normal((B, H, dk, dv)).astype(np.float32) if with_ds else None
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    s0 = _dev(inp["state"]) if with_s0 else None
    gq, gk, gv, gs = ret.chunkwise_backward(
        q, k, v, g, chunk, _dev(d_o), state_in=s0,
        d_state_out=torch.from_numpy(d_s).cuda() if with_ds else None)
    torch.cuda.synchronize()
    rq, rk, rv, rs = oracle.backward(inp["q"].exact, inp["k"].exact, inp["v"].exact,
                                     inp["gammas"], d_o.exact,
                                     inp["state"].exact if with_s0 else None, d_s)
    tol = TOL[dt]
    assert _rel(gq, rq) <= tol
    assert _rel(gk, rk) <= tol
    assert _rel(gv, rv) <= tol
    assert _rel(gs, rs) <= (1e-5 if dt == "f32" else 1e-4)


def test_chunkwise_backward_bf16_special_decays(torch_cuda, ret):
    """The bf16 backward runs as three forward calls; the final-state gradient
    enters two of them divided by gamma, and for gamma = 0 a separate pass
    adds it at the last token.  Decays 0, 0.5, 0.9 and 1, with incoming and
    final-state gradients, on a chunk the tensor cores tile."""
    torch = torch_cuda
    B, H, N, dk, dv, chunk = 1, 4, 300, 128, 128, 128
    gam = [0.0, 0.5, 0.9, 1.0]
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=211, with_state=True, gammas=gam)
    rng = np.random.default_rng(212)
    d_o = wl.from_values(rng.standard_normal((B, H, N, dv)) * 0.1, "bf16")
    d_s = rng.standard_normal((B, H, dk, dv)).astype(np.float32)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    gq, gk, gv, gs = ret.chunkwise_backward(q, k, v, g, chunk, _dev(d_o),
                                            state_in=_dev(inp["state"]),
                                            d_state_out=torch.from_numpy(d_s).cuda())
    torch.cuda.synchronize()
    rq, rk, rv, rs = oracle.backward(inp["q"].exact, inp["k"].exact, inp["v"].exact,
                                     inp["gammas"], d_o.exact, inp["state"].exact, d_s)
    assert _rel(gq, rq) <= TOL["bf16"]
    assert _rel(gk, rk) <= TOL["bf16"]
    assert _rel(gv, rv) <= TOL["bf16"]
    assert _rel(gs, rs) <= 1e-4


# --- the largest supported sizes and many (batch, head) pairs -------------------

EDGE_CASES = [
    # form, dtype, B, H, N, dk, dv, chunk, gn_eps
    ("chunkwise", "bf16", 1, 1, 300, 512, 512, 100, 1e-5),   # d = 512: CUDA-core path
    ("chunkwise", "f32", 1, 1, 150, 512, 64, 64, None),
    ("parallel", "f32", 1, 1, 96, 512, 512, None, 1e-5),
    ("chunkwise", "bf16", 64, 32, 17, 64, 64, 128, 1e-5),    # 2048 pairs, one short chunk
    ("parallel", "bf16", 64, 32, 9, 128, 128, None, None),
]


@pytest.mark.parametrize("case", EDGE_CASES, ids=lambda c: "-".join(map(str, c)))
def test_edge_sizes(torch_cuda, ret, case):
    torch = torch_cuda
    form, dt, B, H, N, dk, dv, chunk, gn = case
    gam = [1.0 - 2.0 ** (-5 - (h % 12)) for h in range(H)]
    inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=111 + N + dk, with_state=(form == "chunkwise"),
                         gammas=gam)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    if form == "chunkwise":
        o, s = ret.chunkwise(q, k, v, g, chunk, state_in=_dev(inp["state"]), return_state=True,
                             gn_eps=gn)
        torch.cuda.synchronize()
        o_ref, s_ref = _ref_chunkwise(inp, chunk, gn, True)
        assert _rel(s, s_ref) <= STATE_TOL
    else:
        o = ret.parallel(q, k, v, g, gn_eps=gn)
        torch.cuda.synchronize()
        o_ref, _ = oracle.parallel(inp["q"].exact, inp["k"].exact, inp["v"].exact, inp["gammas"])
        if gn is not None:
            o_ref = oracle.group_norm(o_ref, gn)
    assert _rel(o, o_ref) <= TOL[dt]


@pytest.mark.parametrize("dk,dv", [(4096, 64), (256, 1024)])
def test_step_largest_sizes(torch_cuda, ret, dk, dv):
    """The decode step at its limits: d_k 4096, and d_v 1024 with GroupNorm
    over a cluster of 8 CTAs."""
    torch = torch_cuda
    B, H = 2, 2
    inp = wl.make_inputs(B, H, 1, dk, dv, "bf16", seed=121 + dk, with_state=True)
    state = _dev(inp["state"])
    o = ret.step(_dev(inp["q"])[:, :, 0].contiguous(), _dev(inp["k"])[:, :, 0].contiguous(),
                 _dev(inp["v"])[:, :, 0].contiguous(), _gam(torch, inp["gammas"]), state,
                 gn_eps=1e-5)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.step(inp["q"].exact[:, :, 0], inp["k"].exact[:, :, 0],
                               inp["v"].exact[:, :, 0], inp["gammas"], inp["state"].exact)
    assert _rel(o, oracle.group_norm(o_ref, 1e-5)) <= TOL["bf16"]
    assert _rel(state, s_ref) <= STATE_TOL


# --- parallel form -----------------------------------------------------------------

PAR_CASES = [
    ("bf16", 2, 2, 777, 128, 128, None),
    ("bf16", 1, 2, 512, 256, 512, 1e-5),
    ("bf16", 1, 3, 300, 64, 256, None),
    ("f32", 1, 2, 257, 64, 64, 1e-5),
]


@pytest.mark.parametrize("case", PAR_CASES, ids=lambda c: "-".join(map(str, c)))
def test_parallel_parity(torch_cuda, ret, case):
    torch = torch_cuda
    dt, B, H, N, dk, dv, gn = case
    inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=200 + N)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    o = ret.parallel(q, k, v, _gam(torch, inp["gammas"]), gn_eps=gn)
    torch.cuda.synchronize()
    o_ref, _ = oracle.parallel(inp["q"].exact, inp["k"].exact, inp["v"].exact, inp["gammas"])
    if gn is not None:
        o_ref = oracle.group_norm(o_ref, gn)
    assert _rel(o, o_ref) <= TOL[dt]


def _random_parallel_cases(n, seed):
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(1, 3)), int(rng.integers(1, 4)), int(rng.integers(1, 1300)),
             int(rng.choice([64, 128, 256])), int(rng.choice([64, 128, 256, 512])),
             1e-5 if rng.random() < 0.5 else None) for _ in range(n)]


@pytest.mark.parametrize("case", _random_parallel_cases(8, 2025), ids=lambda c: "-".join(map(str, c)))
def test_parallel_random_tensor_core_shapes(torch_cuda, ret, case):
    torch = torch_cuda
    B, H, N, dk, dv, gn = case
    inp = wl.make_inputs(B, H, N, dk, dv, "bf16", seed=400 + N)
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    o = ret.parallel(q, k, v, _gam(torch, inp["gammas"]), gn_eps=gn)
    torch.cuda.synchronize()
    o_ref, _ = oracle.parallel(inp["q"].exact, inp["k"].exact, inp["v"].exact, inp["gammas"])
    if gn is not None:
        o_ref = oracle.group_norm(o_ref, gn)
    assert _rel(o, o_ref) <= TOL["bf16"]


# --- decode step -------------------------------------------------------------------

STEP_CASES = [
    ("bf16", 2, 3, 256, 512, None),
    ("bf16", 2, 3, 256, 512, 1e-5),
    ("f32", 3, 2, 64, 64, None),
    ("f32", 1, 2, 136, 200, 1e-5),
    ("bf16", 1, 1, 8, 1024, 1e-5),
]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: "-".join(map(str, c)))
def test_step_parity(torch_cuda, ret, case):
    torch = torch_cuda
    dt, B, H, dk, dv, gn = case
    T = 5
    inp = wl.make_inputs(B, H, T, dk, dv, dt, seed=300 + dk, with_state=True)
    state = _dev(inp["state"])
    S = inp["state"].exact
    for n in range(T):
        qn, kn, vn = (inp[x].exact[:, :, n] for x in ("q", "k", "v"))
        o_ref, S = oracle.step(qn, kn, vn, inp["gammas"], S)
        if gn is not None:
            o_ref = oracle.group_norm(o_ref, gn)
        o = ret.step(_dev(inp["q"])[:, :, n].contiguous(), _dev(inp["k"])[:, :, n].contiguous(),
                     _dev(inp["v"])[:, :, n].contiguous(), _gam(torch, inp["gammas"]), state,
                     gn_eps=gn)
        torch.cuda.synchronize()
        assert _rel(o, o_ref) <= TOL[dt]
    assert _rel(state, S) <= STATE_TOL


# --- degenerate cases --------------------------------------------------------------

@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_gamma_zero_and_one(torch_cuda, ret, dt):
    """gamma = 0 reduces to o_n = (q_n.k_n) v_n; gamma = 1 is causal linear
    attention; both must stay finite (no 0*log(0) NaN)."""
    torch = torch_cuda
    B, H, N, dk, dv, C = 1, 2, 300, 64, 64, 128
    inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=9, gammas=[0.0, 1.0])
    q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
    g = _gam(torch, inp["gammas"])
    o_ref, s_ref = oracle.chunkwise(inp["q"].exact, inp["k"].exact, inp["v"].exact,
                                    inp["gammas"], C)
    o, s = ret.chunkwise(q, k, v, g, C, return_state=True)
    op = ret.parallel(q, k, v, g)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(op.float()).all()
    assert _rel(o, o_ref) <= TOL[dt]
    assert _rel(op, o_ref) <= TOL[dt]
    assert _rel(s, s_ref) <= STATE_TOL


def test_single_token_and_short_sequence(torch_cuda, ret):
    torch = torch_cuda
    for N in (1, 5, 127, 129):
        inp = wl.make_inputs(1, 2, N, 128, 128, "bf16", seed=N, with_state=True)
        q, k, v = _dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"])
        g = _gam(torch, inp["gammas"])
        o, s = ret.chunkwise(q, k, v, g, 256, state_in=_dev(inp["state"]), return_state=True)
        torch.cuda.synchronize()
        o_ref, s_ref = _ref_chunkwise(inp, 256, None, True)
        assert _rel(o, o_ref) <= TOL["bf16"], N
        assert _rel(s, s_ref) <= STATE_TOL, N


def test_empty_sequence_copies_state(torch_cuda, ret):
    torch = torch_cuda
    B, H, dk, dv = 1, 2, 64, 64
    q = torch.empty((B, H, 0, dk), dtype=torch.bfloat16, device="cuda")
    v = torch.empty((B, H, 0, dv), dtype=torch.bfloat16, device="cuda")
    g = _gam(torch, [0.9, 0.5])
    s0 = torch.randn((B, H, dk, dv), device="cuda")
    o, s = ret.chunkwise(q, q, v, g, 128, state_in=s0, return_state=True)
    o2, z = ret.chunkwise(q, q, v, g, 128, return_state=True)
    op = ret.parallel(q, q, v, g)
    torch.cuda.synchronize()
    assert o.numel() == 0 and op.numel() == 0
    assert torch.equal(s, s0)
    assert torch.count_nonzero(z) == 0


# --- xPos rotation ----------------------------------------------------------------

def _rotation_close(y, ref, x_exact, dt):
    """float32: 1e-5 rel-Frobenius.  bf16: one rounding of each output, so
    |y - ref| <= 2^-8 |ref| + 1e-5 max|x| element by element."""
    y = wl.from_torch(y)
    if dt == "f32":
        assert oracle.rel_frobenius(y, ref) < TOL["f32"]
    else:
        bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.max(np.abs(x_exact))
        assert np.all(np.abs(y - ref) <= bound)


# (dtype, B, H, N, d, pos0): d % 8 != 0 takes the one-pair-per-thread path;
# B*H = 17 and 5 leave partial 4-row groups and 16-row shares; a pos0 of 1.2e8
# turns pairs by up to 1.2e8 rad.
ROT_CASES = [("f32", 2, 3, 300, 64, 0), ("bf16", 2, 3, 300, 64, 5), ("f32", 1, 2, 37, 6, 0),
             ("bf16", 1, 2, 129, 10, 1000000), ("f32", 1, 5, 17, 256, 123456789),
             ("bf16", 1, 17, 64, 512, 7), ("bf16", 4, 16, 70, 128, 3)]


@pytest.mark.parametrize("case", ROT_CASES, ids=lambda c: "-".join(map(str, c)))
def test_rotate_parity(torch_cuda, ret, case):
    torch = torch_cuda
    dt, B, H, N, d, pos0 = case
    rng = np.random.Generator(np.random.PCG64(N * 131 + d))
    x = wl.draw(rng, (B, H, N, d), 1.0, dt)
    th = wl.rotation_angles(d, seed=d)
    ref = oracle.rotate(x.exact, th.astype(np.float64), pos0)
    xd = _dev(x)
    y = ret.rotate(xd, torch.from_numpy(th).cuda(), pos0)
    _rotation_close(y, ref, x.exact, dt)
    ret.rotate(xd, torch.from_numpy(th).cuda(), pos0, out=xd)   # in place
    torch.cuda.synchronize()
    assert torch.equal(xd, y)


def test_rotate_decode_row_and_empty(torch_cuda, ret):
    """One position per (batch, head), as in a decode step at position 4095;
    an empty sequence writes nothing."""
    torch = torch_cuda
    rng = np.random.Generator(np.random.PCG64(77))
    x = wl.draw(rng, (2, 4, 256), 1.0, "bf16")
    th = wl.rotation_angles(256, seed=3)
    y = ret.rotate(_dev(x), torch.from_numpy(th).cuda(), 4095)
    ref = oracle.rotate(x.exact[:, :, None, :], th.astype(np.float64), 4095)[:, :, 0]
    _rotation_close(y, ref, x.exact, "bf16")
    e = torch.full((1, 2, 0, 64), 3.0, device="cuda")
    assert ret.rotate(e, torch.from_numpy(wl.rotation_angles(64)).cuda()).shape == e.shape


@pytest.mark.parametrize("dt,gn,gated", [("bf16", None, False), ("bf16", 1e-5, True),
                                         ("f32", None, False), ("f32", 1e-5, False)])
def test_step_rotated_matches_rotation_then_step(torch_cuda, ret, dt, gn, gated):
    """The decode step with the xPos rotation fused into its loads
    (ret_step_rotated) at positions 0, 1, 4095 and 1.2e8, against the oracle's
    rotation of q and k at that position followed by its recurrent step (and
    GroupNorm and the gate where asked)."""
    torch = torch_cuda
    B, H, dk, dv = 2, 3, 256, 512
    inp = wl.make_inputs(B, H, 1, dk, dv, dt, seed=61, with_state=True)
    q, k, v = (_dev(inp[n])[:, :, 0].contiguous() for n in ("q", "k", "v"))
    qe, ke, ve = (inp[n].exact[:, :, 0] for n in ("q", "k", "v"))
    g = _gam(torch, inp["gammas"])
    th = wl.rotation_angles(dk, seed=7)
    tht = torch.from_numpy(th).cuda()
    gate = wl.draw(np.random.Generator(np.random.PCG64(62)), (B, H, dv), 1.0, dt) if gated \
        else None
    for pos in (0, 1, 4095, 123456789):
        state = _dev(inp["state"]).clone()
        o = ret.step(q, k, v, g, state, gn_eps=gn, theta=tht, pos=pos,
                     gate=None if gate is None else _dev(gate))
        torch.cuda.synchronize()
        qr = oracle.rotate(qe[:, :, None, :], th.astype(np.float64), pos)[:, :, 0]
        kr = oracle.rotate(ke[:, :, None, :], th.astype(np.float64), pos)[:, :, 0]
        o_ref, s_ref = oracle.step(qr, kr, ve, inp["gammas"], inp["state"].exact)
        if gn is not None:
            o_ref = oracle.group_norm(o_ref, gn)
        if gate is not None:
            o_ref = oracle.gated(o_ref, gate.exact)
        assert _rel(o, o_ref) <= TOL[dt], pos
        assert _rel(state, s_ref) <= STATE_TOL, pos
    # without theta the call is the plain step
    s1, s2 = _dev(inp["state"]).clone(), _dev(inp["state"]).clone()
    o1 = ret.step(q, k, v, g, s1, gn_eps=gn)
    o2 = ret.step(q, k, v, g, s2, gn_eps=gn, theta=None, pos=77)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_rotated_retention_matches_oracle(torch_cuda, ret):
    """Rotation followed by retention (parallel and chunkwise) against the
    oracle's rotation followed by its recurrence."""
    torch = torch_cuda
    inp = wl.make_inputs(1, 2, 96, 16, 8, "f32", seed=41)
    th = wl.rotation_angles(16, seed=5)
    tht = torch.from_numpy(th).cuda()
    qr = ret.rotate(_dev(inp["q"]), tht, 11)
    kr = ret.rotate(_dev(inp["k"]), tht, 11)
    g = _gam(torch, inp["gammas"])
    o_ref, _ = oracle.recurrent(oracle.rotate(inp["q"].exact, th.astype(np.float64), 11),
                                oracle.rotate(inp["k"].exact, th.astype(np.float64), 11),
                                inp["v"].exact, inp["gammas"])
    v = _dev(inp["v"])
    assert _rel(ret.parallel(qr, kr, v, g), o_ref) < TOL["f32"]
    assert _rel(ret.chunkwise(qr, kr, v, g, 32), o_ref) < TOL["f32"]


def test_rotate_full_size_sampled(torch_cuda, ret):
    """The 6.7B-class 8k layer's q (8 x 16 x 8192 x 256, bf16) rotated in
    place as the bench does; sampled rows against the oracle."""
    torch = torch_cuda
    B, H, N, d = 8, 16, 8192, 256
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    x = torch.randn((B, H, N, d), device="cuda", generator=gen).bfloat16()
    th = wl.rotation_angles(d, seed=9)
    rows = [(0, 0, 0), (7, 15, 8191), (3, 9, 4097), (5, 2, 1), (1, 14, 6000)]
    before = [wl.from_torch(x[b, h, n]) for b, h, n in rows]
    ret.rotate(x, torch.from_numpy(th).cuda(), 0, out=x)
    torch.cuda.synchronize()
    for (b, h, n), xe in zip(rows, before):
        ref = oracle.rotate(xe[None, :], th.astype(np.float64), n)[0]
        _rotation_close(x[b, h, n], ref, xe, "bf16")
    del x
    torch.cuda.empty_cache()
