"""GPU parity: the CUDA path against the fp64 oracle on the same seeded inputs.

Tolerance (max over (batch, head) slices of ||y_hat - y||_inf / ||y||_inf, and
the same for final_state): 1e-4 for fp32 I/O, 2e-2 for bf16 I/O. Small cases
compare every element; the full-size workloads run in the launch
configuration the benchmark times and compare whole (batch, head) slices that
the oracle computes one at a time.
"""
import numpy as np
import pytest

from selective_state_space_17_b200 import inputs as gen
from ssd_testutil import TOL, elementwise_rel_err, slice_rel_err, to_device, to_host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ssd():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_17_b200 import ssd as _ssd
    return _ssd


def _run(ssd, inp, chunk, init=None, D=True):
    t = to_device(inp)
    init_t = None if init is None else torch.from_numpy(init.astype(np.float32)).cuda()
    y, fs = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"] if D else None,
                        chunk=chunk, initial_state=init_t)
    ssd.poll_status()
    return to_host_f64(y), to_host_f64(fs)


def _full_check(ssd, oracle, inp, chunk, init=None, D=True, record=None):
    y, fs = _run(ssd, inp, chunk, init, D)
    x, dt, A, Bm, Cm, Dv = inp.f64()
    yr, fsr = oracle.forward(x, dt, A, Bm, Cm, Dv if D else None, init_state=init)
    tol = TOL[inp.dtype]
    ey = slice_rel_err(y, yr, head_axis=2)
    es = slice_rel_err(fs, fsr, head_axis=1)
    if record is not None:  # the metric and the elementwise diagnostic, for the record
        record("slice_rel_err_y", ey)
        record("slice_rel_err_final_state", es)
        record("elementwise_rel_err_y", elementwise_rel_err(y, yr))
    assert ey < tol and es < tol, (ey, es)
    return ey, es


# ------------------------------------------------------------------ small, full compare

def test_tiny_fp32_workload(ssd, oracle):
    w = gen.TINY_F32
    _full_check(ssd, oracle, w.make(0), w.chunk)


@pytest.mark.parametrize("shape,chunk", [
    ((2, 100, 3, 8, 1, 8), 16),      # ragged tail
    ((1, 257, 4, 5, 2, 7), 32),      # odd P, N
    ((2, 64, 2, 64, 1, 128), 64),
    ((1, 300, 2, 16, 2, 16), 1),     # chunk of one token
])
def test_fp32_small_shapes(ssd, oracle, shape, chunk, record_property):
    _full_check(ssd, oracle, gen.make_inputs(*shape, "f32", seed=3), chunk, record=record_property)


@pytest.mark.parametrize("shape,chunk", [
    ((2, 640, 4, 64, 2, 128), 256),  # 2.5 chunks: ragged tail on the tensor-core path
    ((1, 384, 8, 64, 8, 64), 128),   # G = H
    ((2, 200, 4, 64, 1, 32), 128),   # chunk longer than half the sequence
    ((1, 1000, 2, 64, 1, 256), 256), # N = 256
    ((1, 512, 2, 64, 1, 16), 128),   # N = 16
    ((1, 130, 3, 24, 3, 40), 48),    # SIMT path in bf16 (P, N off the fast path)
])
def test_bf16_small_shapes(ssd, oracle, shape, chunk, record_property):
    _full_check(ssd, oracle, gen.make_inputs(*shape, "bf16", seed=4), chunk, record=record_property)


@pytest.mark.parametrize("kind", ["linear_attention", "retnet", "zero_decay"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_special_cases(ssd, oracle, kind, dtype):
    inp = gen.make_inputs(2, 512, 4, 64, 2, 64, dtype, seed=5, kind=kind)
    _full_check(ssd, oracle, inp, 128 if dtype == "bf16" else 64)


@pytest.mark.parametrize("N,chunk", [(8, 64), (48, 128), (64, 256), (96, 64), (120, 128),
                                     (136, 64), (200, 128), (256, 256)])
def test_tensor_core_state_dims(ssd, oracle, N, chunk):
    """State dims below 128 run on the tensor-core path with the state rows
    zero-padded to 128; above 128 as two passes over the state columns, the
    second adding into y (a ragged tail, an initial state and two groups too)."""
    inp = gen.make_inputs(2, 300, 4, 64, 2, N, "bf16", seed=9)
    rng = np.random.default_rng(1)
    init = rng.standard_normal((2, 4, 64, N)).astype(np.float32)
    assert ssd.forward_path(2, 300, 4, 64, 2, N, chunk, 1) == 2
    assert ssd.kernel_count(2, 300, 4, 64, 2, N, chunk, 1) == (2 if N > 128 else 1)
    _full_check(ssd, oracle, inp, chunk, init=init)


@pytest.mark.parametrize("shape,chunk,with_init", [
    ((1, 4096, 4, 64, 1, 128), 256, False),   # 4 chains of 32 tiles: one tile per segment
    ((2, 3000, 2, 64, 1, 64), 128, True),     # ragged tail, N = 64, initial state
    ((1, 3000, 2, 64, 2, 192), 256, True),    # N = 192: two passes of three launches
])
def test_segment_parallel_form(ssd, oracle, shape, chunk, with_init):
    """Few chains with many tiles: each segment's local state, a scan over the
    segments, then the outputs (three launches instead of a serial look-back)."""
    assert ssd.forward_path(*shape, chunk, 1) == 3
    inp = gen.make_inputs(*shape, "bf16", seed=10)
    init = None
    if with_init:
        B, _, H, P, _, N = shape
        init = np.random.default_rng(2).standard_normal((B, H, P, N)).astype(np.float32)
    _full_check(ssd, oracle, inp, chunk, init=init)


@pytest.mark.parametrize("shape", [(2, 640, 6, 64, 1, 128), (1, 300, 3, 64, 3, 128)])
def test_tensor_core_mixed_decay(ssd, oracle, shape):
    """Tiles whose decay or zero steps rule out the factored mask take the exact
    form; the other tiles of the same launch take the factored one."""
    inp = gen.make_inputs(*shape, "bf16", seed=8, kind="mixed_decay")
    _full_check(ssd, oracle, inp, 128)


@pytest.mark.parametrize("shape,chunk", [
    ((2, 300, 4, 128, 2, 128), 128),   # P = 128: two 64-channel heads per head
    ((1, 200, 3, 192, 3, 200), 64),    # P = 192 with N = 200 (two passes)
    ((1, 3000, 2, 128, 1, 64), 256),   # P = 128, segment-parallel
])
def test_tensor_core_wide_heads(ssd, oracle, shape, chunk):
    """Heads of P = 64m channels run on the tensor-core path as m heads of 64
    channels that share dt, A and D (with an initial state, so its layout is
    checked too)."""
    B, L, H, P, G, N = shape
    assert ssd.forward_path(*shape, chunk, 1) in (2, 3)
    inp = gen.make_inputs(*shape, "bf16", seed=12)
    init = np.random.default_rng(3).standard_normal((B, H, P, N)).astype(np.float32)
    _full_check(ssd, oracle, inp, chunk, init=init)


def test_initial_state_and_no_skip_term(ssd, oracle):
    inp = gen.make_inputs(2, 384, 4, 64, 1, 128, "bf16", seed=6)
    rng = np.random.default_rng(0)
    init = rng.standard_normal((2, 4, 64, 128)).astype(np.float32)
    _full_check(ssd, oracle, inp, 128, init=init, D=False)


def test_continuation_through_initial_state(ssd):
    """forward(L) == forward(first half) then forward(second half, init = state)."""
    inp = gen.make_inputs(1, 1024, 4, 64, 1, 128, "bf16", seed=7)
    t = to_device(inp)
    y, fs = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=256)
    h = 512
    half = {k: (v[:, :h].contiguous() if v.dim() > 1 else v) for k, v in t.items()}
    rest = {k: (v[:, h:].contiguous() if v.dim() > 1 else v) for k, v in t.items()}
    y1, f1 = ssd.forward(half["x"], half["dt"], half["A"], half["Bm"], half["Cm"], half["D"],
                         chunk=256)
    y2, f2 = ssd.forward(rest["x"], rest["dt"], rest["A"], rest["Bm"], rest["Cm"], rest["D"],
                         chunk=256, initial_state=f1)
    ssd.poll_status()
    yy = torch.cat([y1, y2], dim=1)
    assert slice_rel_err(to_host_f64(yy), to_host_f64(y), 2) < 2e-2
    assert slice_rel_err(to_host_f64(f2), to_host_f64(fs), 1) < 2e-2


def test_empty_sequence_returns_initial_state(ssd):
    x = torch.empty((2, 0, 3, 8), device="cuda")
    dt = torch.empty((2, 0, 3), device="cuda")
    Bm = torch.empty((2, 0, 1, 8), device="cuda")
    A = torch.full((3,), -1.0, device="cuda")
    init = torch.randn(2, 3, 8, 8, device="cuda")
    y, fs = ssd.forward(x, dt, A, Bm, Bm, None, chunk=16, initial_state=init)
    ssd.poll_status()
    assert y.shape == x.shape and torch.equal(fs, init)
    _, fs0 = ssd.forward(x, dt, A, Bm, Bm, None, chunk=16)
    ssd.poll_status()
    assert torch.count_nonzero(fs0) == 0


def test_zero_batch_is_a_no_op(ssd):
    x = torch.empty((0, 64, 2, 64), dtype=torch.bfloat16, device="cuda")
    dt = torch.empty((0, 64, 2), device="cuda")
    Bm = torch.empty((0, 64, 1, 128), dtype=torch.bfloat16, device="cuda")
    A = torch.full((2,), -1.0, device="cuda")
    y, fs = ssd.forward(x, dt, A, Bm, Bm, None, chunk=128)
    ssd.poll_status()
    assert y.shape == x.shape and fs.shape == (0, 2, 64, 128)


def test_repeated_calls_reuse_the_workspace(ssd):
    inp = gen.make_inputs(2, 768, 4, 64, 1, 128, "bf16", seed=8)
    t = to_device(inp)
    y0, f0 = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=256)
    for _ in range(3):
        y1, f1 = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=256)
    ssd.poll_status()
    assert torch.equal(y0, y1) and torch.equal(f0, f1)


# Every step of a call has one fixed order of arithmetic, whatever CTA runs it,
# so repeated calls on the same inputs must agree bit for bit; a hand-off that
# lets a stage be overwritten before its last reader is done shows up here as
# an occasional difference (each of the two races this caught changed
# 0.3-8% of calls). The workloads take the head-group kernel (2.7B- and 370M-shaped
# layers) and the per-head kernel's single pass (sweep N = 16).
@pytest.mark.parametrize("w", [gen.LAYER_370M, gen.LAYER_2P7B] +
                         [v for v in gen.sweep_workloads() if v.N == 16 and v.chunk == 256],
                         ids=lambda w: w.name.split()[0])
def test_repeated_calls_are_bit_identical(ssd, w):
    t = to_device(w.make(0))
    y0, f0 = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=w.chunk)
    y0, f0 = y0.clone(), f0.clone()
    differ = 0
    for _ in range(100):
        y1, f1 = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=w.chunk)
        differ += int(not (torch.equal(y0, y1) and torch.equal(f0, f1)))
    ssd.poll_status()
    assert differ == 0, f"{differ} of 100 repeated calls differ"


# ------------------------------------------------------- full-size workloads, sampled heads

def _sampled_check(ssd, oracle, w, samples, seed=0):
    inp = w.make(seed)
    t = to_device(inp)
    y, fs = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=w.chunk)
    ssd.poll_status()
    tol = TOL[w.dtype]
    hpg = w.H // w.G
    worst = 0.0
    for b, g in samples:
        h0, h1 = g * hpg, (g + 1) * hpg
        x, dt, A, Bm, Cm, D = inp.f64(b, b + 1, heads=(h0, h1))
        yr, fsr = oracle.forward(x, dt, A, Bm, Cm, D)
        ey = slice_rel_err(to_host_f64(y[b:b + 1, :, h0:h1]), yr, 2)
        es = slice_rel_err(to_host_f64(fs[b:b + 1, h0:h1]), fsr, 1)
        worst = max(worst, ey, es)
        assert ey < tol and es < tol, (b, g, ey, es)
    assert torch.isfinite(y.float()).all()
    return worst


def test_layer_370m_sampled(ssd, oracle):
    # G = 1: a "group" sample is all 32 heads of one batch row
    _sampled_check(ssd, oracle, gen.LAYER_370M, [(0, 0), (7, 0)])


def test_layer_2p7b_sampled(ssd, oracle):
    _sampled_check(ssd, oracle, gen.LAYER_2P7B, [(0, 0), (3, 0)])


def test_long_context_sampled(ssd, oracle):
    _sampled_check(ssd, oracle, gen.LONG_CONTEXT, [(0, 0)])


@pytest.mark.parametrize("w", gen.sweep_workloads(), ids=lambda w: w.name.split()[-2] + w.name.split()[-1])
def test_sweep_sampled(ssd, oracle, w):
    _sampled_check(ssd, oracle, w, [(0, 0), (1, 7)])


@pytest.mark.parametrize("kind", ["linear_attention", "retnet"])
def test_sweep_special_sampled(ssd, oracle, kind):
    w = [v for v in gen.sweep_workloads((kind,)) if " N128 Q256" in v.name][0]
    _sampled_check(ssd, oracle, w, [(0, 3)])


# ------------------------------------------------------------------------------ decode

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_matches_oracle(ssd, oracle, dtype):
    d = gen.DECODE
    s = gen.make_step_inputs(d["B"], d["H"], d["P"], d["G"], d["N"], dtype, seed=11)
    io = (lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()) \
        if dtype == "bf16" else (lambda a: torch.from_numpy(a).cuda())
    state = torch.from_numpy(s.state).cuda()
    y = ssd.step(io(s.x), torch.from_numpy(s.dt).cuda(), torch.from_numpy(s.A).cuda(),
                 io(s.Bm), io(s.Cm), torch.from_numpy(s.D).cuda(), state)
    ssd.poll_status()
    f = lambda a: gen.to_f64(a, dtype)
    yr, str_ = oracle.step(f(s.x), s.dt, s.A, f(s.Bm), f(s.Cm), s.D, s.state)
    assert slice_rel_err(to_host_f64(y), yr, 1) < TOL[dtype]
    assert slice_rel_err(to_host_f64(state), str_, 1) < 1e-5


@pytest.mark.parametrize("shape", [(41, 8, 64, 2, 128),   # 328 heads
                                   (50, 6, 32, 3, 64),     # smaller state per head
                                   (40, 8, 16, 1, 20)])    # N = 20: rows of 80 bytes
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_shapes(ssd, oracle, shape, dtype):
    """More heads than one wave of CTAs, head counts that do not divide it,
    smaller states and a state dim that is not a multiple of 32."""
    B, H, P, G, N = shape
    s = gen.make_step_inputs(B, H, P, G, N, dtype, seed=13)
    io = (lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()) \
        if dtype == "bf16" else (lambda a: torch.from_numpy(a).cuda())
    state = torch.from_numpy(s.state).cuda()
    y = ssd.step(io(s.x), torch.from_numpy(s.dt).cuda(), torch.from_numpy(s.A).cuda(),
                 io(s.Bm), io(s.Cm), torch.from_numpy(s.D).cuda(), state)
    ssd.poll_status()
    f = lambda a: gen.to_f64(a, dtype)
    yr, str_ = oracle.step(f(s.x), s.dt, s.A, f(s.Bm), f(s.Cm), s.D, s.state)
    assert slice_rel_err(to_host_f64(y), yr, 1) < TOL[dtype]
    assert slice_rel_err(to_host_f64(state), str_, 1) < 1e-5


@pytest.mark.parametrize("N", [128, 13])
def test_steps_reproduce_forward(ssd, N):
    inp = gen.make_inputs(2, 48, 4, 16, 2, N, "f32", seed=12)
    t = to_device(inp)
    y, fs = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=16)
    state = torch.zeros((2, 4, 16, N), device="cuda")
    ys = []
    for i in range(48):
        ys.append(ssd.step(t["x"][:, i].contiguous(), t["dt"][:, i].contiguous(), t["A"],
                           t["Bm"][:, i].contiguous(), t["Cm"][:, i].contiguous(), t["D"],
                           state))
    ssd.poll_status()
    ys = torch.stack(ys, 1)
    assert slice_rel_err(to_host_f64(ys), to_host_f64(y), 2) < 1e-4
    assert slice_rel_err(to_host_f64(state), to_host_f64(fs), 1) < 1e-4
