"""GPU parity of the head-group tensor-core kernel (two heads of one B/C group
per tile, shared tril(C B^T), the scaled form of the decay mask and its exact
form for tiles of large decay) against the fp64 oracle.

The kernel is forced with the ssd_set_forward_variant test hook so that small
cases, which the automatic choice would send to the per-head kernel, run
through it too. Tolerance and metric as in test_parity_gpu.py.
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
    _ssd.set_forward_variant(2)
    yield _ssd
    _ssd.set_forward_variant(0)


def _check(ssd, oracle, inp, chunk, init=None, D=True, record=None):
    B, L, H, P = inp.x.shape
    G, N = inp.Bm.shape[2], inp.Bm.shape[3]
    assert ssd.forward_path(B, L, H, P, G, N, chunk, 1) == 4
    t = to_device(inp)
    init_t = None if init is None else torch.from_numpy(init.astype(np.float32)).cuda()
    y, fs = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"] if D else None,
                        chunk=chunk, initial_state=init_t)
    ssd.poll_status()
    x, dt, A, Bm, Cm, Dv = inp.f64()
    yr, fsr = oracle.forward(x, dt, A, Bm, Cm, Dv if D else None, init_state=init)
    ey = slice_rel_err(to_host_f64(y), yr, head_axis=2)
    es = slice_rel_err(to_host_f64(fs), fsr, head_axis=1)
    tol = TOL["bf16"]
    if record is not None:
        record("slice_rel_err_y", ey)
        record("slice_rel_err_final_state", es)
        record("elementwise_rel_err_y", elementwise_rel_err(to_host_f64(y), yr))
    assert ey < tol and es < tol, (ey, es)
    return ey, es


@pytest.mark.parametrize("shape,chunk", [
    ((2, 640, 4, 64, 2, 128), 256),   # two heads per group, ragged tail
    ((1, 384, 8, 64, 8, 64), 128),    # one head per group (KH = 1), N = 64
    ((2, 300, 4, 64, 1, 32), 128),    # N = 32: half of each C/B tile is padding
    ((1, 500, 2, 64, 1, 8), 64),      # N = 8
    ((1, 520, 4, 64, 2, 120), 256),   # N not a multiple of 16
    ((2, 300, 2, 128, 1, 128), 128),  # P = 128: the two halves of a head share a tile
    ((1, 1000, 3, 192, 3, 96), 256),  # P = 192, one model head per group
    ((1, 4096, 4, 64, 1, 128), 256),  # many segments per chain (look-back)
])
def test_grouped_shapes(ssd, oracle, shape, chunk, record_property):
    _check(ssd, oracle, gen.make_inputs(*shape, "bf16", seed=21), chunk, record=record_property)


@pytest.mark.parametrize("kind", ["linear_attention", "retnet", "zero_decay", "mixed_decay"])
@pytest.mark.parametrize("shape", [(2, 512, 4, 64, 2, 64), (1, 700, 6, 64, 3, 128)])
def test_grouped_special_and_exact_form(ssd, oracle, kind, shape, record_property):
    """a = 1 and a = 0.99 stay on the scaled form; a = 0 (dt A = -1000) and the
    strongly decaying heads of the mixed kind take the exact form, tile by tile,
    next to scaled tiles of the same launch."""
    _check(ssd, oracle, gen.make_inputs(*shape, "bf16", seed=22, kind=kind), 128,
           record=record_property)


@pytest.mark.parametrize("shape,D", [((2, 900, 4, 64, 2, 128), True),
                                     ((1, 3000, 2, 128, 1, 64), False)])
def test_grouped_initial_state(ssd, oracle, shape, D):
    B, L, H, P, G, N = shape
    inp = gen.make_inputs(*shape, "bf16", seed=23)
    init = np.random.default_rng(4).standard_normal((B, H, P, N)).astype(np.float32)
    _check(ssd, oracle, inp, 256, init=init, D=D)


def test_grouped_matches_per_head_kernel(ssd):
    """Both tensor-core kernels on one input: same result within bf16 rounding."""
    inp = gen.make_inputs(2, 1536, 8, 64, 2, 128, "bf16", seed=24)
    t = to_device(inp)
    y2, f2 = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=256)
    ssd.set_forward_variant(1)
    try:
        y1, f1 = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=256)
    finally:
        ssd.set_forward_variant(2)
    ssd.poll_status()
    assert slice_rel_err(to_host_f64(y2), to_host_f64(y1), 2) < 2e-2
    assert slice_rel_err(to_host_f64(f2), to_host_f64(f1), 1) < 2e-2


def test_grouped_repeated_calls(ssd):
    """One workspace reused by repeated calls (its control words carry the tag
    of the call that wrote them): the calls agree bit for bit."""
    inp = gen.make_inputs(2, 2048, 8, 64, 1, 128, "bf16", seed=25)
    t = to_device(inp)
    y0, f0 = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=256)
    for _ in range(3):
        y1, f1 = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=256)
    ssd.poll_status()
    assert torch.equal(y0, y1) and torch.equal(f0, f1)


def test_workspace_shared_by_every_path(ssd, oracle):
    """One workspace, never cleared, taken in turn by the SIMT path (fp32, which
    fills it with chunk states), the per-head kernel and the head-group kernel
    at different sizes: every call still matches the oracle, because no path
    reads another call's leftovers as its own control words."""
    ws = torch.full((64 << 20,), 0x5A, dtype=torch.uint8, device="cuda")  # garbage
    cases = [((2, 700, 8, 64, 2, 128), "f32", 0), ((2, 1500, 8, 64, 2, 128), "bf16", 1),
             ((4, 1300, 8, 64, 1, 128), "bf16", 2), ((2, 700, 8, 64, 2, 128), "f32", 0),
             ((4, 1300, 8, 64, 1, 128), "bf16", 1), ((2, 1500, 8, 64, 2, 128), "bf16", 2)]
    try:
        for i, (shape, dtype, variant) in enumerate(cases):
            ssd.set_forward_variant(variant)
            inp = gen.make_inputs(*shape, dtype, seed=30 + i)
            t = to_device(inp)
            y, fs = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=128,
                                workspace=ws)
            ssd.poll_status()
            yr, fsr = oracle.forward(*inp.f64())
            assert slice_rel_err(to_host_f64(y), yr, 2) < TOL[dtype], (i, shape, dtype)
            assert slice_rel_err(to_host_f64(fs), fsr, 1) < TOL[dtype], (i, shape, dtype)
    finally:
        ssd.set_forward_variant(2)
