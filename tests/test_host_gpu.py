"""The host-buffer entry point, ssd_forward_host: inputs on pinned host memory,
results copied back. It runs the batch in slices over two streams so that the
copies overlap the forward pass; every slice must give what ssd_forward gives
on device buffers, and the oracle's result."""
import numpy as np
import pytest

from selective_state_space_17_b200 import inputs as gen
from ssd_testutil import TOL, slice_rel_err, to_device, to_host_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ssd():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_17_b200 import ssd as _ssd
    return _ssd


def _host(inp):
    def io(a):
        if inp.dtype == "bf16":
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
        return torch.from_numpy(a).pin_memory()
    return dict(x=io(inp.x), dt=torch.from_numpy(inp.dt).pin_memory(),
                A=torch.from_numpy(inp.A).pin_memory(), Bm=io(inp.Bm), Cm=io(inp.Cm),
                D=torch.from_numpy(inp.D).pin_memory())


@pytest.mark.parametrize("shape,dtype,with_init", [
    ((5, 300, 4, 64, 2, 128), "bf16", True),    # four slices, the last one short
    ((3, 256, 8, 64, 1, 64), "bf16", False),    # three slices of one row
    ((1, 200, 2, 16, 1, 16), "f32", True),      # one slice, SIMT path
])
def test_forward_host_matches_device_entry_point_and_oracle(ssd, oracle, shape, dtype, with_init):
    B, L, H, P, G, N = shape
    inp = gen.make_inputs(*shape, dtype, seed=41)
    h = _host(inp)
    init = None
    if with_init:
        init = np.random.default_rng(5).standard_normal((B, H, P, N)).astype(np.float32)
    y = torch.empty_like(h["x"]).pin_memory()
    fs = torch.empty((B, H, P, N), dtype=torch.float32).pin_memory()
    init_h = None if init is None else torch.from_numpy(init).pin_memory()
    for _ in range(2):  # twice: the device buffer's workspaces are reused
        y.fill_(7.0)
        fs.fill_(7.0)
        ssd.forward_host(h["x"], h["dt"], h["A"], h["Bm"], h["Cm"], h["D"], y, fs,
                         initial_state=init_h, chunk=128)
        t = to_device(inp)
        yd, fd = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=128,
                             initial_state=None if init is None else init_h.cuda())
        ssd.poll_status()
        tol = TOL[dtype]
        assert slice_rel_err(to_host_f64(y), to_host_f64(yd), 2) < tol
        assert slice_rel_err(to_host_f64(fs), to_host_f64(fd), 1) < tol
    x, dt, A, Bm, Cm, D = inp.f64()
    yr, fsr = oracle.forward(x, dt, A, Bm, Cm, D, init_state=init)
    assert slice_rel_err(to_host_f64(y), yr, 2) < TOL[dtype]
    assert slice_rel_err(to_host_f64(fs), fsr, 1) < TOL[dtype]
