"""The allocation-free entry point, ssd_forward_noalloc, called through the C ABI.

It serves callers that cannot allocate device memory (code where cudaMalloc
is not allowed or the memory pool is full, or that has nowhere to keep a
workspace alive): its scratch is a fixed array inside the library. Its output
must match ssd_forward (the workspace entry point) and the fp64 oracle within
the bf16 tolerance of the other tests, on two calls in a row, since the second
call finds the first call's leftovers in the shared array. That covers the
single pass, the two passes over the state columns and the segment-parallel
form (per-segment states and the scan, in the shared array too). Oversized and
unsupported sizes must be refused before anything runs.

This file is named so that pytest collects it last.
"""
import ctypes

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
    fn = _ssd.lib.ssd_forward_noalloc
    fn.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 8 + [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return _ssd


def _noalloc(ssd, t, y, fs, shape, chunk, stream):
    Bsz, L, H, P, G, N = shape
    return ssd.lib.ssd_forward_noalloc(
        t["x"].data_ptr(), t["dt"].data_ptr(), t["A"].data_ptr(), t["Bm"].data_ptr(),
        t["Cm"].data_ptr(), t["D"].data_ptr(), None, y.data_ptr(), fs.data_ptr(),
        Bsz, L, H, P, G, N, chunk, ssd.SSD_BF16, stream.cuda_stream)


@pytest.mark.parametrize("shape,chunk,seed", [
    ((2, 1000, 8, 64, 1, 128), 256, 31),   # ragged last tile
    ((1, 640, 6, 64, 2, 128), 128, 32),
    ((1, 640, 4, 64, 2, 256), 128, 35),    # two passes over the state columns
    ((1, 16384, 2, 64, 1, 128), 256, 36),  # few long chains: segment-parallel form
])
def test_noalloc_matches_workspace_entry_point_and_oracle_on_two_calls(ssd, oracle, shape,
                                                                       chunk, seed):
    stream = torch.cuda.current_stream()
    inp = gen.make_inputs(*shape, "bf16", seed=seed)
    t = to_device(inp)
    y_ref, fs_ref = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=chunk)
    ssd.poll_status()
    x, dt, A, Bm, Cm, D = inp.f64()
    y_or, fs_or = oracle.forward(x, dt, A, Bm, Cm, D)
    for _ in range(2):
        y = torch.full_like(y_ref, 7.0)
        fs = torch.full_like(fs_ref, 7.0)
        rc = _noalloc(ssd, t, y, fs, shape, chunk, stream)
        assert rc == 0, ssd.STATUS.get(rc, rc)
        ssd.poll_status()
        yh, fh = to_host_f64(y), to_host_f64(fs)
        assert slice_rel_err(yh, to_host_f64(y_ref), 2) < TOL["bf16"]
        assert slice_rel_err(fh, to_host_f64(fs_ref), 1) < TOL["bf16"]
        assert slice_rel_err(yh, y_or, 2) < TOL["bf16"]
        assert slice_rel_err(fh, fs_or, 1) < TOL["bf16"]


def test_noalloc_refuses_what_it_cannot_run(ssd):
    stream = torch.cuda.current_stream()
    # 8 x 64 = 512 heads need 32 MiB of state ring: more than the fixed array
    big = (8, 128, 64, 64, 1, 128)
    t = to_device(gen.make_inputs(*big, "bf16", seed=33))
    y = torch.empty_like(t["x"])
    fs = torch.empty((8, 64, 64, 128), dtype=torch.float32, device="cuda")
    assert _noalloc(ssd, t, y, fs, big, 128, stream) == 6  # SSD_ERR_WORKSPACE
    # P = 32 is not a tensor-core size (the tiles hold P = 64)
    small = (1, 256, 2, 32, 1, 128)
    t = to_device(gen.make_inputs(*small, "bf16", seed=34))
    y = torch.empty_like(t["x"])
    fs = torch.empty((1, 2, 32, 128), dtype=torch.float32, device="cuda")
    assert _noalloc(ssd, t, y, fs, small, 128, stream) == 2  # SSD_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert np.isfinite(to_host_f64(t["x"][:1, :1])).all()
