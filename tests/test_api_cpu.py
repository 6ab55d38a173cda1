"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every entry point ``include/ssd.h`` declares, sizes its
workspace, and rejects bad arguments before anything reaches the device.
Every call here fails validation before the first CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_17_b200 import build
    build.build()
    from selective_state_space_17_b200 import ssd
    return ssd.lib


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(ssd_[a-z_0-9]+)\s*\(", text))
    return names


def test_library_exports_every_declared_entry_point(lib):
    names = _declared()
    assert {"ssd_forward", "ssd_step", "ssd_workspace_size", "ssd_poll_status"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_forward_path_query(lib):
    # bf16 with P = 64 and N a multiple of 8 up to 256 takes a tensor-core
    # path: the head-group kernel when there are enough (batch, head pair)
    # chains and N <= 128, else the per-head kernel; few chains on a long
    # sequence run segment-parallel; fp32 and other sizes take the SIMT path
    assert lib.ssd_forward_path(4, 4096, 80, 64, 1, 128, 256, 1) == 4
    assert lib.ssd_forward_path(8, 2048, 32, 64, 1, 128, 256, 1) == 4
    assert lib.ssd_forward_path(1, 4096, 4, 64, 1, 128, 256, 1) == 3
    assert lib.ssd_forward_path(1, 64, 2, 8, 1, 8, 16, 0) == 1
    assert lib.ssd_forward_path(1, 512, 2, 64, 1, 256, 128, 1) == 2   # N = 256: two passes
    assert lib.ssd_forward_path(1, 512, 2, 64, 1, 252, 128, 1) == 1   # N % 8 != 0: SIMT
    assert lib.ssd_forward_path(1, 512, 2, 32, 1, 128, 128, 1) == 1   # P = 32: SIMT
    assert lib.ssd_forward_path(1, 512, 2, 128, 1, 128, 128, 1) == 2  # P = 128: two 64-wide heads
    assert lib.ssd_forward_path(1, 512, 2, 96, 1, 128, 128, 1) == 1   # P = 96: SIMT
    assert lib.ssd_forward_path(1, 64, 3, 8, 2, 8, 16, 0) == 0        # H % G != 0
    assert lib.ssd_forward_path(0, 64, 2, 8, 1, 8, 16, 0) == 0        # no tokens


def test_kernel_count_query(lib):
    # one launch per 128 state columns on the tensor-core single pass (no SM
    # count is readable here, so the query assumes 148)
    assert lib.ssd_forward_kernel_count(1, 512, 2, 64, 1, 128, 128, 1) == 1
    assert lib.ssd_forward_kernel_count(1, 512, 2, 64, 1, 256, 128, 1) == 2
    assert lib.ssd_forward_kernel_count(1, 4096, 4, 64, 1, 200, 256, 1) == 6
    assert lib.ssd_forward_kernel_count(1, 64, 2, 8, 1, 8, 16, 0) == 3


def test_workspace_size_formula(lib):
    """Per-head kernel's single pass (the larger of the two tensor-core
    layouts): 256 B of control words, one 8-byte tagged flag per chain rounded
    up to 256 B, and a two-slot [128][64] fp32 state ring per chain, where a
    chain is one 64-channel head slice of one batch row (M = B*H*P/64); the
    query adds 256 bytes of slack."""
    def single(M):
        return 256 + (8 * M + 255) // 256 * 256 + M * 2 * 64 * 128 * 4 + 256
    assert lib.ssd_workspace_size(4, 4096, 80, 64, 1, 128, 256, 1) == single(4 * 80)
    assert lib.ssd_workspace_size(8, 2048, 32, 64, 1, 128, 256, 1) == single(8 * 32)
    assert lib.ssd_workspace_size(2, 8192, 64, 64, 8, 256, 256, 1) == single(2 * 64)  # two passes share it
    assert lib.ssd_workspace_size(2, 512, 4, 128, 2, 128, 128, 1) == single(2 * 4 * 2)  # wide heads


def test_segment_parallel_workspace_adds_per_segment_states(lib):
    # long context: 32 chains of 512 tiles; with 148 SMs (the value assumed
    # without a GPU) each chain is cut into 37 segments of 14 tiles
    M, nseg = 32, 37
    base = 256 + 256 + M * 2 * 64 * 128 * 4 + 256  # control, flags (8 B each), ring, slack
    slot = 64 * 128 * 4
    extra = M * nseg * slot + (4 * M * nseg + 255) // 256 * 256 + M * nseg * slot
    assert lib.ssd_forward_path(1, 65536, 32, 64, 1, 128, 256, 1) == 3
    assert lib.ssd_forward_kernel_count(1, 65536, 32, 64, 1, 128, 256, 1) == 3
    assert lib.ssd_workspace_size(1, 65536, 32, 64, 1, 128, 256, 1) == base + extra


def test_benchmark_workloads_take_the_tensor_core_path(lib):
    # the layers with many (batch, head pair) chains take the head-group kernel
    assert lib.ssd_forward_path(4, 4096, 80, 64, 1, 128, 256, 1) == 4      # 2.7B layer
    assert lib.ssd_forward_kernel_count(4, 4096, 80, 64, 1, 128, 256, 1) == 1
    assert lib.ssd_forward_path(8, 2048, 32, 64, 1, 128, 256, 1) == 4      # 370M layer
    for N in (16, 32, 64, 128, 256):                                       # sweep
        for Q in (128, 256):
            assert lib.ssd_forward_path(2, 8192, 64, 64, 8, N, Q, 1) == 2
            assert lib.ssd_forward_kernel_count(2, 8192, 64, 64, 8, N, Q, 1) == (2 if N > 128 else 1)


def test_status_strings(lib):
    for code in range(7):
        s = lib.ssd_status_string(code).decode()
        assert s.startswith("SSD_")
    assert lib.ssd_status_string(99).decode() == "SSD_ERR_UNKNOWN"


def test_workspace_size(lib):
    assert lib.ssd_workspace_size(4, 4096, 80, 64, 1, 128, 256, 1) > 0
    assert lib.ssd_workspace_size(1, 64, 2, 8, 1, 8, 16, 0) > 0
    assert lib.ssd_workspace_size(1, 64, 3, 8, 2, 8, 16, 0) == 0   # H % G != 0
    assert lib.ssd_workspace_size(1, 64, 2, 8, 1, 8, 0, 0) == 0    # chunk 0
    assert lib.ssd_workspace_size(1, 64, 2, 512, 1, 8, 16, 0) == 0  # P too large
    assert lib.ssd_workspace_size(1, 64, 2, 8, 1, 8, 16, 7) == 0   # bad dtype
    a = lib.ssd_workspace_size(1, 4096, 2, 64, 1, 64, 128, 1)
    b = lib.ssd_workspace_size(1, 8192, 2, 64, 1, 64, 128, 1)
    assert b >= a


P16 = [0x10000 * (i + 1) for i in range(10)]  # aligned, never dereferenced


def _fwd(lib, ptrs, dims, ws_bytes=1 << 40):
    x, dt, A, Bm, Cm, D, init, y, fs, ws = ptrs
    return lib.ssd_forward(x, dt, A, Bm, Cm, D, init, y, fs, *dims, ws, ws_bytes, None)


def test_forward_rejects_bad_arguments_before_launch(lib):
    dims = (1, 64, 2, 8, 1, 8, 16, 0)
    bad_dims = [(1, 64, 3, 8, 2, 8, 16, 0), (-1, 64, 2, 8, 1, 8, 16, 0),
                (1, -5, 2, 8, 1, 8, 16, 0), (1, 64, 0, 8, 1, 8, 16, 0),
                (1, 64, 2, 8, 1, 8, 0, 0), (1, 64, 2, 8, 1, 8, 16, 5)]
    for d in bad_dims:
        assert _fwd(lib, P16, d) == 1, d
    for d in [(1, 64, 2, 300, 1, 8, 16, 0), (1, 64, 2, 8, 1, 300, 16, 0),
              (1, 64, 2, 8, 1, 8, 512, 0)]:
        assert _fwd(lib, P16, d) == 2, d
    for k in (0, 1, 2, 3, 4, 7):  # required pointers
        ptrs = list(P16)
        ptrs[k] = None
        assert _fwd(lib, ptrs, dims) == 1, k
    for k in range(10):  # every pointer, optional ones included, must be aligned
        ptrs = list(P16)
        ptrs[k] += 4
        assert _fwd(lib, ptrs, dims) == 3, k
    ptrs = list(P16)
    ptrs[9] = None
    assert _fwd(lib, ptrs, dims) == 6
    assert _fwd(lib, P16, dims, ws_bytes=16) == 6


def test_step_rejects_bad_arguments_before_launch(lib):
    ok = P16[:8]
    assert lib.ssd_step(*ok, 2, 3, 8, 2, 8, 0, None) == 1   # H % G
    assert lib.ssd_step(*ok, 2, 2, 8, 1, 8, 9, None) == 1   # dtype
    assert lib.ssd_step(*ok, 2, 2, 999, 1, 8, 0, None) == 2
    for k in (0, 1, 2, 3, 4, 6, 7):
        ptrs = list(ok)
        ptrs[k] = None
        assert lib.ssd_step(*ptrs, 2, 2, 8, 1, 8, 0, None) == 1, k
    ptrs = list(ok)
    ptrs[6] += 8
    assert lib.ssd_step(*ptrs, 2, 2, 8, 1, 8, 0, None) == 3


def test_host_entry_rejects_small_buffer(lib):
    need = lib.ssd_forward_host_buffer_size(1, 64, 2, 8, 1, 8, 16, 0)
    assert need > lib.ssd_workspace_size(1, 64, 2, 8, 1, 8, 16, 0)
    rc = lib.ssd_forward_host(*P16[:9], 1, 64, 2, 8, 1, 8, 16, 0, P16[9], need - 1, None)
    assert rc == 6


def test_binding_fails_loudly_without_library(tmp_path):
    """The Python binding has no fallback: a missing library is an ImportError."""
    import subprocess
    import sys
    code = ("import os, sys, importlib.util; "
            "spec = importlib.util.spec_from_file_location('ssd_copy', sys.argv[1]); "
            "m = importlib.util.module_from_spec(spec); spec.loader.exec_module(m)")
    src = os.path.join(ROOT, "selective_state_space_17_b200", "ssd.py")
    copy = tmp_path / "ssd.py"
    copy.write_text(open(src).read())
    r = subprocess.run([sys.executable, "-c", code, str(copy)], capture_output=True, text=True)
    assert r.returncode != 0 and "ImportError" in r.stderr and "no CPU" in r.stderr
