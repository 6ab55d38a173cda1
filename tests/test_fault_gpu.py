"""Failure detection without a GPU fault: the look-back waits of the
tensor-core path are bounded. With the fault-injection hook no tile publishes
its end state, every wait runs out after a short iteration limit, the kernel
records the timeout in the device status word and returns, and the context
stays usable for the next (normal) call."""
import numpy as np
import pytest

from selective_state_space_17_b200 import inputs as gen
from ssd_testutil import slice_rel_err, to_device, to_host_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ssd():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_17_b200 import ssd as _ssd
    return _ssd


def test_bench_workload_takes_the_tensor_core_path(ssd):
    w = gen.LAYER_2P7B
    assert ssd.forward_path(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, ssd.SSD_BF16) == 4
    assert ssd.kernel_count(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, ssd.SSD_BF16) == 1
    assert ssd.forward_path(1, 64, 2, 8, 1, 8, 16, ssd.SSD_F32) == 1


@pytest.mark.parametrize("variant", [1, 2], ids=["per_head_kernel", "head_group_kernel"])
def test_lookback_timeout_is_reported_and_context_survives(ssd, oracle, variant):
    inp = gen.make_inputs(1, 512, 2, 64, 1, 128, "bf16", seed=21)
    t = to_device(inp)
    ssd.poll_status()  # clean slate
    try:
        ssd.set_forward_variant(variant)
        ssd.set_fault_injection(True)
        ssd.set_wait_limit(200)
        ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=128)
        with pytest.raises(ssd.SSDError) as ei:
            ssd.poll_status()
        assert ei.value.name == "SSD_ERR_TIMEOUT"
        ssd.set_fault_injection(False)
        ssd.set_wait_limit(0)
        # the status word was cleared by the poll and the next call is correct
        y, fs = ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"], chunk=128)
        ssd.poll_status()
    finally:
        ssd.set_fault_injection(False)
        ssd.set_wait_limit(0)
        ssd.set_forward_variant(0)
    yr, fsr = oracle.forward(*inp.f64())
    assert slice_rel_err(to_host_f64(y), yr, 2) < 2e-2
    assert slice_rel_err(to_host_f64(fs), fsr, 1) < 2e-2
