"""The Python binding rejects bad tensor arguments before anything reaches the
library (no GPU needed: every case fails validation first). A host tensor given
to a device entry point would otherwise become a wild pointer in a kernel."""
import pytest

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ssd():
    from selective_state_space_17_b200 import build
    build.build()
    from selective_state_space_17_b200 import ssd as _ssd
    return _ssd


def _host_inputs(B=1, L=64, H=2, P=64, G=1, N=16, dtype=torch.bfloat16):
    return dict(x=torch.zeros(B, L, H, P, dtype=dtype), dt=torch.zeros(B, L, H),
                A=torch.zeros(H), Bm=torch.zeros(B, L, G, N, dtype=dtype),
                Cm=torch.zeros(B, L, G, N, dtype=dtype), D=torch.zeros(H))


def test_forward_rejects_host_tensors(ssd):
    t = _host_inputs()
    with pytest.raises(ValueError, match="CUDA"):
        ssd.forward(t["x"], t["dt"], t["A"], t["Bm"], t["Cm"], t["D"])


def test_step_rejects_host_tensors(ssd):
    x = torch.zeros(2, 2, 64, dtype=torch.bfloat16)
    Bm = torch.zeros(2, 1, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ssd.step(x, torch.zeros(2, 2), torch.zeros(2), Bm, Bm, None, torch.zeros(2, 2, 64, 16))


def test_forward_host_checks_shapes_dtypes_and_layout(ssd):
    t = _host_inputs()
    y = torch.empty_like(t["x"])
    ok = dict(t)
    with pytest.raises(ValueError, match="y must have shape"):
        ssd.forward_host(**ok, y=torch.empty(1, 64, 2, 32, dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="dt must be torch.float32"):
        ssd.forward_host(**dict(ok, dt=ok["dt"].double()), y=y)
    with pytest.raises(ValueError, match="A must have shape"):
        ssd.forward_host(**dict(ok, A=torch.zeros(3)), y=y)
    with pytest.raises(ValueError, match="contiguous"):
        ssd.forward_host(**dict(ok, x=torch.zeros(1, 64, 64, 2, dtype=torch.bfloat16).transpose(2, 3)),
                         y=y)
    with pytest.raises(TypeError, match="Cm must be torch.bfloat16"):
        ssd.forward_host(**dict(ok, Cm=ok["Cm"].float()), y=y)
    with pytest.raises(ValueError, match="final_state must have shape"):
        ssd.forward_host(**ok, y=y, final_state=torch.zeros(1, 2, 64, 8))
    with pytest.raises(ValueError, match=r"x must be \[B, L, H, P\]"):
        ssd.forward_host(**dict(ok, x=ok["x"][0]), y=y)


def test_io_dtype_must_be_bf16_or_fp32(ssd):
    t = _host_inputs(dtype=torch.float16)
    with pytest.raises(TypeError, match="bfloat16 or float32"):
        ssd.forward_host(**t, y=torch.empty_like(t["x"]))
