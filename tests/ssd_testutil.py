"""Helpers shared by the tests: device upload of generated inputs, the error
metric (max over (batch, head) slices of ||y_hat - y||_inf / ||y||_inf) and an
elementwise diagnostic that is reported beside it."""
import numpy as np

TOL = {"f32": 1e-4, "bf16": 2e-2}


def slice_rel_err(got: np.ndarray, ref: np.ndarray, head_axis: int) -> float:
    """got/ref [B, ..., H, ...]: max over (b, h) of max|got-ref| / max|ref|."""
    got = np.moveaxis(np.asarray(got, np.float64), head_axis, 1)
    ref = np.moveaxis(np.asarray(ref, np.float64), head_axis, 1)
    B, H = ref.shape[:2]
    diff = np.abs(got - ref).reshape(B, H, -1).max(axis=2)
    mag = np.abs(ref).reshape(B, H, -1).max(axis=2)
    return float((diff / np.maximum(mag, 1e-30)).max())


def elementwise_rel_err(got: np.ndarray, ref: np.ndarray, eps: float = 1e-2) -> float:
    """Diagnostic: max over elements of |got - ref| / (|ref| + eps * rms(ref)),
    which looks at every token rather than at each slice's largest value."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float((np.abs(got - ref) / (np.abs(ref) + eps * rms + 1e-300)).max())


def to_device(inp, device="cuda"):
    """Upload an SSDInputs to torch tensors (bf16 stays bit-exact)."""
    import torch

    def io(a):
        if inp.dtype == "bf16":
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a).to(device)

    return dict(x=io(inp.x), dt=torch.from_numpy(inp.dt).to(device),
                A=torch.from_numpy(inp.A).to(device), Bm=io(inp.Bm), Cm=io(inp.Cm),
                D=torch.from_numpy(inp.D).to(device))


def to_host_f64(t) -> np.ndarray:
    import torch
    return t.detach().to("cpu", torch.float64).numpy()
