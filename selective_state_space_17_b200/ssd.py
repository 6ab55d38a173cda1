"""ctypes binding of libssd_b200.so (see include/ssd.h for the contracts).

Argument marshalling only: every step of the SSD computation runs in the CUDA
library. PyTorch supplies device memory and the current stream. The library
must have been built (``python -m selective_state_space_17_b200.build``);
there is no fallback, so a missing library raises at import.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libssd_b200.so")

if not os.path.exists(library_path):
    raise ImportError(
        f"{library_path} is missing: build it with `python -m selective_state_space_17_b200.build`"
        " (the SSD layer has no CPU or Python fallback)")

lib = ctypes.CDLL(library_path)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

lib.ssd_status_string.argtypes = [_i]
lib.ssd_status_string.restype = ctypes.c_char_p
lib.ssd_workspace_size.argtypes = [_i] * 8
lib.ssd_workspace_size.restype = _sz
lib.ssd_forward.argtypes = [_vp] * 9 + [_i] * 8 + [_vp, _sz, _vp]
lib.ssd_forward.restype = _i
lib.ssd_forward_host_buffer_size.argtypes = [_i] * 8
lib.ssd_forward_host_buffer_size.restype = _sz
lib.ssd_forward_host.argtypes = [_vp] * 9 + [_i] * 8 + [_vp, _sz, _vp]
lib.ssd_forward_host.restype = _i
lib.ssd_step.argtypes = [_vp] * 8 + [_i] * 6 + [_vp]
lib.ssd_step.restype = _i
lib.ssd_poll_status.argtypes = [_vp]
lib.ssd_poll_status.restype = _i
lib.ssd_forward_kernel_count.argtypes = [_i] * 8
lib.ssd_forward_kernel_count.restype = _i
lib.ssd_forward_path.argtypes = [_i] * 8
lib.ssd_forward_path.restype = _i
lib.ssd_set_fault_injection.argtypes = [_i]
lib.ssd_set_fault_injection.restype = None
lib.ssd_set_wait_limit.argtypes = [ctypes.c_uint64]
lib.ssd_set_wait_limit.restype = None
lib.ssd_set_forward_variant.argtypes = [_i]
lib.ssd_set_forward_variant.restype = None

SSD_F32, SSD_BF16 = 0, 1
STATUS = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED",
          3: "SSD_ERR_MISALIGNED", 4: "SSD_ERR_CUDA", 5: "SSD_ERR_TIMEOUT",
          6: "SSD_ERR_WORKSPACE"}


class SSDError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.name = STATUS.get(code, f"status {code}")
        super().__init__(f"{where}: {lib.ssd_status_string(code).decode()}")


def _check(code: int, where: str) -> None:
    if code != 0:
        raise SSDError(code, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    if t.dtype == torch.float32:
        return SSD_F32
    raise TypeError(f"I/O dtype must be bfloat16 or float32, got {t.dtype}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t, name, dtype=None, device=None, shape=None, cuda=True):
    """Checks one tensor argument before anything reaches the library: a host
    tensor handed to a device entry point (or the reverse) would otherwise
    become a wild pointer inside a kernel."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (got one on {t.device})")
    if not cuda and t.is_cuda:
        raise ValueError(f"{name} must be a host tensor (got one on {t.device})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _dims4(x, name):
    if x.dim() != 4:
        raise ValueError(f"{name} must be [B, L, H, P], got shape {tuple(x.shape)}")
    return tuple(x.shape)


_ws_lock = threading.Lock()
_ws_cache: dict = {}


def workspace_size(B, L, H, P, G, N, chunk, dtype_code) -> int:
    return int(lib.ssd_workspace_size(B, L, H, P, G, N, chunk, dtype_code))


def _workspace(device, nbytes: int, stream_handle: int) -> torch.Tensor:
    """A workspace of at least nbytes, cached per (device, stream): calls on
    one stream are ordered and may share it (the library tags the control words
    it keeps there with the call, so no clearing is needed); calls on two
    streams may overlap on the GPU, so each stream gets its own."""
    dev_index = device.index if device.index is not None else torch.cuda.current_device()
    key = (dev_index, stream_handle)
    with _ws_lock:
        ws = _ws_cache.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
            _ws_cache[key] = ws
    return ws


def forward(x, dt, A, Bm, Cm, D=None, chunk: int = 256, initial_state=None, y=None,
            final_state=None, return_final_state: bool = True, workspace=None, stream=None):
    """SSD forward on CUDA tensors. x[B,L,H,P], dt[B,L,H] f32, A[H] f32,
    Bm/Cm[B,L,G,N], D[H] f32 or None, initial_state[B,H,P,N] f32 or None.
    Returns (y, final_state) (final_state None if not requested).

    The call is asynchronous on `stream`. A device-side wait that gives up
    (the per-head kernel's look-back when other work keeps some of its CTAs off
    the SMs for seconds, or a test's fault injection) leaves y and final_state
    undefined and records it in the stream's status word: poll_status() at a
    synchronisation point raises SSDError then."""
    _need(x, "x")
    dev = x.device
    code = _dtype_code(x)
    Bsz, L, H, P = _dims4(x, "x")
    _need(Bm, "Bm", x.dtype, dev)
    if Bm.dim() != 4:
        raise ValueError(f"Bm must be [B, L, G, N], got shape {tuple(Bm.shape)}")
    G, N = Bm.shape[2], Bm.shape[3]
    _need(Bm, "Bm", shape=(Bsz, L, G, N))
    _need(Cm, "Cm", x.dtype, dev, (Bsz, L, G, N))
    _need(dt, "dt", torch.float32, dev, (Bsz, L, H))
    _need(A, "A", torch.float32, dev, (H,))
    if D is not None:
        _need(D, "D", torch.float32, dev, (H,))
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, dev, (Bsz, H, P, N))
    if y is None:
        y = torch.empty_like(x)
    else:
        _need(y, "y", x.dtype, dev, (Bsz, L, H, P))
    if final_state is None and return_final_state:
        final_state = torch.empty((Bsz, H, P, N), dtype=torch.float32, device=dev)
    elif final_state is not None:
        _need(final_state, "final_state", torch.float32, dev, (Bsz, H, P, N))
    nbytes = workspace_size(Bsz, L, H, P, G, N, chunk, code)
    if nbytes == 0:
        raise SSDError(1, "ssd_workspace_size")
    sh = _stream_handle(stream)
    if workspace is None:
        workspace = _workspace(dev, nbytes, sh)
    else:
        _need(workspace, "workspace", device=dev)
    rc = lib.ssd_forward(_ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                         _ptr(initial_state), _ptr(y), _ptr(final_state),
                         Bsz, L, H, P, G, N, chunk, code, _ptr(workspace),
                         workspace.numel() * workspace.element_size(), sh)
    _check(rc, "ssd_forward")
    return y, final_state


def kernel_count(B, L, H, P, G, N, chunk, dtype_code) -> int:
    """Kernels one forward call with these sizes launches (host-side query)."""
    return int(lib.ssd_forward_kernel_count(B, L, H, P, G, N, chunk, dtype_code))


def forward_path(B, L, H, P, G, N, chunk, dtype_code) -> int:
    """Path of one forward call with these sizes (host-side query): 0 invalid or
    empty, 1 SIMT, 2 per-head tensor-core single pass, 3 its segment-parallel
    form, 4 head-group tensor-core kernel."""
    return int(lib.ssd_forward_path(B, L, H, P, G, N, chunk, dtype_code))


def forward_host_buffer_size(B, L, H, P, G, N, chunk, dtype_code) -> int:
    return int(lib.ssd_forward_host_buffer_size(B, L, H, P, G, N, chunk, dtype_code))


def forward_host(x, dt, A, Bm, Cm, D, y, final_state=None, initial_state=None, chunk: int = 256,
                 device_buffer=None, stream=None):
    """SSD forward on HOST tensors (pinned for asynchronous copies): the library
    copies the inputs in, runs the forward, copies y / final_state out and
    synchronises the stream. Shapes as ``forward``; y (and final_state) are
    caller-provided host tensors that receive the result."""
    _need(x, "x", cuda=False)
    code = _dtype_code(x)
    Bsz, L, H, P = _dims4(x, "x")
    _need(Bm, "Bm", x.dtype, cuda=False)
    if Bm.dim() != 4:
        raise ValueError(f"Bm must be [B, L, G, N], got shape {tuple(Bm.shape)}")
    G, N = Bm.shape[2], Bm.shape[3]
    _need(Bm, "Bm", shape=(Bsz, L, G, N), cuda=False)
    _need(Cm, "Cm", x.dtype, shape=(Bsz, L, G, N), cuda=False)
    _need(dt, "dt", torch.float32, shape=(Bsz, L, H), cuda=False)
    _need(A, "A", torch.float32, shape=(H,), cuda=False)
    if D is not None:
        _need(D, "D", torch.float32, shape=(H,), cuda=False)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, shape=(Bsz, H, P, N), cuda=False)
    _need(y, "y", x.dtype, shape=(Bsz, L, H, P), cuda=False)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, shape=(Bsz, H, P, N), cuda=False)
    need = forward_host_buffer_size(Bsz, L, H, P, G, N, chunk, code)
    if need == 0:
        raise SSDError(1, "ssd_forward_host_buffer_size")
    if device_buffer is None:
        device_buffer = torch.zeros(need, dtype=torch.uint8, device="cuda")
    else:
        _need(device_buffer, "device_buffer")
    rc = lib.ssd_forward_host(_ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                              _ptr(initial_state), _ptr(y), _ptr(final_state),
                              Bsz, L, H, P, G, N, chunk, code, _ptr(device_buffer),
                              device_buffer.numel() * device_buffer.element_size(),
                              _stream_handle(stream))
    _check(rc, "ssd_forward_host")
    return y, final_state


def step(x, dt, A, Bm, Cm, D, state, y=None, stream=None):
    """One decode step; ``state`` [B,H,P,N] f32 is updated in place. Returns y."""
    _need(x, "x")
    dev = x.device
    code = _dtype_code(x)
    if x.dim() != 3:
        raise ValueError(f"x must be [B, H, P], got shape {tuple(x.shape)}")
    Bsz, H, P = x.shape
    _need(Bm, "Bm", x.dtype, dev)
    if Bm.dim() != 3:
        raise ValueError(f"Bm must be [B, G, N], got shape {tuple(Bm.shape)}")
    G, N = Bm.shape[1], Bm.shape[2]
    _need(Bm, "Bm", shape=(Bsz, G, N))
    _need(Cm, "Cm", x.dtype, dev, (Bsz, G, N))
    _need(dt, "dt", torch.float32, dev, (Bsz, H))
    _need(A, "A", torch.float32, dev, (H,))
    if D is not None:
        _need(D, "D", torch.float32, dev, (H,))
    _need(state, "state", torch.float32, dev, (Bsz, H, P, N))
    if y is None:
        y = torch.empty_like(x)
    else:
        _need(y, "y", x.dtype, dev, (Bsz, H, P))
    rc = lib.ssd_step(_ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(state),
                      _ptr(y), Bsz, H, P, G, N, code, _stream_handle(stream))
    _check(rc, "ssd_step")
    return y


def poll_status(stream=None) -> None:
    """Synchronise and raise SSDError if a device-side wait gave up."""
    _check(lib.ssd_poll_status(_stream_handle(stream)), "ssd_poll_status")


def set_wait_limit(iterations: int) -> None:
    """Iteration limit of device-side look-back waits (0 restores the default)."""
    lib.ssd_set_wait_limit(int(iterations))


def set_fault_injection(skip_publish: bool) -> None:
    """Test hook: tiles stop publishing end states (see include/ssd.h)."""
    lib.ssd_set_fault_injection(1 if skip_publish else 0)


def set_forward_variant(variant: int) -> None:
    """Test hook: 0 automatic, 1 per-head tensor-core kernel, 2 head-group
    tensor-core kernel (see include/ssd.h)."""
    lib.ssd_set_forward_variant(int(variant))
