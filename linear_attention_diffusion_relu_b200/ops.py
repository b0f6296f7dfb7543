"""Python binding of ``libsana_linattn.so`` (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; this module
checks torch tensors (dtype, shape, contiguity, device), passes raw device
pointers and the current CUDA stream, and raises on any non-OK status. There is
no CPU path: CPU tensors are rejected (except by forward_host, whose host
buffers the library copies to the device itself) and a missing library raises.

The functions mirror the C ABI in ``include/sana_linattn.h``:

    workspace_bytes(B, N, H, d)
    kv_state(K, V, state=None, workspace=None)             -> state (B, H, d, d+1) fp32
    apply(Q, state, out_dtype=torch.bfloat16, eps=1e-15, out=None) -> O (B, N, H, d)
    forward(Q, K, V, out_dtype=torch.bfloat16, eps=1e-15, out=None, workspace=None) -> O

each with ``feature_map="relu" | "elu1" | "cos"`` (the ``*_fm`` entry points),

the forward from and to host memory, copies overlapped by the library:

    forward_host(Q, K, V, out_dtype=..., eps=..., out=None, workspace=None) -> O (CPU)

the state built inside the key-value projection (K and V never stored):

    kv_projection_state(X, Wk, Wv, H, state=None, workspace=None) -> (B, H, d, d+1) fp32

the Mix-FFN that follows the attention in a Sana block:

    mix_ffn(X, W1, Kdw, W2, grid_hw, out=None, workspace=None) -> Y (B, N, C) bf16

and the block-causal form (blocks of L tokens, L a multiple of 128):

    block_causal_workspace_bytes(B, N, H, d, L)
    block_causal_kv_state(K, V, L, states=None, workspace=None) -> (B, H, nblk, d, d+1) fp32
    block_causal_apply(Q, states, L, out_dtype=..., eps=..., out=None) -> O
    block_causal_forward(Q, K, V, L, out_dtype=..., eps=..., out=None, workspace=None,
                         single_launch=False) -> O
    block_causal_forward_host(Q, K, V, L, out_dtype=..., eps=..., out=None, workspace=None) -> O (CPU)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_PKG, "libsana_linattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA = range(5)
OUT_F32, OUT_BF16 = 0, 1
FEATURE_MAPS = {"relu": 0, "elu1": 1, "cos": 2}

SYMBOLS = (
    "sana_linattn_workspace_bytes",
    "sana_linattn_kv_state",
    "sana_linattn_apply",
    "sana_linattn_forward",
    "sana_linattn_forward_launches",
    "sana_linattn_kv_state_fm",
    "sana_linattn_apply_fm",
    "sana_linattn_forward_fm",
    "sana_linattn_mix_ffn_workspace_bytes",
    "sana_linattn_mix_ffn",
    "sana_linattn_mix_ffn_launches",
    "sana_linattn_kv_projection_workspace_bytes",
    "sana_linattn_kv_projection_state",
    "sana_linattn_kv_projection_state_launches",
    "sana_linattn_block_causal_workspace_bytes",
    "sana_linattn_block_causal_kv_state",
    "sana_linattn_block_causal_apply",
    "sana_linattn_block_causal_forward",
    "sana_linattn_block_causal_forward_launches",
    "sana_linattn_block_causal_forward_single",
    "sana_linattn_block_causal_forward_single_launches",
    "sana_linattn_block_causal_forward_host_workspace_bytes",
    "sana_linattn_block_causal_forward_host",
    "sana_linattn_block_causal_forward_host_launches",
    "sana_linattn_forward_host_workspace_bytes",
    "sana_linattn_forward_host",
    "sana_linattn_forward_host_launches",
    "sana_linattn_build_info",
    "sana_linattn_device_error",
    "sana_linattn_selftest_wait_timeout",
    "sana_linattn_status_string",
    "sana_linattn_last_error",
)

_lock = threading.Lock()
_lib = None


class LinAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


def load_library(path: str = LIBRARY) -> ctypes.CDLL:
    """Load the C-ABI library and declare its signatures. Raises if absent."""
    global _lib
    with _lock:
        if _lib is not None and path == LIBRARY:
            return _lib
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build it with "
                "`python -m linear_attention_diffusion_relu_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(path)
        vp, i, sz, f, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_int
        lib.sana_linattn_workspace_bytes.argtypes = [i, i, i, i]
        lib.sana_linattn_workspace_bytes.restype = sz
        lib.sana_linattn_kv_state.argtypes = [vp, vp, i, i, i, i, vp, vp, sz, vp]
        lib.sana_linattn_kv_state.restype = st
        lib.sana_linattn_apply.argtypes = [vp, vp, i, i, i, i, vp, i, f, vp]
        lib.sana_linattn_apply.restype = st
        lib.sana_linattn_forward.argtypes = [vp, vp, vp, i, i, i, i, vp, i, f, vp, sz, vp]
        lib.sana_linattn_forward.restype = st
        lib.sana_linattn_status_string.argtypes = [st]
        lib.sana_linattn_status_string.restype = ctypes.c_char_p
        lib.sana_linattn_forward_launches.argtypes = [i, i, i, i]
        lib.sana_linattn_forward_launches.restype = ctypes.c_int
        lib.sana_linattn_build_info.argtypes = []
        lib.sana_linattn_build_info.restype = ctypes.c_char_p
        lib.sana_linattn_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), i]
        lib.sana_linattn_device_error.restype = st
        lib.sana_linattn_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
        lib.sana_linattn_selftest_wait_timeout.restype = st
        lib.sana_linattn_kv_state_fm.argtypes = [vp, vp, i, i, i, i, i, vp, vp, sz, vp]
        lib.sana_linattn_kv_state_fm.restype = st
        lib.sana_linattn_apply_fm.argtypes = [vp, vp, i, i, i, i, i, vp, i, f, vp]
        lib.sana_linattn_apply_fm.restype = st
        lib.sana_linattn_forward_fm.argtypes = [vp, vp, vp, i, i, i, i, i, vp, i, f, vp, sz, vp]
        lib.sana_linattn_forward_fm.restype = st
        lib.sana_linattn_forward_host_workspace_bytes.argtypes = [i, i, i, i, i]
        lib.sana_linattn_forward_host_workspace_bytes.restype = sz
        lib.sana_linattn_forward_host.argtypes = [vp, vp, vp, i, i, i, i, i, vp, i, f, vp, sz, vp]
        lib.sana_linattn_forward_host.restype = st
        lib.sana_linattn_forward_host_launches.argtypes = [i, i, i, i]
        lib.sana_linattn_forward_host_launches.restype = ctypes.c_int
        lib.sana_linattn_mix_ffn_workspace_bytes.argtypes = [i, i, i, i, i]
        lib.sana_linattn_mix_ffn_workspace_bytes.restype = sz
        lib.sana_linattn_mix_ffn.argtypes = [vp, vp, vp, vp, i, i, i, i, i, vp, vp, sz, vp]
        lib.sana_linattn_mix_ffn.restype = st
        lib.sana_linattn_mix_ffn_launches.argtypes = [i, i, i, i, i]
        lib.sana_linattn_mix_ffn_launches.restype = ctypes.c_int
        lib.sana_linattn_kv_projection_workspace_bytes.argtypes = [i, i, i, i, i]
        lib.sana_linattn_kv_projection_workspace_bytes.restype = sz
        lib.sana_linattn_kv_projection_state.argtypes = [vp, vp, vp, i, i, i, i, i, vp, vp, sz, vp]
        lib.sana_linattn_kv_projection_state.restype = st
        lib.sana_linattn_kv_projection_state_launches.argtypes = [i, i, i, i, i]
        lib.sana_linattn_kv_projection_state_launches.restype = ctypes.c_int
        lib.sana_linattn_block_causal_workspace_bytes.argtypes = [i, i, i, i, i]
        lib.sana_linattn_block_causal_workspace_bytes.restype = sz
        lib.sana_linattn_block_causal_kv_state.argtypes = [vp, vp, i, i, i, i, i, vp, vp, sz, vp]
        lib.sana_linattn_block_causal_kv_state.restype = st
        lib.sana_linattn_block_causal_apply.argtypes = [vp, vp, i, i, i, i, i, vp, i, f, vp]
        lib.sana_linattn_block_causal_apply.restype = st
        lib.sana_linattn_block_causal_forward.argtypes = [vp, vp, vp, i, i, i, i, i, vp, i, f, vp, sz, vp]
        lib.sana_linattn_block_causal_forward.restype = st
        lib.sana_linattn_block_causal_forward_launches.argtypes = [i, i, i, i, i]
        lib.sana_linattn_block_causal_forward_launches.restype = ctypes.c_int
        lib.sana_linattn_block_causal_forward_single.argtypes = [vp, vp, vp, i, i, i, i, i, vp, i, f, vp, sz, vp]
        lib.sana_linattn_block_causal_forward_single.restype = st
        lib.sana_linattn_block_causal_forward_single_launches.argtypes = [i, i, i, i, i]
        lib.sana_linattn_block_causal_forward_single_launches.restype = ctypes.c_int
        lib.sana_linattn_block_causal_forward_host_workspace_bytes.argtypes = [i, i, i, i, i, i]
        lib.sana_linattn_block_causal_forward_host_workspace_bytes.restype = sz
        lib.sana_linattn_block_causal_forward_host.argtypes = [vp, vp, vp, i, i, i, i, i, vp, i, f, vp, sz, vp]
        lib.sana_linattn_block_causal_forward_host.restype = st
        lib.sana_linattn_block_causal_forward_host_launches.argtypes = [i, i, i, i, i]
        lib.sana_linattn_block_causal_forward_host_launches.restype = ctypes.c_int
        lib.sana_linattn_last_error.argtypes = []
        lib.sana_linattn_last_error.restype = ctypes.c_char_p
        if path == LIBRARY:
            _lib = lib
        return lib


def _check(lib, status: int, what: str):
    if status != OK:
        msg = lib.sana_linattn_status_string(status).decode()
        extra = lib.sana_linattn_last_error().decode()
        raise LinAttnError(status, f"{what}: {msg}" + (f" [{extra}]" if extra else ""))


def _out_code(dtype) -> int:
    if dtype == torch.float32:
        return OUT_F32
    if dtype == torch.bfloat16:
        return OUT_BF16
    raise ValueError(f"output dtype must be float32 or bfloat16, got {dtype}")


def _check_bnhd(name, t, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (this library has no CPU path)")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != 4:
        raise ValueError(f"{name} must have shape (B, N, H, d), got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (B, N, H, d) row-major")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} shape {tuple(t.shape)} != {tuple(shape)}")


def _feature_code(feature_map: str) -> int:
    if feature_map not in FEATURE_MAPS:
        raise ValueError(f"feature_map must be one of {sorted(FEATURE_MAPS)}, got {feature_map!r}")
    return FEATURE_MAPS[feature_map]


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def workspace_bytes(B: int, N: int, H: int, d: int) -> int:
    return int(load_library().sana_linattn_workspace_bytes(B, N, H, d))


def forward_launches(B: int, N: int, H: int, d: int) -> int:
    """Kernel launches one forward call enqueues for these sizes."""
    return int(load_library().sana_linattn_forward_launches(B, N, H, d))


def implementation() -> dict:
    """Kernel set compiled into the loaded library, e.g. {"name": ..., "bound": ...}."""
    info = load_library().sana_linattn_build_info().decode()
    kv = dict(part.split("=", 1) for part in info.split(";") if "=" in part)
    return {"name": kv.get("impl", "?"), "bound": kv.get("bound", "hbm"), "raw": info}


def device_error(clear: bool = False) -> int:
    """First error code a kernel recorded on the current device (0 = none).
    Synchronising diagnostic: call after the covered work has completed."""
    lib = load_library()
    code = ctypes.c_uint(0)
    _check(lib, lib.sana_linattn_device_error(ctypes.byref(code), int(clear)),
           "sana_linattn_device_error")
    return int(code.value)


def selftest_wait_timeout(limit_us: int = 20000) -> None:
    """Run the bounded-wait self-test kernel on the current stream (see the header)."""
    lib = load_library()
    _check(lib, lib.sana_linattn_selftest_wait_timeout(int(limit_us), _stream(torch.cuda.current_device())),
           "sana_linattn_selftest_wait_timeout")


def make_workspace(B: int, N: int, H: int, d: int, device="cuda") -> torch.Tensor:
    n = workspace_bytes(B, N, H, d)
    if n == 0:
        raise ValueError(f"unsupported sizes B={B} N={N} H={H} d={d}")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kv_state(K: torch.Tensor, V: torch.Tensor, state: torch.Tensor | None = None,
             workspace: torch.Tensor | None = None, feature_map: str = "relu") -> torch.Tensor:
    """state = phi(K)^T [V | 1] per (b, h), fp32 (B, H, d, d+1)."""
    fm = _feature_code(feature_map)
    _check_bnhd("K", K)
    _check_bnhd("V", V, K.shape)
    B, N, H, d = K.shape
    if state is None:
        state = torch.empty((B, H, d, d + 1), dtype=torch.float32, device=K.device)
    elif (state.dtype != torch.float32 or tuple(state.shape) != (B, H, d, d + 1)
          or not state.is_contiguous() or state.device != K.device):
        raise ValueError("state must be contiguous float32 (B, H, d, d+1) on K's device")
    if workspace is None:
        workspace = make_workspace(B, N, H, d, K.device)
    lib = load_library()
    st = lib.sana_linattn_kv_state_fm(K.data_ptr(), V.data_ptr(), B, N, H, d, fm, state.data_ptr(),
                                      workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                      _stream(K.device))
    _check(lib, st, "sana_linattn_kv_state_fm")
    return state


def _prep_out(out, shape, dtype, device):
    if out is None:
        return torch.empty(shape, dtype=dtype, device=device)
    if tuple(out.shape) != tuple(shape) or out.dtype != dtype or not out.is_contiguous() \
            or out.device != device:
        raise ValueError(f"out must be contiguous {dtype} {tuple(shape)} on {device}")
    return out


def apply(Q: torch.Tensor, state: torch.Tensor, out_dtype=torch.bfloat16, eps: float = 1e-15,
          out: torch.Tensor | None = None, feature_map: str = "relu") -> torch.Tensor:
    """O = (phi(Q) state[..., :d]) / (phi(Q) state[..., d] + eps)."""
    fm = _feature_code(feature_map)
    _check_bnhd("Q", Q)
    B, N, H, d = Q.shape
    if (state.dtype != torch.float32 or tuple(state.shape) != (B, H, d, d + 1)
            or not state.is_contiguous() or state.device != Q.device):
        raise ValueError("state must be contiguous float32 (B, H, d, d+1) on Q's device")
    code = _out_code(out_dtype)
    out = _prep_out(out, Q.shape, out_dtype, Q.device)
    lib = load_library()
    st = lib.sana_linattn_apply_fm(Q.data_ptr(), state.data_ptr(), B, N, H, d, fm, out.data_ptr(), code,
                                   float(eps), _stream(Q.device))
    _check(lib, st, "sana_linattn_apply_fm")
    return out


def forward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, out_dtype=torch.bfloat16,
            eps: float = 1e-15, out: torch.Tensor | None = None,
            workspace: torch.Tensor | None = None, feature_map: str = "relu") -> torch.Tensor:
    """Whole linear-attention forward; bit-identical to kv_state + apply."""
    fm = _feature_code(feature_map)
    _check_bnhd("Q", Q)
    _check_bnhd("K", K, Q.shape)
    _check_bnhd("V", V, Q.shape)
    B, N, H, d = Q.shape
    code = _out_code(out_dtype)
    out = _prep_out(out, Q.shape, out_dtype, Q.device)
    if workspace is None:
        workspace = make_workspace(B, N, H, d, Q.device)
    lib = load_library()
    st = lib.sana_linattn_forward_fm(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, N, H, d, fm,
                                     out.data_ptr(), code, float(eps), workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(), _stream(Q.device))
    _check(lib, st, "sana_linattn_forward_fm")
    return out


def forward_host_workspace_bytes(B: int, N: int, H: int, d: int, out_dtype=torch.bfloat16) -> int:
    return int(load_library().sana_linattn_forward_host_workspace_bytes(B, N, H, d, _out_code(out_dtype)))


def forward_host_launches(B: int, N: int, H: int, d: int) -> int:
    return int(load_library().sana_linattn_forward_host_launches(B, N, H, d))


def forward_host(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, out_dtype=torch.bfloat16,
                 eps: float = 1e-15, out: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, feature_map: str = "relu",
                 device=None) -> torch.Tensor:
    """The forward from host tensors to a host tensor, with the copies done by the
    library (K, V in; the state; Q streamed through in chunks whose outputs are
    copied back while the next chunk comes in). Q, K, V: CPU (B, N, H, d) bf16,
    page-locked for the copies to overlap; out: CPU, allocated page-locked when
    None. Enqueued on the current stream of `device` (default: the current CUDA
    device); the result is ready once that stream is done. Bit-identical to
    forward() on the same inputs."""
    fm = _feature_code(feature_map)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    for name, t in (("Q", Q), ("K", K), ("V", V)):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
            raise ValueError(f"{name} must be a CPU tensor (the device copy is made by the library)")
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous (B, N, H, d) bf16 tensor")
        if t.shape != Q.shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(Q.shape)}")
    B, N, H, d = Q.shape
    code = _out_code(out_dtype)
    if out is None:
        out = torch.empty(Q.shape, dtype=out_dtype).pin_memory()
    elif (out.device.type != "cpu" or out.dtype != out_dtype or tuple(out.shape) != tuple(Q.shape)
          or not out.is_contiguous()):
        raise ValueError(f"out must be a contiguous CPU {out_dtype} tensor of shape {tuple(Q.shape)}")
    if workspace is None:
        n = forward_host_workspace_bytes(B, N, H, d, out_dtype)
        if n == 0:
            raise ValueError(f"unsupported sizes B={B} N={N} H={H} d={d}")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    lib = load_library()
    st = lib.sana_linattn_forward_host(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, N, H, d, fm,
                                       out.data_ptr(), code, float(eps), workspace.data_ptr(),
                                       workspace.numel() * workspace.element_size(), _stream(dev))
    _check(lib, st, "sana_linattn_forward_host")
    return out


def _host_inputs(Q, K, V, out, out_dtype):
    for name, t in (("Q", Q), ("K", K), ("V", V)):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
            raise ValueError(f"{name} must be a CPU tensor (the device copy is made by the library)")
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous (B, N, H, d) bf16 tensor")
        if t.shape != Q.shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(Q.shape)}")
    if out is None:
        return torch.empty(Q.shape, dtype=out_dtype).pin_memory()
    if (out.device.type != "cpu" or out.dtype != out_dtype or tuple(out.shape) != tuple(Q.shape)
            or not out.is_contiguous()):
        raise ValueError(f"out must be a contiguous CPU {out_dtype} tensor of shape {tuple(Q.shape)}")
    return out


# ------------------------------------------------------------ block-causal --

def num_blocks(N: int, L: int) -> int:
    return -(-N // L)


def block_causal_workspace_bytes(B: int, N: int, H: int, d: int, L: int) -> int:
    return int(load_library().sana_linattn_block_causal_workspace_bytes(B, N, H, d, L))


def block_causal_forward_launches(B: int, N: int, H: int, d: int, L: int, single_launch: bool = False) -> int:
    lib = load_library()
    if single_launch:
        return int(lib.sana_linattn_block_causal_forward_single_launches(B, N, H, d, L))
    return int(lib.sana_linattn_block_causal_forward_launches(B, N, H, d, L))


def make_block_causal_workspace(B: int, N: int, H: int, d: int, L: int, device="cuda") -> torch.Tensor:
    n = block_causal_workspace_bytes(B, N, H, d, L)
    if n == 0:
        raise ValueError(f"unsupported sizes B={B} N={N} H={H} d={d} L={L}")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _check_states(states, B, N, H, d, L, device):
    shape = (B, H, num_blocks(N, L), d, d + 1)
    if (states.dtype != torch.float32 or tuple(states.shape) != shape
            or not states.is_contiguous() or states.device != device):
        raise ValueError(f"states must be contiguous float32 {shape} on {device}")


def block_causal_kv_state(K: torch.Tensor, V: torch.Tensor, L: int, states: torch.Tensor | None = None,
                          workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Inclusive prefix states over blocks of L tokens, fp32 (B, H, nblk, d, d+1)."""
    _check_bnhd("K", K)
    _check_bnhd("V", V, K.shape)
    B, N, H, d = K.shape
    if states is None:
        states = torch.empty((B, H, num_blocks(N, L), d, d + 1), dtype=torch.float32, device=K.device)
    _check_states(states, B, N, H, d, L, K.device)
    if workspace is None:
        workspace = make_block_causal_workspace(B, N, H, d, L, K.device)
    lib = load_library()
    st = lib.sana_linattn_block_causal_kv_state(K.data_ptr(), V.data_ptr(), B, N, H, d, int(L),
                                                states.data_ptr(), workspace.data_ptr(),
                                                workspace.numel() * workspace.element_size(),
                                                _stream(K.device))
    _check(lib, st, "sana_linattn_block_causal_kv_state")
    return states


def block_causal_apply(Q: torch.Tensor, states: torch.Tensor, L: int, out_dtype=torch.bfloat16,
                       eps: float = 1e-15, out: torch.Tensor | None = None) -> torch.Tensor:
    """O for block-causal attention: row n uses the prefix state of block n // L."""
    _check_bnhd("Q", Q)
    B, N, H, d = Q.shape
    _check_states(states, B, N, H, d, L, Q.device)
    code = _out_code(out_dtype)
    out = _prep_out(out, Q.shape, out_dtype, Q.device)
    lib = load_library()
    st = lib.sana_linattn_block_causal_apply(Q.data_ptr(), states.data_ptr(), B, N, H, d, int(L),
                                             out.data_ptr(), code, float(eps), _stream(Q.device))
    _check(lib, st, "sana_linattn_block_causal_apply")
    return out


def block_causal_forward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, L: int,
                         out_dtype=torch.bfloat16, eps: float = 1e-15, out: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None, single_launch: bool = False) -> torch.Tensor:
    """Whole block-causal forward; bit-identical to block_causal_kv_state + block_causal_apply.
    single_launch: the one-launch form (sana_linattn_block_causal_forward_single)."""
    _check_bnhd("Q", Q)
    _check_bnhd("K", K, Q.shape)
    _check_bnhd("V", V, Q.shape)
    B, N, H, d = Q.shape
    code = _out_code(out_dtype)
    out = _prep_out(out, Q.shape, out_dtype, Q.device)
    if workspace is None:
        workspace = make_block_causal_workspace(B, N, H, d, L, Q.device)
    lib = load_library()
    name = "sana_linattn_block_causal_forward" + ("_single" if single_launch else "")
    st = getattr(lib, name)(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, N, H, d, int(L), out.data_ptr(), code,
                            float(eps), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                            _stream(Q.device))
    _check(lib, st, name)
    return out


def block_causal_forward_host_workspace_bytes(B: int, N: int, H: int, d: int, L: int,
                                             out_dtype=torch.bfloat16) -> int:
    return int(load_library().sana_linattn_block_causal_forward_host_workspace_bytes(
        B, N, H, d, int(L), _out_code(out_dtype)))


def block_causal_forward_host_launches(B: int, N: int, H: int, d: int, L: int) -> int:
    return int(load_library().sana_linattn_block_causal_forward_host_launches(B, N, H, d, int(L)))


def block_causal_forward_host(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, L: int,
                              out_dtype=torch.bfloat16, eps: float = 1e-15, out: torch.Tensor | None = None,
                              workspace: torch.Tensor | None = None, device=None) -> torch.Tensor:
    """The block-causal forward from host tensors to a host tensor, with the
    copies done by the library (K, V in; the prefix states; Q streamed through
    in chunks of whole blocks whose outputs are copied back while the next chunk
    comes in). Bit-identical to block_causal_forward() on the same inputs."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = _host_inputs(Q, K, V, out, out_dtype)
    B, N, H, d = Q.shape
    code = _out_code(out_dtype)
    if workspace is None:
        n = block_causal_forward_host_workspace_bytes(B, N, H, d, L, out_dtype)
        if n == 0:
            raise ValueError(f"unsupported sizes B={B} N={N} H={H} d={d} L={L}")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    lib = load_library()
    st = lib.sana_linattn_block_causal_forward_host(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, N, H, d, int(L),
                                                    out.data_ptr(), code, float(eps), workspace.data_ptr(),
                                                    workspace.numel() * workspace.element_size(), _stream(dev))
    _check(lib, st, "sana_linattn_block_causal_forward_host")
    return out


# ------------------------------------------------ key-value projection + state --

def kv_projection_workspace_bytes(B: int, N: int, C: int, H: int, d: int) -> int:
    return int(load_library().sana_linattn_kv_projection_workspace_bytes(B, N, C, H, d))


def kv_projection_state(X: torch.Tensor, Wk: torch.Tensor, Wv: torch.Tensor, H: int,
                        state: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None) -> torch.Tensor:
    """state = phi(K)^T [V | 1] with K = bf16(X Wk^T), V = bf16(X Wv^T), computed
    without storing K or V. X bf16 (B, N, C); Wk, Wv bf16 (H*d, C)."""
    for name, t in (("X", X), ("Wk", Wk), ("Wv", Wv)):
        if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
            raise ValueError(f"{name} must be a CUDA tensor (this library has no CPU path)")
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous bfloat16")
    if X.dim() != 3:
        raise ValueError(f"X must have shape (B, N, C), got {tuple(X.shape)}")
    B, N, C = X.shape
    if Wk.dim() != 2 or Wk.shape[1] != C or Wk.shape[0] % H or tuple(Wv.shape) != tuple(Wk.shape):
        raise ValueError("Wk and Wv must both have shape (H*d, C)")
    d = Wk.shape[0] // H
    if state is None:
        state = torch.empty((B, H, d, d + 1), dtype=torch.float32, device=X.device)
    elif (state.dtype != torch.float32 or tuple(state.shape) != (B, H, d, d + 1)
          or not state.is_contiguous() or state.device != X.device):
        raise ValueError("state must be contiguous float32 (B, H, d, d+1) on X's device")
    if workspace is None:
        n = kv_projection_workspace_bytes(B, N, C, H, d)
        if n == 0:
            raise ValueError(f"unsupported sizes B={B} N={N} C={C} H={H} d={d}")
        workspace = torch.empty(n, dtype=torch.uint8, device=X.device)
    lib = load_library()
    st = lib.sana_linattn_kv_projection_state(X.data_ptr(), Wk.data_ptr(), Wv.data_ptr(), B, N, C, H, d,
                                              state.data_ptr(), workspace.data_ptr(),
                                              workspace.numel() * workspace.element_size(), _stream(X.device))
    _check(lib, st, "sana_linattn_kv_projection_state")
    return state


# ---------------------------------------------------------------------- Mix-FFN --

def mix_ffn_workspace_bytes(B: int, Hg: int, Wg: int, C: int, Ch: int) -> int:
    return int(load_library().sana_linattn_mix_ffn_workspace_bytes(B, Hg, Wg, C, Ch))


def mix_ffn(X: torch.Tensor, W1: torch.Tensor, Kdw: torch.Tensor, W2: torch.Tensor, grid_hw,
            out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Y = (a * sigmoid(g)) W2^T with [a | g] = depthwise3x3(X W1^T) over the token
    grid. X bf16 (B, Hg*Wg, C); W1 bf16 (2*Ch, C); Kdw fp32 (2*Ch, 3, 3); W2 bf16 (C, Ch)."""
    for name, t, dt in (("X", X, torch.bfloat16), ("W1", W1, torch.bfloat16), ("Kdw", Kdw, torch.float32),
                        ("W2", W2, torch.bfloat16)):
        if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
            raise ValueError(f"{name} must be a CUDA tensor (this library has no CPU path)")
        if t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous {dt}")
    Hg, Wg = grid_hw
    B, N, C = X.shape
    Ch2 = W1.shape[0]
    if N != Hg * Wg or W1.shape != (Ch2, C) or Ch2 % 2 or tuple(Kdw.shape) != (Ch2, 3, 3) \
            or tuple(W2.shape) != (C, Ch2 // 2):
        raise ValueError("shapes do not match: X (B, Hg*Wg, C), W1 (2Ch, C), Kdw (2Ch, 3, 3), W2 (C, Ch)")
    Ch = Ch2 // 2
    out = _prep_out(out, (B, N, C), torch.bfloat16, X.device)
    if workspace is None:
        n = mix_ffn_workspace_bytes(B, Hg, Wg, C, Ch)
        if n == 0:
            raise ValueError(f"unsupported sizes B={B} grid={grid_hw} C={C} Ch={Ch}")
        workspace = torch.empty(n, dtype=torch.uint8, device=X.device)
    lib = load_library()
    st = lib.sana_linattn_mix_ffn(X.data_ptr(), W1.data_ptr(), Kdw.data_ptr(), W2.data_ptr(), B, Hg, Wg, C, Ch,
                                  out.data_ptr(), workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(), _stream(X.device))
    _check(lib, st, "sana_linattn_mix_ffn")
    return out
