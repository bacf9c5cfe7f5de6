"""Block-causal ReLU linear attention with numerator-only 3D RoPE on B200.

Python binding of ``libblin.so`` (C ABI declared in ``include/blin.h``).  This
module only marshals arguments: every step of the computation runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current stream.

    import block_causal_linear_rope_b200 as blin
    o = blin.prefill(q, k, v, grid=(T, Hg, Wg), block_frames=3, rope_split=(8, 12, 12))
    st = blin.BlockState(B, H, d)
    o_b = blin.block_step(q_b, k_b, v_b, Hg, Wg, frames=3, rope_split=(8, 12, 12), state=st)

Tensors are contiguous [B, H, N, d] (d = 32 or 64) in float32 or bfloat16 on
the current CUDA device.  If the library is missing this import raises: there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

__all__ = ["BlinError", "BlockState", "TConvState", "tconv", "Layout", "prefill", "prefill_nvfp4", "block_step_nvfp4",
           "Nvfp4Tensor", "block_step", "workspace_size", "device_status",
           "last_path", "LaunchTimer", "KERNELS", "lib", "LIB_PATH", "F32", "BF16"]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libblin.so")

F32, BF16 = 0, 1
_STATUS = {0: "BLIN_OK", -1: "BLIN_ERR_INVALID_ARG", -2: "BLIN_ERR_SHAPE", -3: "BLIN_ERR_DTYPE",
           -4: "BLIN_ERR_ALIGN", -5: "BLIN_ERR_WORKSPACE", -6: "BLIN_ERR_STATE", -7: "BLIN_ERR_CUDA",
           -8: "BLIN_ERR_DEVICE"}


class Layout(ctypes.Structure):
    _fields_ = [("token", ctypes.c_longlong), ("head", ctypes.c_longlong), ("batch", ctypes.c_longlong)]


class Nvfp4(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("global_scale", ctypes.c_float)]


class BlinError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class Geom(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("Hgt", ctypes.c_int), ("Wid", ctypes.c_int),
                ("block_frames", ctypes.c_int), ("rope_split", ctypes.c_int * 3),
                ("theta", ctypes.c_float), ("eps", ctypes.c_float)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python block_causal_linear_rope_b200/build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    L.blin_state_init.argtypes = [I, I, I, P, ctypes.POINTER(P)]
    L.blin_state_free.argtypes = [P]
    L.blin_state_reset.argtypes = [P, P]
    L.blin_state_tensors.argtypes = [P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(I)]
    L.blin_state_bytes.argtypes = [P]
    L.blin_state_bytes.restype = S
    L.blin_state_copy_to_host.argtypes = [P, P, S, P]
    L.blin_state_copy_from_host.argtypes = [P, P, S, I, P]
    L.blin_state_reserve.argtypes = [P, ctypes.c_long, P]
    L.blin_prefill_workspace_size.argtypes = [I, I, I, ctypes.POINTER(Geom)]
    L.blin_prefill_workspace_size.restype = S
    L.blin_prefill.argtypes = [P, P, P, P, I, I, I, I, ctypes.POINTER(Geom), P, P, S, P]
    L.blin_block_step.argtypes = [P, P, P, P, I, I, I, I, ctypes.POINTER(Geom), P, I, P]
    LP = ctypes.POINTER(Layout)
    L.blin_prefill_strided.argtypes = [P, P, P, P, I, I, I, I, ctypes.POINTER(Geom), LP, LP, P, P, S, P]
    L.blin_prefill_strided.restype = I
    L.blin_block_step_strided.argtypes = [P, P, P, P, I, I, I, I, ctypes.POINTER(Geom), LP, LP, P, I, P]
    L.blin_block_step_strided.restype = I
    L.blin_last_path.argtypes = []
    L.blin_last_path.restype = I
    L.blin_last_error.restype = ctypes.c_char_p
    L.blin_device_status.argtypes = [ctypes.POINTER(I)]
    L.blin_version.restype = ctypes.c_char_p
    L.blin_set_timing_events.argtypes = [P, I]
    L.blin_set_timing_events.restype = I
    L.blin_prefill_static.argtypes = [P, P, P, P, I, I, I, I, ctypes.POINTER(Geom), P, P]
    L.blin_prefill_static.restype = I
    L.blin_prefill_static_capacity.argtypes = []
    L.blin_prefill_static_capacity.restype = S
    NP_ = ctypes.POINTER(Nvfp4)
    L.blin_prefill_nvfp4.argtypes = [NP_, NP_, NP_, P, I, I, I, ctypes.POINTER(Geom), P, P, S, P]
    L.blin_prefill_nvfp4.restype = I
    L.blin_block_step_nvfp4.argtypes = [NP_, NP_, NP_, P, I, I, I, ctypes.POINTER(Geom), P, I, P]
    L.blin_block_step_nvfp4.restype = I
    L.blin_tconv_state_init.argtypes = [I, I, I, I, I, P, ctypes.POINTER(P)]
    L.blin_tconv_state_free.argtypes = [P]
    L.blin_tconv_state_reset.argtypes = [P, P]
    L.blin_tconv_state_frame.argtypes = [P, ctypes.POINTER(P), ctypes.POINTER(I)]
    L.blin_tconv_state_bytes.argtypes = [P]
    L.blin_tconv_state_bytes.restype = S
    L.blin_tconv.argtypes = [P, P, P, P, I, I, I, ctypes.POINTER(Geom), P, I, P]
    for fn in ("blin_tconv_state_init", "blin_tconv_state_free", "blin_tconv_state_reset", "blin_tconv_state_frame",
               "blin_tconv"):
        getattr(L, fn).restype = I
    L.blin_launch_count.argtypes = []
    L.blin_launch_count.restype = ctypes.c_ulonglong
    for fn in ("blin_state_init", "blin_state_free", "blin_state_reset", "blin_state_tensors",
               "blin_state_copy_to_host", "blin_state_copy_from_host", "blin_state_reserve",
               "blin_prefill", "blin_block_step", "blin_device_status"):
        getattr(L, fn).restype = I
    return L


lib = _load()


def _check(status: int) -> None:
    if status != 0:
        raise BlinError(status, lib.blin_last_error().decode())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _geom(T, Hg, Wg, block_frames, rope_split, theta, eps) -> Geom:
    g = Geom()
    g.T, g.Hgt, g.Wid, g.block_frames = int(T), int(Hg), int(Wg), int(block_frames)
    g.rope_split[:] = [int(x) for x in rope_split]
    g.theta, g.eps = float(theta), float(eps)
    return g


class BlockState:
    """Constant-size (S, z) cache: S [B,H,d,d], z [B,H,d] fp32 on one device."""

    def __init__(self, B: int, H: int, d: int, stream=None):
        self.B, self.H, self.d = B, H, d
        h = ctypes.c_void_p()
        _check(lib.blin_state_init(B, H, d, _stream(stream), ctypes.byref(h)))
        self._h = h

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise BlinError(-6, "state already freed")
        return self._h

    def free(self) -> None:
        if self._h is not None:
            _check(lib.blin_state_free(self._h))
            self._h = None

    def __del__(self):
        try:
            if getattr(self, "_h", None) is not None:
                lib.blin_state_free(self._h)
        except Exception:
            pass

    @property
    def t_next(self) -> int:
        t = ctypes.c_int()
        _check(lib.blin_state_tensors(self.handle, None, None, ctypes.byref(t)))
        return t.value

    @property
    def nbytes(self) -> int:
        return int(lib.blin_state_bytes(self.handle))

    def reset(self, stream=None) -> None:
        _check(lib.blin_state_reset(self.handle, _stream(stream)))

    def reserve(self, max_block_tokens: int, stream=None) -> None:
        _check(lib.blin_state_reserve(self.handle, int(max_block_tokens), _stream(stream)))

    def to_host(self, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
        """Copy (S, z) into new pinned host tensors (synchronises the stream)."""
        buf = torch.empty(self.nbytes // 4, dtype=torch.float32, pin_memory=True)
        s = stream or torch.cuda.current_stream()
        _check(lib.blin_state_copy_to_host(self.handle, ctypes.c_void_p(buf.data_ptr()), self.nbytes,
                                           _stream(s)))
        s.synchronize()
        n = self.B * self.H * self.d * self.d
        return (buf[:n].view(self.B, self.H, self.d, self.d).clone(),
                buf[n:].view(self.B, self.H, self.d).clone())

    def from_host(self, S: torch.Tensor, z: torch.Tensor, t_next: int, stream=None) -> None:
        """Restore (S, z) and t_next from host tensors (checkpoint resume)."""
        buf = torch.cat([S.reshape(-1), z.reshape(-1)]).to(torch.float32).contiguous().pin_memory()
        s = stream or torch.cuda.current_stream()
        _check(lib.blin_state_copy_from_host(self.handle, ctypes.c_void_p(buf.data_ptr()),
                                             buf.numel() * 4, int(t_next), _stream(s)))
        s.synchronize()


def _check_qkv(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dim() != 4 or t.stride(3) != 1:
            raise ValueError(f"{name} must be a [B, H, N, d] tensor with d contiguous")
    if not (q.shape == k.shape == v.shape and q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k and v must share shape and dtype")
    if not (q.stride() == k.stride() == v.stride()):
        raise ValueError("q, k and v must share strides (one layout for the three)")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k and v must be on one device")
    _check_device(q)


def _check_device(t: torch.Tensor) -> None:
    """The library launches on the current device: the call's tensors must live there."""
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {t.device} but the current device is cuda:{torch.cuda.current_device()}; "
                         "call under torch.cuda.device(...)")


def _check_out(out, shape, dtype, device, contiguous: bool = False) -> None:
    """A caller-given output must match the call (the library cannot see its extent)."""
    if (not isinstance(out, torch.Tensor) or out.device != device or out.dtype != dtype
            or tuple(out.shape) != tuple(shape) or out.stride(-1) != 1 or (contiguous and not out.is_contiguous())):
        what = "contiguous " if contiguous else ""
        raise ValueError(f"out must be a {what}{dtype} tensor of shape {tuple(shape)} on {device}, last dimension "
                         "contiguous")


def _check_no_overlap(out: torch.Tensor, *inputs: torch.Tensor) -> None:
    """The output must not overlap an input (the kernels read inputs after writing outputs).
    Contiguous tensors are compared by address range; strided views, which may interleave
    without sharing an element, only by start address."""
    def span(t):
        return t.data_ptr(), t.data_ptr() + t.numel() * t.element_size()
    for t in inputs:
        if out.data_ptr() == t.data_ptr():
            raise ValueError("out must not overlap the inputs")
        if out.is_contiguous() and t.is_contiguous():
            (a0, a1), (b0, b1) = span(out), span(t)
            if a0 < b1 and b0 < a1:
                raise ValueError("out must not overlap the inputs")


def _workspace_arg(workspace, need: int, device):
    """(pointer, bytes) of a caller-given workspace, or of a new one of `need` bytes."""
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    elif not isinstance(workspace, torch.Tensor) or workspace.device != device or not workspace.is_contiguous():
        raise ValueError(f"workspace must be a contiguous tensor on {device}")
    return workspace, ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()


def _layouts(q: torch.Tensor, out: torch.Tensor):
    """(qkv layout, o layout) for the strided entry points, or None when all are contiguous."""
    if q.is_contiguous() and out.is_contiguous():
        return None
    lay = lambda t: Layout(t.stride(2), t.stride(1), t.stride(0))
    return lay(q), lay(out)


def workspace_size(B: int, H: int, d: int, grid: Sequence[int], block_frames: int,
                   rope_split: Sequence[int], theta: float = 1e4, eps: float = 1e-6) -> int:
    g = _geom(*grid, block_frames, rope_split, theta, eps)
    n = int(lib.blin_prefill_workspace_size(B, H, d, ctypes.byref(g)))
    if n == 0:
        raise ValueError("invalid shape for blin_prefill")
    return n


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid: Sequence[int], block_frames: int,
            rope_split: Sequence[int], theta: float = 1e4, eps: float = 1e-6,
            state: Optional[BlockState] = None, out: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Block-causal linear attention over the frames grid=(T, Hg, Wg) (N = T*Hg*Wg).

    q, k, v are [B, H, N, d] views with d contiguous; they may be strided (for
    instance the q/k/v slices of a fused [B, N, 3, H, d] projection output, seen
    as [B, H, N, d]) as long as the three share one layout.  `out` may be a
    strided view too (default: a new contiguous tensor)."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    T, Hg, Wg = (int(x) for x in grid)
    if N != T * Hg * Wg:
        raise ValueError(f"N={N} but T*Hg*Wg={T * Hg * Wg}")
    g = _geom(T, Hg, Wg, block_frames, rope_split, theta, eps)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=q.dtype, device=q.device)
    else:
        _check_out(out, (B, H, N, d), q.dtype, q.device)
        _check_no_overlap(out, q, k, v)
    need = int(lib.blin_prefill_workspace_size(B, H, d, ctypes.byref(g)))
    workspace, ws_ptr, ws_bytes = _workspace_arg(workspace, need, q.device)
    args = (ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
            ctypes.c_void_p(out.data_ptr()), _dtype_code(q), B, H, d, ctypes.byref(g))
    tail = (state.handle if state is not None else None, ws_ptr, ws_bytes, _stream(stream))
    lays = _layouts(q, out)
    if lays is None:
        _check(lib.blin_prefill(*args, *tail))
    else:
        _check(lib.blin_prefill_strided(*args, ctypes.byref(lays[0]), ctypes.byref(lays[1]), *tail))
    return out


def block_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, Hg: int, Wg: int, frames: int,
               rope_split: Sequence[int], state: BlockState, theta: float = 1e4, eps: float = 1e-6,
               commit: bool = True, out: Optional[torch.Tensor] = None, stream=None,
               block_frames: Optional[int] = None) -> torch.Tensor:
    """One autoregressive block of `frames` latent frames read against (and, if
    commit, added to) the cached state.  `block_frames` is the causal block
    length F (default: `frames`); the call's frames must lie in one block.
    Strided views are accepted as for prefill()."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    if N != frames * Hg * Wg:
        raise ValueError(f"N={N} but frames*Hg*Wg={frames * Hg * Wg}")
    if out is None:
        out = torch.empty((B, H, N, d), dtype=q.dtype, device=q.device)
    else:
        _check_out(out, (B, H, N, d), q.dtype, q.device)
        _check_no_overlap(out, q, k, v)
    g = _geom(frames, Hg, Wg, frames if block_frames is None else block_frames, rope_split, theta, eps)
    args = (ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
            ctypes.c_void_p(out.data_ptr()), _dtype_code(q), B, H, d, ctypes.byref(g))
    lays = _layouts(q, out)
    if lays is None:
        _check(lib.blin_block_step(*args, state.handle, 1 if commit else 0, _stream(stream)))
    else:
        _check(lib.blin_block_step_strided(*args, ctypes.byref(lays[0]), ctypes.byref(lays[1]), state.handle,
                                           1 if commit else 0, _stream(stream)))
    return out


PATHS = {0: "none", 1: "tensor_core", 2: "cuda_core"}


def last_path() -> str:
    """Which kernels this thread's last prefill / block_step ran: "tensor_core" or "cuda_core"."""
    return PATHS[int(lib.blin_last_path())]


# Launch slots of one call, in order.  The tensor-core path launches three
# kernels (partial states, block scan, output); the CUDA-core path also builds
# a RoPE table first.
KERNELS = ("rope_table", "partial_states", "block_scan", "output")
# Algorithmic HBM bytes per token*head of each launch, in units of d * element
# size: pass 1 reads K and V, pass 2 reads Q and writes O (the scan and the
# table move no per-token bytes).
KERNEL_BYTES_PER_UNIT = {"partial_states": 2, "output": 2}


class LaunchTimer:
    """Records CUDA events around each of the library's launches (profiling aid).

    Use ``with LaunchTimer() as t: ...`` around calls on the current thread, then
    ``t.elapsed_ms()`` (after synchronising) for per-kernel times of the last
    call.  ``arm()`` re-arms a fresh set of events for the next call.
    """

    def __init__(self):
        self.sets = []

    def new_set(self):
        """Create (and keep) one set of 8 events; returns the C array to arm with."""
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
        for e in evs:  # force creation of the underlying cudaEvent_t
            e.record()
        torch.cuda.current_stream().synchronize()
        arr = (ctypes.c_void_p * 8)(*[e.cuda_event for e in evs])
        self.sets.append((evs, arr))
        return arr

    @staticmethod
    def arm_set(arr) -> None:
        _check(lib.blin_set_timing_events(ctypes.cast(arr, ctypes.c_void_p), 8))

    def arm(self):
        arr = self.new_set()
        self.arm_set(arr)
        return self.sets[-1][0]

    def __enter__(self):
        self.arm()
        return self

    def __exit__(self, *exc):
        lib.blin_set_timing_events(None, 0)
        return False

    def elapsed_ms(self):
        """[{kernel name: ms}] for every armed call (events must have completed)."""
        out = []
        for evs, _ in self.sets:
            out.append({k: evs[2 * i].elapsed_time(evs[2 * i + 1]) for i, k in enumerate(KERNELS)})
        return out


def device_status() -> int:
    """Synchronise, then read and clear the kernels' watchdog word (0 = clean)."""
    code = ctypes.c_int(0)
    rc = lib.blin_device_status(ctypes.byref(code))
    if rc not in (0, -8):
        _check(rc)
    return code.value


def launch_count() -> int:
    """Kernels this library has launched in this process so far."""
    return int(lib.blin_launch_count())


# ----------------------------------------------------------------------------- temporal convolution
class TConvState:
    """One-frame cache of the causal block temporal convolution: [B, Hg*Wg, C]."""

    def __init__(self, B: int, C: int, Hg: int, Wg: int, dtype=torch.bfloat16, stream=None):
        self.B, self.C, self.Hg, self.Wg = B, C, Hg, Wg
        self.dtype = dtype
        h = ctypes.c_void_p()
        dt = BF16 if dtype == torch.bfloat16 else F32
        _check(lib.blin_tconv_state_init(B, C, Hg, Wg, dt, _stream(stream), ctypes.byref(h)))
        self._h = h

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise BlinError(-6, "state already freed")
        return self._h

    def free(self) -> None:
        if self._h is not None:
            _check(lib.blin_tconv_state_free(self._h))
            self._h = None

    def __del__(self):
        try:
            if getattr(self, "_h", None) is not None:
                lib.blin_tconv_state_free(self._h)
        except Exception:
            pass

    @property
    def t_next(self) -> int:
        t = ctypes.c_int()
        _check(lib.blin_tconv_state_frame(self.handle, None, ctypes.byref(t)))
        return t.value

    @property
    def nbytes(self) -> int:
        return int(lib.blin_tconv_state_bytes(self.handle))

    def reset(self, stream=None) -> None:
        _check(lib.blin_tconv_state_reset(self.handle, _stream(stream)))

    def frame_ptr(self) -> int:
        """Device address of the cached frame [B, Hg*Wg, C]."""
        ptr = ctypes.c_void_p()
        _check(lib.blin_tconv_state_frame(self.handle, ctypes.byref(ptr), None))
        return int(ptr.value)


def tconv(x: torch.Tensor, taps: torch.Tensor, bias: Optional[torch.Tensor], grid: Sequence[int], block_frames: int,
          state: Optional[TConvState] = None, commit: bool = True, out: Optional[torch.Tensor] = None,
          stream=None) -> torch.Tensor:
    """Causal block temporal convolution of x [B, T*Hg*Wg, C] (frame-major tokens, channels
    innermost) with taps [C, 3] (previous, current, next) and bias [C] (fp32, or None).
    With a state, the call continues its video and (if commit) updates its cache; without
    one it is the start of a video and nothing is cached."""
    if x.dim() != 3 or not x.is_contiguous() or not x.is_cuda:
        raise ValueError("x must be a contiguous CUDA [B, T*Hg*Wg, C] tensor")
    B, N, C = x.shape
    T, Hg, Wg = (int(v) for v in grid)
    if N != T * Hg * Wg:
        raise ValueError(f"N={N} but T*Hg*Wg={T * Hg * Wg}")
    _check_device(x)
    if taps.numel() != 3 * C or (bias is not None and bias.numel() != C):
        raise ValueError(f"taps must hold [C, 3] = {3 * C} values and bias [C] = {C}")
    taps = taps.to(device=x.device, dtype=torch.float32).contiguous()
    if bias is not None:
        bias = bias.to(device=x.device, dtype=torch.float32).contiguous()
    if out is None:
        out = torch.empty_like(x)
    else:
        _check_out(out, x.shape, x.dtype, x.device, contiguous=True)
        _check_no_overlap(out, x)
    g = _geom(T, Hg, Wg, block_frames, (0, 0, 0), 1e4, 0.0)
    _check(lib.blin_tconv(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(taps.data_ptr()),
                          None if bias is None else ctypes.c_void_p(bias.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                          _dtype_code(x), B, C, ctypes.byref(g), None if state is None else state.handle,
                          1 if (commit and state is not None) else 0, _stream(stream)))
    return out


# ----------------------------------------------------------------------------- NVFP4 inputs
class Nvfp4Tensor:
    """An NVFP4 [B, H, N, d] operand on the device: packed E2M1 codes [B, H, N, d/2] (uint8,
    even element in the low nibble), E4M3 block scales [B, H, N, d/16] (uint8, one per 16
    elements; stored in an allocation padded to 16 bytes) and a global scale."""

    def __init__(self, data: torch.Tensor, scale: torch.Tensor, global_scale: float):
        if data.dtype != torch.uint8 or scale.dtype != torch.uint8 or data.dim() != 4 or scale.dim() != 4:
            raise ValueError("data and scale must be 4D uint8 tensors")
        B, H, N, half = data.shape
        d = 2 * half
        if tuple(scale.shape) != (B, H, N, d // 16):
            raise ValueError("scale must be [B, H, N, d/16]")
        self.shape = (B, H, N, d)
        self.data = data.contiguous().cuda()
        n = scale.numel()
        buf = torch.zeros((n + 15) // 16 * 16, dtype=torch.uint8, device=self.data.device)
        buf[:n].copy_(scale.reshape(-1))
        self._scale_buf = buf
        self.scale = buf[:n].view(B, H, N, d // 16)
        self.global_scale = float(global_scale)

    def c(self) -> Nvfp4:
        return Nvfp4(ctypes.c_void_p(self.data.data_ptr()), ctypes.c_void_p(self.scale.data_ptr()), self.global_scale)


def _nvfp4_device(q: "Nvfp4Tensor", k: "Nvfp4Tensor", v: "Nvfp4Tensor") -> torch.device:
    dev = q.data.device
    if not all(t.data.device == dev and t.scale.device == dev for t in (q, k, v)):
        raise ValueError("q, k and v must be on one device")
    _check_device(q.data)
    return dev


def prefill_nvfp4(q: Nvfp4Tensor, k: Nvfp4Tensor, v: Nvfp4Tensor, grid: Sequence[int], block_frames: int,
                  rope_split: Sequence[int], theta: float = 1e4, eps: float = 1e-6,
                  state: Optional[BlockState] = None, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """prefill() on NVFP4 q, k, v; the output is bf16 [B, H, N, d]."""
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k and v must share a shape")
    B, H, N, d = q.shape
    T, Hg, Wg = (int(x) for x in grid)
    if N != T * Hg * Wg:
        raise ValueError(f"N={N} but T*Hg*Wg={T * Hg * Wg}")
    g = _geom(T, Hg, Wg, block_frames, rope_split, theta, eps)
    dev = _nvfp4_device(q, k, v)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    else:
        _check_out(out, (B, H, N, d), torch.bfloat16, dev, contiguous=True)
    need = int(lib.blin_prefill_workspace_size(B, H, d, ctypes.byref(g)))
    workspace, ws_ptr, ws_bytes = _workspace_arg(workspace, need, dev)
    qc, kc, vc = q.c(), k.c(), v.c()
    _check(lib.blin_prefill_nvfp4(ctypes.byref(qc), ctypes.byref(kc), ctypes.byref(vc), ctypes.c_void_p(out.data_ptr()),
                                  B, H, d, ctypes.byref(g), state.handle if state is not None else None,
                                  ws_ptr, ws_bytes, _stream(stream)))
    return out


def block_step_nvfp4(q: Nvfp4Tensor, k: Nvfp4Tensor, v: Nvfp4Tensor, Hg: int, Wg: int, frames: int,
                     rope_split: Sequence[int], state: BlockState, theta: float = 1e4, eps: float = 1e-6,
                     commit: bool = True, out: Optional[torch.Tensor] = None, stream=None,
                     block_frames: Optional[int] = None) -> torch.Tensor:
    """block_step() on NVFP4 q, k, v; the output is bf16."""
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k and v must share a shape")
    B, H, N, d = q.shape
    if N != frames * Hg * Wg:
        raise ValueError(f"N={N} but frames*Hg*Wg={frames * Hg * Wg}")
    dev = _nvfp4_device(q, k, v)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    else:
        _check_out(out, (B, H, N, d), torch.bfloat16, dev, contiguous=True)
    g = _geom(frames, Hg, Wg, frames if block_frames is None else block_frames, rope_split, theta, eps)
    qc, kc, vc = q.c(), k.c(), v.c()
    _check(lib.blin_block_step_nvfp4(ctypes.byref(qc), ctypes.byref(kc), ctypes.byref(vc),
                                     ctypes.c_void_p(out.data_ptr()), B, H, d, ctypes.byref(g), state.handle,
                                     1 if commit else 0, _stream(stream)))
    return out
