"""Python binding of the C ABI in include/stepq.h (libstepq.so, sm_100a).

Argument marshalling only: tensors are checked for dtype, device, shape and
contiguity, then their device pointers and torch's current CUDA stream are
passed to the library.  Every step of the computation runs in the library's
kernels; there is no fallback.  If the library has not been built the import of
this module raises.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstepq.so")

GDN, KDA = 0, 1
PIVOT_BITS = 16
DK = DV = 128

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_STATE = 0, 1, 2, 3, 4


class StepqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


class Desc(C.Structure):
    _fields_ = [("variant", C.c_int), ("batch", C.c_int), ("heads", C.c_int), ("dk", C.c_int),
                ("dv", C.c_int), ("ls_iters", C.c_int), ("bits", C.c_void_p), ("rho", C.c_void_p)]


EXPORTS = ("stepq_pool_bytes", "stepq_state_bytes", "stepq_pool_create", "stepq_pool_destroy",
           "stepq_pool_set_stream", "stepq_pack", "stepq_unpack", "stepq_decode_step",
           "stepq_fp32_step", "stepq_pool_check", "stepq_status_string", "stepq_last_error",
           "stepq_decode_step_noalloc", "stepq_decode_step_split", "stepq_pool_set_active")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -c 'import __graft_entry__ as g; g.build()'`")
    L = C.CDLL(LIB_PATH)
    P, D = C.c_void_p, C.POINTER(Desc)
    L.stepq_pool_bytes.argtypes = [D]; L.stepq_pool_bytes.restype = C.c_size_t
    L.stepq_state_bytes.argtypes = [D]; L.stepq_state_bytes.restype = C.c_size_t
    L.stepq_pool_create.argtypes = [D, P, C.c_size_t, P, C.POINTER(P)]
    L.stepq_pool_destroy.argtypes = [P]
    L.stepq_pool_set_stream.argtypes = [P, P]
    L.stepq_pool_check.argtypes = [P]
    L.stepq_pack.argtypes = [P, P]
    L.stepq_unpack.argtypes = [P, P]
    L.stepq_decode_step.argtypes = [P, P, P, P, P, P, P]
    L.stepq_fp32_step.argtypes = [D, P, P, P, P, P, P, P, P]
    L.stepq_decode_step_noalloc.argtypes = [D, P, C.c_size_t, P, P, P, P, P, P, P]
    L.stepq_decode_step_split.argtypes = [P, P, P, P, P, P, P, P, P]
    L.stepq_pool_set_active.argtypes = [P, P, C.c_int]
    for fn in ("stepq_pool_create", "stepq_pool_destroy", "stepq_pool_set_stream", "stepq_pool_check", "stepq_pack",
               "stepq_unpack", "stepq_decode_step", "stepq_fp32_step", "stepq_decode_step_noalloc",
               "stepq_decode_step_split", "stepq_pool_set_active"):
        getattr(L, fn).restype = C.c_int
    L.stepq_status_string.argtypes = [C.c_int]; L.stepq_status_string.restype = C.c_char_p
    L.stepq_last_error.argtypes = []; L.stepq_last_error.restype = C.c_char_p
    return L


lib = _load()


def _check(status: int):
    if status != OK:
        msg = lib.stepq_last_error().decode(errors="replace")
        raise StepqError(status, f"{lib.stepq_status_string(status).decode()}: {msg}")


def _stream_ptr(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, shape) -> C.c_void_p:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.float32 or not t.is_cuda:
        raise TypeError(f"{name} must be a float32 CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


def make_desc(variant: int, batch: int, heads: int, bits: np.ndarray, rho: np.ndarray, ls_iters: int = 1):
    bits = np.ascontiguousarray(bits, dtype=np.uint8)
    rho = np.ascontiguousarray(rho, dtype=np.float32)
    if bits.shape != (heads, DK) or rho.shape != (heads, DK):
        raise ValueError("bits and rho must have shape [heads, 128]")
    d = Desc(variant, batch, heads, DK, DV, ls_iters, bits.ctypes.data_as(C.c_void_p),
             rho.ctypes.data_as(C.c_void_p))
    return d, (bits, rho)  # keep the host tables alive while the desc is used


def pool_bytes(variant, batch, heads, bits, rho, ls_iters=1) -> int:
    d, keep = make_desc(variant, batch, heads, bits, rho, ls_iters)
    n = lib.stepq_pool_bytes(C.byref(d))
    if n == 0:
        _check(ERR_INVALID_ARG)
    return int(n)


class PackedStatePool:
    """Packed recurrent states of batch x heads (request, head) items on one GPU.

    The device buffer is a torch uint8 tensor owned by this object; the library
    works in it in place.  Kernels run on torch's current CUDA stream.
    """

    def __init__(self, variant: int, batch: int, heads: int, bits, rho, ls_iters: int = 1,
                 device=None):
        self.variant, self.batch, self.heads, self.ls_iters = variant, batch, heads, ls_iters
        self._desc, self._keep = make_desc(variant, batch, heads, bits, rho, ls_iters)
        self.nbytes = int(lib.stepq_pool_bytes(C.byref(self._desc)))
        if self.nbytes == 0:
            _check(ERR_INVALID_ARG)
        self.state_nbytes = int(lib.stepq_state_bytes(C.byref(self._desc)))
        dev = torch.device("cuda") if device is None else torch.device(device)
        self.buffer = torch.empty(self.nbytes, dtype=torch.uint8, device=dev)
        h = C.c_void_p()
        _check(lib.stepq_pool_create(C.byref(self._desc), C.c_void_p(self.buffer.data_ptr()),
                                     self.nbytes, _stream_ptr(), C.byref(h)))
        self._h = h
        self.n_active = batch

    @property
    def n_items(self) -> int:
        return self.batch * self.heads

    def set_active(self, requests=None):
        """Restrict later decode steps to the listed requests (distinct slot
        indices in 0 .. batch-1); None = all.  decode_step keeps its
        [batch, heads, ...] shapes: it reads and writes only the listed
        requests' rows and updates only their states."""
        if requests is None:
            self._check_active(lib.stepq_pool_set_active(self._h, None, 0))
            self.n_active = self.batch
            return
        arr = np.ascontiguousarray(np.asarray(requests, dtype=np.int32).reshape(-1))
        self._sync_stream()
        self._check_active(lib.stepq_pool_set_active(self._h, arr.ctypes.data_as(C.c_void_p), int(arr.size)))
        self._active_host = arr  # the upload reads it on the stream
        self.n_active = int(arr.size)

    @staticmethod
    def _check_active(status):
        _check(status)

    @property
    def state(self) -> torch.Tensor:
        """The packed states (a view of the first state_nbytes bytes of the buffer)."""
        return self.buffer[: self.state_nbytes]

    def _sync_stream(self):
        _check(lib.stepq_pool_set_stream(self._h, _stream_ptr()))

    def pack(self, S: torch.Tensor):
        self._sync_stream()
        _check(lib.stepq_pack(self._h, _dev(S, "S", (self.batch, self.heads, DK, DV))))

    def unpack(self, out: torch.Tensor | None = None) -> torch.Tensor:
        if out is None:
            out = torch.empty((self.batch, self.heads, DK, DV), dtype=torch.float32, device=self.buffer.device)
        self._sync_stream()
        _check(lib.stepq_unpack(self._h, _dev(out, "S_out", (self.batch, self.heads, DK, DV))))
        return out

    def decode_step(self, q, k, v, alpha, beta, out=None) -> torch.Tensor:
        B, H = self.batch, self.heads
        if out is None:
            out = torch.empty((B, H, DV), dtype=torch.float32, device=self.buffer.device)
        ash = (B, H, DK) if self.variant == KDA else (B, H)
        self._sync_stream()
        _check(lib.stepq_decode_step(self._h, _dev(q, "q", (B, H, DK)), _dev(k, "k", (B, H, DK)),
                                     _dev(v, "v", (B, H, DV)), _dev(alpha, "alpha", ash),
                                     _dev(beta, "beta", (B, H)), _dev(out, "out", (B, H, DV))))
        return out

    def decode_step_split(self, q, k, v, alpha, beta, S_work, out=None, side_stream=None) -> torch.Tensor:
        """The same step as decode_step, split the way the pages' kernels split
        it: update + readout into S_work (fp32 [B, H, 128, 128]), then fit and
        packed writeback on side_stream (a torch.cuda.Stream; None = the
        current stream)."""
        B, H = self.batch, self.heads
        if out is None:
            out = torch.empty((B, H, DV), dtype=torch.float32, device=self.buffer.device)
        ash = (B, H, DK) if self.variant == KDA else (B, H)
        self._sync_stream()
        side = None if side_stream is None else C.c_void_p(side_stream.cuda_stream)
        _check(lib.stepq_decode_step_split(self._h, _dev(S_work, "S_work", (B, H, DK, DV)),
                                           _dev(q, "q", (B, H, DK)), _dev(k, "k", (B, H, DK)),
                                           _dev(v, "v", (B, H, DV)), _dev(alpha, "alpha", ash),
                                           _dev(beta, "beta", (B, H)), _dev(out, "out", (B, H, DV)), side))
        return out

    def check(self):
        """Synchronise the pool's stream and raise if a kernel reported an error."""
        self._sync_stream()
        _check(lib.stepq_pool_check(self._h))

    def close(self):
        if getattr(self, "_h", None):
            lib.stepq_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fp32_step(variant: int, S: torch.Tensor, q, k, v, alpha, beta, out=None) -> torch.Tensor:
    """Unquantised fp32-state update + readout, in place on S [B, H, 128, 128]."""
    B, H = S.shape[0], S.shape[1]
    if out is None:
        out = torch.empty((B, H, DV), dtype=torch.float32, device=S.device)
    d = Desc(variant, B, H, DK, DV, 1, None, None)
    ash = (B, H, DK) if variant == KDA else (B, H)
    _check(lib.stepq_fp32_step(C.byref(d), _dev(S, "S", (B, H, DK, DV)), _dev(q, "q", (B, H, DK)),
                               _dev(k, "k", (B, H, DK)), _dev(v, "v", (B, H, DV)),
                               _dev(alpha, "alpha", ash), _dev(beta, "beta", (B, H)),
                               _dev(out, "out", (B, H, DV)), _stream_ptr()))
    return out


def decode_step_noalloc(variant: int, bits, rho, states: torch.Tensor, q, k, v, alpha, beta, out=None,
                        ls_iters: int = 1) -> torch.Tensor:
    """The fused decode step on packed states held in `states` (a uint8 CUDA
    tensor laid out as a pool's packed states), without a pool: the library
    keeps the kernel's tables in its own fixed device scratch and allocates
    nothing.  Calls must not overlap (one stream); see include/stepq.h."""
    bits = np.ascontiguousarray(bits, dtype=np.uint8)
    H = bits.shape[0]
    B = q.shape[0]
    d, keep = make_desc(variant, B, H, bits, rho, ls_iters)
    if not isinstance(states, torch.Tensor) or states.dtype != torch.uint8 or not states.is_cuda:
        raise TypeError("states must be a uint8 CUDA tensor")
    if not states.is_contiguous():
        raise ValueError("states must be contiguous")
    if out is None:
        out = torch.empty((B, H, DV), dtype=torch.float32, device=states.device)
    ash = (B, H, DK) if variant == KDA else (B, H)
    _check(lib.stepq_decode_step_noalloc(C.byref(d), C.c_void_p(states.data_ptr()), states.numel(),
                                         _dev(q, "q", (B, H, DK)), _dev(k, "k", (B, H, DK)),
                                         _dev(v, "v", (B, H, DV)), _dev(alpha, "alpha", ash),
                                         _dev(beta, "beta", (B, H)), _dev(out, "out", (B, H, DV)),
                                         _stream_ptr()))
    return out
