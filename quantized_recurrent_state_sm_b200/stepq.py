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
# STEPQ_CHECK=1 in the environment selects the checking build (the kernels
# validate the pool's tables before touching memory; include/stepq.h).
CHECK_BUILD = os.environ.get("STEPQ_CHECK", "0") == "1"
LIB_PATH = os.path.join(_HERE, "libstepq_check.so" if CHECK_BUILD else "libstepq.so")

GDN, KDA = 0, 1
SCALE_DUAL, SCALE_ROW, SCALE_COL, SCALE_HEAD = 0, 1, 2, 3
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


class Regions(C.Structure):
    _fields_ = [("states", C.c_size_t), ("state_bytes", C.c_size_t), ("head_records", C.c_size_t),
                ("head_offsets", C.c_size_t), ("item_sizes", C.c_size_t), ("status_word", C.c_size_t),
                ("item_order", C.c_size_t), ("staging_records", C.c_size_t), ("guards", C.c_size_t * 7),
                ("guard_bytes", C.c_size_t), ("total", C.c_size_t)]


class CalibDesc(C.Structure):
    _fields_ = [("variant", C.c_int), ("batch", C.c_int), ("heads", C.c_int), ("dk", C.c_int),
                ("dv", C.c_int), ("steps", C.c_int), ("sample_every", C.c_int), ("ls_iters", C.c_int),
                ("n_widths", C.c_int), ("widths", C.c_void_p), ("avg_bits", C.c_double),
                ("pivot_frac", C.c_double)]


EXPORTS = ("stepq_pool_bytes", "stepq_state_bytes", "stepq_pool_layout", "stepq_pool_check_guards", "stepq_pool_create", "stepq_pool_destroy",
           "stepq_pool_set_stream", "stepq_pack", "stepq_unpack", "stepq_decode_step",
           "stepq_fp32_step", "stepq_pool_check", "stepq_status_string", "stepq_last_error", "stepq_selftest_bounded_wait",
           "stepq_decode_step_noalloc", "stepq_decode_step_split", "stepq_pool_set_active",
           "stepq_pool_set_scale_mode", "stepq_calib_scratch_bytes", "stepq_calibrate", "stepq_calib_accumulate", "stepq_calib_row_error",
           "stepq_calib_reduce", "stepq_calib_rho", "stepq_calib_bits")


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
    L.stepq_pool_check_guards.argtypes = [P]
    L.stepq_pool_layout.argtypes = [D, C.POINTER(Regions)]
    L.stepq_selftest_bounded_wait.argtypes = [P, C.c_longlong, C.c_int, P]
    L.stepq_pack.argtypes = [P, P]
    L.stepq_unpack.argtypes = [P, P]
    L.stepq_decode_step.argtypes = [P, P, P, P, P, P, P]
    L.stepq_fp32_step.argtypes = [D, P, P, P, P, P, P, P, P]
    L.stepq_decode_step_noalloc.argtypes = [D, P, C.c_size_t, P, P, P, P, P, P, P]
    L.stepq_decode_step_split.argtypes = [P, P, P, P, P, P, P, P, P]
    L.stepq_pool_set_active.argtypes = [P, P, C.c_int]
    L.stepq_pool_set_scale_mode.argtypes = [P, C.c_int]
    CD, i, dbl = C.POINTER(CalibDesc), C.c_int, C.c_double
    L.stepq_calib_scratch_bytes.argtypes = [CD]; L.stepq_calib_scratch_bytes.restype = C.c_size_t
    L.stepq_calibrate.argtypes = [CD, P, P, P, P, P, P, P, C.c_size_t, P, P, P]
    L.stepq_calib_accumulate.argtypes = [i, i, i, P, P, P, P, P]
    L.stepq_calib_row_error.argtypes = [i, i, P, P, i, P, i, P, P, P]
    L.stepq_calib_reduce.argtypes = [i, i, i, P, P, P]
    L.stepq_calib_rho.argtypes = [i, dbl, P, P]
    L.stepq_calib_bits.argtypes = [i, i, dbl, P, P, P, i, P, dbl, dbl, P]
    for fn in ("stepq_pool_create", "stepq_pool_destroy", "stepq_pool_set_stream", "stepq_pool_check",
               "stepq_selftest_bounded_wait", "stepq_pack",
               "stepq_unpack", "stepq_decode_step", "stepq_fp32_step", "stepq_decode_step_noalloc",
               "stepq_decode_step_split", "stepq_pool_set_active", "stepq_pool_set_scale_mode", "stepq_calibrate", "stepq_calib_accumulate",
               "stepq_calib_row_error", "stepq_calib_reduce", "stepq_calib_rho", "stepq_calib_bits"):
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

    def set_scale_mode(self, mode: int):
        """The scale fit of later pack / decode calls: SCALE_DUAL (the method)
        or an ablation variant SCALE_ROW, SCALE_COL, SCALE_HEAD."""
        _check(lib.stepq_pool_set_scale_mode(self._h, int(mode)))

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

    def check_guards(self):
        """Raise if a guard word after any region of the pool buffer changed."""
        self._sync_stream()
        _check(lib.stepq_pool_check_guards(self._h))

    @property
    def regions(self) -> dict:
        """Byte offsets of the buffer's regions (stepq_pool_layout)."""
        r = Regions()
        _check(lib.stepq_pool_layout(C.byref(self._desc), C.byref(r)))
        out = {f: getattr(r, f) for f, _ in Regions._fields_ if f != "guards"}
        out["guards"] = list(r.guards)
        return out

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


def selftest_bounded_wait(limit_cycles: int, arrive: bool, device=None) -> tuple[int, int]:
    """Run the kernels' bounded barrier wait once (include/stepq.h,
    stepq_selftest_bounded_wait): (0 or 1 = gave up, cycles waited)."""
    res = torch.full((2,), -1, dtype=torch.int32, device=device or "cuda")
    _check(lib.stepq_selftest_bounded_wait(C.c_void_p(res.data_ptr()), int(limit_cycles), int(bool(arrive)),
                                           _stream_ptr()))
    torch.cuda.current_stream().synchronize()
    r = res.cpu().tolist()
    return r[0], r[1]


# ---- calibration -------------------------------------------------------------

def _dev_any(t: torch.Tensor, name: str, dtype, shape) -> C.c_void_p:
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_cuda:
        raise TypeError(f"{name} must be a {dtype} CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


def _host(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(C.c_void_p)


def calibrate(variant: int, S0: torch.Tensor, q, k, v, alpha, beta, widths, avg_bits: float,
              pivot_frac: float, sample_every: int, ls_iters: int = 1):
    """The library's calibration (stepq_calibrate): S0 [B, H, 128, 128] and the
    rollout's inputs q, k [T, B, H, 128], v [T, B, H, 128], alpha [T, B, H] or
    [T, B, H, 128], beta [T, B, H], all float32 CUDA tensors.  Returns
    (rho [H, 128] float32, bits [H, 128] uint8) as numpy arrays."""
    T, B, H = q.shape[0], q.shape[1], q.shape[2]
    w, wp = _host(widths, np.int32)
    cd = CalibDesc(variant, B, H, DK, DV, T, int(sample_every), int(ls_iters), int(w.size), wp,
                   float(avg_bits), float(pivot_frac))
    nbytes = lib.stepq_calib_scratch_bytes(C.byref(cd))
    if nbytes == 0:
        _check(ERR_INVALID_ARG)
    scratch = torch.empty(nbytes, dtype=torch.uint8, device=S0.device)
    rho = np.zeros((H, DK), np.float32); bits = np.zeros((H, DK), np.uint8)
    ash = (T, B, H, DK) if variant == KDA else (T, B, H)
    _check(lib.stepq_calibrate(C.byref(cd), _dev(S0, "S0", (B, H, DK, DV)), _dev(q, "q", (T, B, H, DK)),
                               _dev(k, "k", (T, B, H, DK)), _dev(v, "v", (T, B, H, DV)), _dev(alpha, "alpha", ash),
                               _dev(beta, "beta", (T, B, H)), C.c_void_p(scratch.data_ptr()), nbytes,
                               _stream_ptr(), rho.ctypes.data_as(C.c_void_p), bits.ctypes.data_as(C.c_void_p)))
    return rho, bits


def calib_accumulate(variant: int, q: torch.Tensor, alpha: torch.Tensor, acc_q2: torch.Tensor,
                     acc_loga: torch.Tensor):
    """One step's q [B, H, 128] and alpha into the float64 CUDA sums acc_q2
    [H, 128] and acc_loga ([H] or [H, 128])."""
    B, H = q.shape[0], q.shape[1]
    ash = (B, H, DK) if variant == KDA else (B, H)
    _check(lib.stepq_calib_accumulate(variant, B, H, _dev(q, "q", (B, H, DK)), _dev(alpha, "alpha", ash),
                                      _dev_any(acc_q2, "acc_q2", torch.float64, (H, DK)),
                                      _dev_any(acc_loga, "acc_loga", torch.float64, (H, DK) if variant == KDA else (H,)),
                                      _stream_ptr()))


def calib_row_error(S: torch.Tensor, rho: torch.Tensor, widths, ls_iters: int = 1):
    """Per-row squared errors of the states S [B, H, 128, 128] stored at each of
    `widths`: returns (err [B, H, nW, 128], rc [B, H, nW, 256]) float32 CUDA tensors."""
    B, H = S.shape[0], S.shape[1]
    w, wp = _host(widths, np.int32)
    err = torch.empty((B, H, w.size, DK), dtype=torch.float32, device=S.device)
    rc = torch.empty((B, H, w.size, DK + DV), dtype=torch.float32, device=S.device)
    _check(lib.stepq_calib_row_error(B, H, _dev(S, "S", (B, H, DK, DV)), _dev(rho, "rho", (H, DK)), int(w.size), wp,
                                     int(ls_iters), C.c_void_p(err.data_ptr()), C.c_void_p(rc.data_ptr()),
                                     _stream_ptr()))
    return err, rc


def calib_reduce(err: torch.Tensor, err_sum: torch.Tensor):
    """err_sum [H, nW, 128] (float64 CUDA) += err [B, H, nW, 128], request by request."""
    B, H, nW = err.shape[0], err.shape[1], err.shape[2]
    _check(lib.stepq_calib_reduce(B, H, nW, _dev(err, "err", (B, H, nW, DK)),
                                  _dev_any(err_sum, "err_sum", torch.float64, (H, nW, DK)), _stream_ptr()))


def calib_rho(acc_q2: np.ndarray, n_samples: float) -> np.ndarray:
    """Host: impact scores [H, 128] from the sums of q^2."""
    a, ap = _host(acc_q2, np.float64)
    H = a.shape[0]
    rho = np.zeros((H, DK), np.float32)
    _check(lib.stepq_calib_rho(H, float(n_samples), ap, rho.ctypes.data_as(C.c_void_p)))
    return rho


def calib_bits(variant: int, acc_loga, rho, err_sum, widths, avg_bits, pivot_frac, n_samples) -> np.ndarray:
    """Host: the row widths [H, 128] from the calibration sums (err_sum [H, nW, 128])."""
    la, lap = _host(acc_loga, np.float64)
    r, rp = _host(rho, np.float32)
    e, ep = _host(err_sum, np.float64)
    w, wp = _host(widths, np.int32)
    H = e.shape[0]
    bits = np.zeros((H, DK), np.uint8)
    _check(lib.stepq_calib_bits(variant, H, float(n_samples), lap, rp, ep, int(w.size), wp, float(avg_bits),
                                float(pivot_frac), bits.ctypes.data_as(C.c_void_p)))
    return bits
