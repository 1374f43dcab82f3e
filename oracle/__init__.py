"""ctypes wrapper around the CPU oracle (oracle/liboracle.so).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by
bench.py's CPU-baseline leg.  The product path never imports this package.
Every function takes and returns numpy arrays; the arithmetic is in C.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        i = C.c_int
        L.oracle_fit_quantise_f32.argtypes = [i, i, P, P, P, i, i, P, P, P, P, P, P]
        L.oracle_fit_quantise_f64.argtypes = [i, i, P, P, P, i, i, P, P, P, P, P, P]
        L.oracle_quantise_f32.argtypes = [i, i, P, P, P, P, P, P]
        L.oracle_quantise_f64.argtypes = [i, i, P, P, P, P, P, P]
        L.oracle_dequant_f32.argtypes = [i, i, P, P, P, P, P, P]
        L.oracle_dequant_f64.argtypes = [i, i, P, P, P, P, P, P]
        L.oracle_update_f32.argtypes = [i, i, P, P, P, P, P, C.c_float, P]
        L.oracle_update_f64.argtypes = [i, i, P, P, P, P, P, C.c_double, P]
        L.oracle_column_error_f64.argtypes = [i, i, i, P, P, P, P, C.c_double, P]
        L.oracle_column_error_f64.restype = C.c_double
        L.oracle_to_fp16.argtypes = [C.c_double]
        L.oracle_to_fp16.restype = C.c_uint16
        L.oracle_from_fp16.argtypes = [C.c_uint16]
        L.oracle_from_fp16.restype = C.c_double
        L.oracle_item_bytes.argtypes = [i, i, P]
        L.oracle_item_bytes.restype = C.c_size_t
        L.oracle_pack_item.argtypes = [i, i, P, P, P, P, P, P]
        L.oracle_unpack_item.argtypes = [i, i, P, P, P, P, P, P]
        L.oracle_pool_bytes.argtypes = [i, P, i, i, P]
        L.oracle_pool_bytes.restype = C.c_size_t
        L.oracle_pack_pool.argtypes = [i, P, i, i, P, P, i, P, P]
        L.oracle_unpack_pool.argtypes = [i, P, i, i, P, P, P]
        L.oracle_decode_step.argtypes = [i, P, i, i, P, P, i, i, P, P, P, P, P, P, P, P, P, P]
        L.oracle_fp32_step.argtypes = [i, i, i, i, P, P, P, P, P, P, P]
        L.oracle_fp64_step.argtypes = [i, i, i, i, P, P, P, P, P, P, P]
        L.oracle_fit_quantise_mode_f32.argtypes = [i, i, i, P, P, P, i, i, P, P, P, P, P]
        L.oracle_pack_pool_mode.argtypes = [i, i, P, i, i, P, P, i, P, P]
        L.oracle_decode_step_mode.argtypes = [i, i, P, i, i, P, P, i, i, P, P, P, P, P, P, P, P, P]
        L.oracle_calib_accumulate.argtypes = [i, i, i, i, P, P, P, P]
        L.oracle_calib_rho.argtypes = [i, i, C.c_double, P, P]
        L.oracle_calib_row_error.argtypes = [i, i, P, i, P, i, P, P, P]
        L.oracle_calib_weight.argtypes = [C.c_double]
        L.oracle_calib_weight.restype = C.c_double
        L.oracle_calib_allocate.argtypes = [i, P, P, i, P, C.c_double, i, P]
        L.oracle_calib_allocate.restype = C.c_int
        L.oracle_calib_bits.argtypes = [i, i, i, C.c_double, P, P, P, i, P, C.c_double, C.c_double, P]
        L.oracle_calib_bits.restype = C.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


PIVOT_FP16, PIVOT_EXACT = 0, 1
SCALE_DUAL, SCALE_ROW, SCALE_COL, SCALE_HEAD = 0, 1, 2, 3


def fit_quantise(S, bits, rho, ls_iters=1, pivot_mode=PIVOT_FP16, dtype=np.float32, diag=False):
    """Fit + quantise one state S [dk, dv].  Returns dict r, c, code, piv (+ tpre, lsgap)."""
    S = _c(S, dtype)
    dk, dv = S.shape
    bits = _c(bits, np.uint8); rho = _c(rho, np.float32)
    r = np.zeros(dk, dtype); c = np.zeros(dv, dtype)
    code = np.zeros((dk, dv), np.int32); piv = np.zeros((dk, dv), dtype)
    tpre = np.zeros((dk, dv), dtype) if diag else None
    gap = np.zeros(dv, dtype) if diag else None
    fn = lib().oracle_fit_quantise_f32 if dtype == np.float32 else lib().oracle_fit_quantise_f64
    fn(dk, dv, _ptr(S), _ptr(bits), _ptr(rho), ls_iters, pivot_mode, _ptr(r), _ptr(c),
       _ptr(code), _ptr(piv), _ptr(tpre), _ptr(gap))
    out = {"r": r, "c": c, "code": code, "piv": piv}
    if diag:
        out["tpre"] = tpre; out["lsgap"] = gap
    return out


def fit_quantise_mode(mode, S, bits, rho, ls_iters=1):
    """Fit variant `mode` (SCALE_*) + quantise one state S [dk, dv] (fp32).
    Returns dict r, c, code, piv, tpre (the pre-rounding values p / c)."""
    S = _c(S, np.float32)
    dk, dv = S.shape
    bits = _c(bits, np.uint8); rho = _c(rho, np.float32)
    r = np.zeros(dk, np.float32); c = np.zeros(dv, np.float32)
    code = np.zeros((dk, dv), np.int32); piv = np.zeros((dk, dv), np.float32)
    tpre = np.zeros((dk, dv), np.float32)
    lib().oracle_fit_quantise_mode_f32(int(mode), dk, dv, _ptr(S), _ptr(bits), _ptr(rho), ls_iters, PIVOT_FP16,
                                       _ptr(r), _ptr(c), _ptr(code), _ptr(piv), _ptr(tpre))
    return {"r": r, "c": c, "code": code, "piv": piv, "tpre": tpre}


def quantise(S, bits, r, c, dtype=np.float32):
    """Codes of S under given scales; returns (code, tpre)."""
    S = _c(S, dtype); bits = _c(bits, np.uint8); r = _c(r, dtype); c = _c(c, dtype)
    dk, dv = S.shape
    code = np.zeros((dk, dv), np.int32); tpre = np.zeros((dk, dv), dtype)
    fn = lib().oracle_quantise_f32 if dtype == np.float32 else lib().oracle_quantise_f64
    fn(dk, dv, _ptr(S), _ptr(bits), _ptr(r), _ptr(c), _ptr(code), _ptr(tpre))
    return code, tpre


def dequant(bits, r, c, code, piv, dtype=np.float32):
    r = _c(r, dtype); c = _c(c, dtype); code = _c(code, np.int32); piv = _c(piv, dtype)
    bits = _c(bits, np.uint8)
    dk, dv = code.shape
    S = np.zeros((dk, dv), dtype)
    fn = lib().oracle_dequant_f32 if dtype == np.float32 else lib().oracle_dequant_f64
    fn(dk, dv, _ptr(bits), _ptr(r), _ptr(c), _ptr(code), _ptr(piv), _ptr(S))
    return S


def update(S, alpha_rows, q, k, v, beta, dtype=np.float32):
    """Gated Delta update of S (copied) + readout.  Returns (S_new, o)."""
    S = _c(S, dtype).copy()
    dk, dv = S.shape
    a = _c(alpha_rows, dtype); q = _c(q, dtype); k = _c(k, dtype); v = _c(v, dtype)
    o = np.zeros(dv, dtype)
    fn = lib().oracle_update_f32 if dtype == np.float32 else lib().oracle_update_f64
    fn(dk, dv, _ptr(S), _ptr(a), _ptr(q), _ptr(k), _ptr(v), float(beta), _ptr(o))
    return S, o


def column_error(S, bits, rho, r, cj, code, j):
    S = _c(S, np.float64); r = _c(r, np.float64); code = _c(code, np.int32)
    bits = _c(bits, np.uint8); rho = _c(rho, np.float32)
    dk, dv = S.shape
    return lib().oracle_column_error_f64(dk, dv, j, _ptr(S), _ptr(bits), _ptr(rho), _ptr(r),
                                         float(cj), _ptr(code))


def to_fp16_bits(x: float) -> int:
    return int(lib().oracle_to_fp16(float(x)))


def from_fp16_bits(h: int) -> float:
    return float(lib().oracle_from_fp16(int(h)))


def item_bytes(bits_head) -> int:
    bits_head = _c(bits_head, np.uint8)
    return int(lib().oracle_item_bytes(bits_head.shape[0], 128, _ptr(bits_head)))


def pack_item(bits, r, c, code, piv, dv=None):
    bits = _c(bits, np.uint8); code = _c(code, np.int32)
    dk, dv_ = code.shape
    out = np.zeros(int(lib().oracle_item_bytes(dk, dv_, _ptr(bits))), np.uint8)
    lib().oracle_pack_item(dk, dv_, _ptr(bits), _ptr(_c(r, np.float32)), _ptr(_c(c, np.float32)),
                           _ptr(code), _ptr(_c(piv, np.float32)), _ptr(out))
    return out


def unpack_item(bits, item, dk, dv):
    bits = _c(bits, np.uint8); item = _c(item, np.uint8)
    r = np.zeros(dk, np.float32); c = np.zeros(dv, np.float32)
    code = np.zeros((dk, dv), np.int32); piv = np.zeros((dk, dv), np.float32)
    lib().oracle_unpack_item(dk, dv, _ptr(bits), _ptr(item), _ptr(r), _ptr(c), _ptr(code), _ptr(piv))
    return {"r": r, "c": c, "code": code, "piv": piv}


class SlotPool:
    """The oracle's compact pool over a list of slots (one (request, head) state each).

    slot_head[s] is the head of slot s; bits and rho are per-head tables [H, dk].
    """

    def __init__(self, slot_head, bits, rho, dk=128, dv=128, ls_iters=1, kda=False, mode=SCALE_DUAL):
        self.mode = int(mode)
        self.slot_head = _c(slot_head, np.int32)
        self.n = int(self.slot_head.shape[0])
        self.bits = _c(bits, np.uint8); self.rho = _c(rho, np.float32)
        self.dk, self.dv, self.ls_iters, self.kda = dk, dv, ls_iters, bool(kda)
        self.nbytes = int(lib().oracle_pool_bytes(self.n, _ptr(self.slot_head), dk, dv, _ptr(self.bits)))
        self.pool = np.zeros(self.nbytes, np.uint8)
        sizes = [item_bytes(self.bits[h]) if dv == 128 else None for h in self.slot_head]
        self.offsets = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64) if self.n else np.zeros(0, np.int64)
        self.sizes = np.asarray(sizes, dtype=np.int64)

    def pack(self, S):
        S = _c(S, np.float32).reshape(self.n, self.dk, self.dv)
        if self.mode != SCALE_DUAL:
            lib().oracle_pack_pool_mode(self.mode, self.n, _ptr(self.slot_head), self.dk, self.dv, _ptr(self.bits),
                                        _ptr(self.rho), self.ls_iters, _ptr(S), _ptr(self.pool))
            return
        lib().oracle_pack_pool(self.n, _ptr(self.slot_head), self.dk, self.dv, _ptr(self.bits),
                               _ptr(self.rho), self.ls_iters, _ptr(S), _ptr(self.pool))

    def unpack(self):
        S = np.zeros((self.n, self.dk, self.dv), np.float32)
        lib().oracle_unpack_pool(self.n, _ptr(self.slot_head), self.dk, self.dv, _ptr(self.bits),
                                 _ptr(self.pool), _ptr(S))
        return S

    def item(self, s):
        return self.pool[self.offsets[s]: self.offsets[s] + self.sizes[s]]

    def set_item(self, s, data):
        self.pool[self.offsets[s]: self.offsets[s] + self.sizes[s]] = data

    def step(self, q, k, v, alpha, beta, diag=False):
        """One decode step.  Inputs are per slot: q, k [n, dk], v [n, dv], beta [n],
        alpha [n] (GDN) or [n, dk] (KDA).  Returns o [n, dv] (+ S_new, tpre, lsgap)."""
        n, dk, dv = self.n, self.dk, self.dv
        q = _c(q, np.float32); k = _c(k, np.float32); v = _c(v, np.float32)
        alpha = _c(alpha, np.float32); beta = _c(beta, np.float32)
        assert alpha.size == (n * dk if self.kda else n)
        out = np.zeros((n, dv), np.float32)
        if self.mode != SCALE_DUAL:  # no least squares: no least-squares gaps
            S_new = np.zeros((n, dk, dv), np.float32) if diag else None
            tpre = np.zeros((n, dk, dv), np.float32) if diag else None
            lib().oracle_decode_step_mode(self.mode, n, _ptr(self.slot_head), dk, dv, _ptr(self.bits),
                                          _ptr(self.rho), self.ls_iters, int(self.kda), _ptr(self.pool), _ptr(q),
                                          _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(out), _ptr(S_new),
                                          _ptr(tpre))
            if diag:
                return out, {"S_new": S_new, "tpre": tpre, "lsgap": np.full((n, dv), np.inf, np.float32)}
            return out
        S_new = np.zeros((n, dk, dv), np.float32) if diag else None
        tpre = np.zeros((n, dk, dv), np.float32) if diag else None
        gap = np.zeros((n, dv), np.float32) if diag else None
        lib().oracle_decode_step(n, _ptr(self.slot_head), dk, dv, _ptr(self.bits), _ptr(self.rho),
                                 self.ls_iters, int(self.kda), _ptr(self.pool), _ptr(q), _ptr(k),
                                 _ptr(v), _ptr(alpha), _ptr(beta), _ptr(out), _ptr(S_new),
                                 _ptr(tpre), _ptr(gap))
        if diag:
            return out, {"S_new": S_new, "tpre": tpre, "lsgap": gap}
        return out


def fp32_step(S, q, k, v, alpha, beta, kda=False):
    """Unquantised fp32 recursion in place on S [n, dk, dv]; returns o [n, dv]."""
    n, dk, dv = S.shape
    assert S.dtype == np.float32 and S.flags.c_contiguous
    out = np.zeros((n, dv), np.float32)
    lib().oracle_fp32_step(n, dk, dv, int(kda), _ptr(S), _ptr(_c(q, np.float32)), _ptr(_c(k, np.float32)),
                           _ptr(_c(v, np.float32)), _ptr(_c(alpha, np.float32)), _ptr(_c(beta, np.float32)),
                           _ptr(out))
    return out


def fp64_step(S, q, k, v, alpha, beta, kda=False):
    """Unquantised fp64 recursion in place on S [n, dk, dv] (float64); returns o."""
    n, dk, dv = S.shape
    assert S.dtype == np.float64 and S.flags.c_contiguous
    out = np.zeros((n, dv), np.float64)
    lib().oracle_fp64_step(n, dk, dv, int(kda), _ptr(S), _ptr(_c(q, np.float64)), _ptr(_c(k, np.float64)),
                           _ptr(_c(v, np.float64)), _ptr(_c(alpha, np.float64)), _ptr(_c(beta, np.float64)),
                           _ptr(out))
    return out


def initial_state(cfg, requests=None, workload=None):
    """S0 of a workload config: the unquantised fp64 recursion run over the
    config's warm-up steps from a zero state, rounded to fp32.  [R, H, dk, dv]."""
    if workload is None:
        from quantized_recurrent_state_sm_b200 import workload
    req = np.arange(cfg.batch) if requests is None else np.asarray(requests)
    R, H = len(req), cfg.heads
    S = np.zeros((R * H, cfg.dk, cfg.dv), np.float64)
    for t in range(-cfg.warmup, 0):
        x = workload.step_inputs(cfg, t, req)
        fp64_step(S, x["q"].reshape(R * H, -1), x["k"].reshape(R * H, -1), x["v"].reshape(R * H, -1),
                  x["alpha"].reshape(R * H, -1) if cfg.variant == 1 else x["alpha"].reshape(-1),
                  x["beta"].reshape(-1), kda=cfg.variant == 1)
    return S.astype(np.float32).reshape(R, H, cfg.dk, cfg.dv)


# ---- calibration (oracle/stepq_oracle_calib.c) -------------------------------

def calib_accumulate(kda, q, alpha, acc_q2, acc_loga):
    """Add one step's sums into acc_q2 [H, dk] and acc_loga ([H] or [H, dk]),
    float64 arrays updated in place.  q [B, H, dk]; alpha [B, H] or [B, H, dk]."""
    q = _c(q, np.float32); alpha = _c(alpha, np.float32)
    B, H, dk = q.shape
    assert acc_q2.dtype == np.float64 and acc_loga.dtype == np.float64
    assert acc_q2.flags.c_contiguous and acc_loga.flags.c_contiguous
    lib().oracle_calib_accumulate(int(kda), B, H, dk, _ptr(q), _ptr(alpha), _ptr(acc_q2), _ptr(acc_loga))


def calib_rho(acc_q2, n_samples):
    acc_q2 = _c(acc_q2, np.float64)
    H, dk = acc_q2.shape
    rho = np.zeros((H, dk), np.float32)
    lib().oracle_calib_rho(H, dk, float(n_samples), _ptr(acc_q2), _ptr(rho))
    return rho


def calib_row_error(S, b, rho, ls_iters=1):
    """(r, c, err) of S [dk, dv] stored with every row at width b."""
    S = _c(S, np.float32); rho = _c(rho, np.float32)
    dk, dv = S.shape
    r = np.zeros(dk, np.float32); c = np.zeros(dv, np.float32); err = np.zeros(dk, np.float64)
    lib().oracle_calib_row_error(dk, dv, _ptr(S), int(b), _ptr(rho), int(ls_iters), _ptr(r), _ptr(c), _ptr(err))
    return r, c, err


def calib_weight(mean_log_alpha):
    return float(lib().oracle_calib_weight(float(mean_log_alpha)))


def calib_allocate(weight, D, choices, avg_bits, n_piv):
    weight = _c(weight, np.float64); D = _c(D, np.float64); ch = _c(choices, np.int32)
    n, nc = D.shape
    bits = np.zeros(n, np.uint8)
    if lib().oracle_calib_allocate(n, _ptr(weight), _ptr(D), nc, _ptr(ch), float(avg_bits), int(n_piv), _ptr(bits)):
        raise ValueError("bit budget below the pivots and the narrowest width")
    return bits


def calib_bits(kda, acc_loga, rho, err, choices, avg_bits, pivot_frac, n_samples):
    """Row widths [H, dk] from the calibration sums; err [H, nc, dk]."""
    rho = _c(rho, np.float32); err = _c(err, np.float64); acc_loga = _c(acc_loga, np.float64)
    ch = _c(choices, np.int32)
    H, nc, dk = err.shape
    bits = np.zeros((H, dk), np.uint8)
    if lib().oracle_calib_bits(int(kda), H, dk, float(n_samples), _ptr(acc_loga), _ptr(rho), _ptr(err), nc,
                               _ptr(ch), float(avg_bits), float(pivot_frac), _ptr(bits)):
        raise ValueError("bit budget below the pivots and the narrowest width")
    return bits


def calibrate(cfg, batch, steps, sample_every, workload=None):
    """The whole calibration on the CPU: impact scores from the calibration
    inputs, then per-row errors at every candidate width of the fp32 rollout's
    states at steps t with (t + 1) % sample_every == 0 (after the step's
    update), then the widths.  Returns dict rho [H, dk], bits [H, dk],
    acc_q2, acc_loga, err [H, nc, dk]."""
    if workload is None:
        from quantized_recurrent_state_sm_b200 import workload
    W = workload
    kda = cfg.variant == 1
    H, dk, dv = cfg.heads, cfg.dk, cfg.dv
    choices = sorted(cfg.bits_choices)
    acc_q2 = np.zeros((H, dk)); acc_loga = np.zeros((H, dk) if kda else (H,))
    for t in range(steps):
        x = W.calibration_inputs(cfg, t, batch)
        calib_accumulate(kda, x["q"], x["alpha"], acc_q2, acc_loga)
    n_samples = batch * steps
    rho = calib_rho(acc_q2, n_samples)
    S = initial_state(cfg, W.calibration_requests(batch), W).reshape(batch * H, dk, dv).copy()
    err = np.zeros((H, len(choices), dk))
    for t in range(steps):
        x = W.calibration_inputs(cfg, t, batch)
        n = batch * H
        fp32_step(S, x["q"].reshape(n, dk), x["k"].reshape(n, dk), x["v"].reshape(n, dv),
                  x["alpha"].reshape(n, dk) if kda else x["alpha"].reshape(n), x["beta"].reshape(n), kda=kda)
        if (t + 1) % sample_every == 0:
            for s in range(n):
                h = s % H
                for xw, b in enumerate(choices):
                    err[h, xw] += calib_row_error(S[s], b, rho[h], cfg.ls_iters)[2]
    bits = calib_bits(kda, acc_loga, rho, err, choices, cfg.avg_bits, cfg.pivot_frac, n_samples)
    return {"rho": rho, "bits": bits, "acc_q2": acc_q2, "acc_loga": acc_loga, "err": err}
