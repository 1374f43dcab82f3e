"""Comparison of packed pools produced by the CUDA path and by the oracle.

Acceptance (fp32 arithmetic, sums in a different order on the two sides):
  * readout: relative L2 error over the batch <= 1e-4 at every step;
  * codes: identical, except at most a 1e-4 fraction that differ by exactly
    one step, and only where a rounding decision of the oracle was within a
    relative 1e-5 of a rounding boundary: the final decision itself
    (|t - (n + 1/2)| <= 1e-5 max(1, |t|)), or a least-squares decision of the
    same column (after which that column's scale legitimately differs);
  * row scales within 1e-5 relative; column scales within 1e-5 relative except
    in columns with such a least-squares boundary decision;
  * pivot rows: binary16 values identical except one-ulp differences where the
    oracle's fp32 value lies within 1e-5 of the midpoint of the two, relative
    to the larger of the value and its row's root-mean-square (the update adds
    terms of the row's size, so a small value can carry an error of that
    size's order).
"""
import numpy as np

import oracle

WINDOW = 1e-5
MAX_FRACTION = 1e-4


def boundary_gap(t, Q):
    x = np.clip(t.astype(np.float64), -Q, Q)
    f = x - np.floor(x)
    return np.abs(f - 0.5) / np.maximum(1.0, np.abs(t.astype(np.float64)))


def rel_l2(a, b):
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


class PoolComparison:
    def __init__(self):
        self.codes = 0
        self.diff = 0
        self.items = 0

    @property
    def fraction(self):
        return self.diff / max(1, self.codes)

    def check_fraction(self):
        assert self.diff <= MAX_FRACTION * self.codes, \
            f"{self.diff} of {self.codes} codes differ (> {MAX_FRACTION:g})"

    def item(self, bits_head, got_bytes, want_bytes, tpre=None, lsgap=None, S_new=None, where=""):
        """Compare one item.  tpre, lsgap, S_new: the oracle's diagnostics for it
        (None when the item was produced by a fit without an update, e.g. pack:
        then tpre/lsgap still come from the oracle's fit)."""
        dk = bits_head.shape[0]
        g = oracle.unpack_item(bits_head, got_bytes, dk, 128)
        w = oracle.unpack_item(bits_head, want_bytes, dk, 128)
        self.items += 1
        quant = bits_head != 16
        Q = ((1 << (bits_head.astype(np.int64) - 1)) - 1)[:, None]
        # row scales
        np.testing.assert_allclose(g["r"], w["r"], rtol=WINDOW, atol=0, err_msg=f"row scales {where}")
        # columns with a near-boundary least-squares decision
        free_col = np.zeros(128, bool) if lsgap is None else (lsgap <= WINDOW)
        if quant.any():
            ok_c = np.isclose(g["c"], w["c"], rtol=WINDOW, atol=0) | free_col
            assert ok_c.all(), f"column scales differ {where}: cols {np.flatnonzero(~ok_c)[:8]} " \
                               f"{g['c'][~ok_c][:4]} vs {w['c'][~ok_c][:4]}"
        dcode = g["code"] - w["code"]
        bad = dcode[quant]
        assert np.all(np.abs(bad) <= 1), f"codes differ by more than one step {where}"
        diff = (dcode != 0) & quant[:, None]
        if diff.any():
            assert tpre is not None, f"codes differ and no oracle diagnostics given {where}"
            near = boundary_gap(tpre, Q) <= WINDOW
            allowed = near | free_col[None, :]
            assert np.all(allowed[diff]), \
                f"code differs away from a rounding boundary {where}: {np.argwhere(diff & ~allowed)[:4]}"
        self.codes += int(quant.sum()) * 128
        self.diff += int(diff.sum())
        # pivot rows
        piv = ~quant
        if piv.any():
            hg = g["piv"][piv]; hw = w["piv"][piv]
            neq = hg != hw
            if neq.any():
                assert S_new is not None, f"pivot values differ {where}"
                Sp = S_new[piv].astype(np.float64)
                row_rms = np.sqrt(np.mean(Sp * Sp, axis=1, keepdims=True)) * np.ones_like(Sp)
                x = Sp[neq]
                mid = (hg[neq].astype(np.float64) + hw[neq].astype(np.float64)) / 2
                scale = np.maximum(np.abs(x), row_rms[neq])
                h_ulp = np.abs(hg[neq].astype(np.float64) - hw[neq].astype(np.float64))
                assert np.all(h_ulp <= 2.0 ** -10 * np.maximum(np.abs(hw[neq]), 2.0 ** -14) * 1.001), \
                    f"pivot values differ by more than one binary16 step {where}"
                assert np.all(np.abs(x - mid) <= WINDOW * scale), f"pivot values differ {where}"
                self.codes += 0
                self.diff += int(neq.sum())
            self.codes += int(piv.sum()) * 128
