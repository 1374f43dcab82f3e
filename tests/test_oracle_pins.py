"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, an independent matrix formulation, an invariant of the recurrence, a
library routine, or brute force on a tiny case.  Pages cited:
  ai.info summary of STEPQuant ("Key Contributions", "Main Findings",
  "Methodology in Plain English"); ai-papers.net article ("STEPQuantの仕組み");
  ai-trend.me review ("핵심 용어").
"""
import math

import numpy as np
import pytest

import oracle
from quantized_recurrent_state_sm_b200 import workload as W


def rng(seed):
    return np.random.default_rng(seed)


def unit(x):
    return x / np.linalg.norm(x)


# --------------------------------------------------------------------------
# IEEE binary16 rounding (pivot storage) against numpy's float16 conversion
# --------------------------------------------------------------------------

def test_fp16_rounding_matches_numpy():
    r = rng(1)
    xs = np.concatenate([
        r.standard_normal(20000) * 10.0 ** r.uniform(-9, 5, 20000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -24, 2.0 ** -25,
                  3 * 2.0 ** -26, 2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, np.inf, -np.inf]),
    ])
    for x in xs:
        h = oracle.to_fp16_bits(x)
        with np.errstate(over="ignore"):
            ref = int(np.array([x], np.float64).astype(np.float16).view(np.uint16)[0])
        assert h == ref, (x, hex(h), hex(ref))
        back = oracle.from_fp16_bits(h)
        want = float(np.array([ref], np.uint16).view(np.float16)[0])
        assert back == want or (math.isnan(back) and math.isnan(want))


# --------------------------------------------------------------------------
# (a) every unit a pivot: the packed recursion is the unquantised one
# --------------------------------------------------------------------------

def matrix_delta_rule(S, alpha_rows, q, k, v, beta):
    """Textbook matrix form: S <- (I - beta k k^T) diag(alpha) S + beta k v^T, o = S^T q."""
    dk = S.shape[0]
    A = (np.eye(dk) - beta * np.outer(k, k)) @ np.diag(alpha_rows)
    Sn = A @ S + beta * np.outer(k, v)
    return Sn, Sn.T @ q


@pytest.mark.parametrize("kda", [False, True])
def test_all_pivot_exact_storage_is_unquantised_recursion(kda):
    r = rng(2)
    dk, dv = 32, 24
    bits = np.full(dk, 16, np.uint8)
    rho = np.ones(dk, np.float32)
    S = r.standard_normal((dk, dv))
    S_ref = S.copy()
    for t in range(20):
        alpha = r.uniform(0.3, 1.0, dk) if kda else np.full(dk, r.uniform(0.3, 1.0))
        q, k = unit(r.standard_normal(dk)), unit(r.standard_normal(dk))
        v = r.standard_normal(dv); beta = r.uniform(0, 1)
        st = oracle.fit_quantise(S, bits, rho, pivot_mode=oracle.PIVOT_EXACT, dtype=np.float64)
        Sd = oracle.dequant(bits, st["r"], st["c"], st["code"], st["piv"], dtype=np.float64)
        assert np.array_equal(Sd, S)  # exact pivot storage round-trips bit for bit
        S, o = oracle.update(Sd, alpha, q, k, v, beta, dtype=np.float64)
        S_ref, o_ref = matrix_delta_rule(S_ref, alpha, q, k, v, beta)
        np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-12 * np.abs(S_ref).max())
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12 * np.abs(o_ref).max())


def test_all_pivot_fp16_error_obeys_contraction_bound():
    """With FP16 pivots the error is transported previous error plus new rounding
    error ("Methodology in Plain English"), and the transition has spectral norm
    <= 1 ("Main Findings"), so ||E_t|| <= sum of the per-step rounding errors."""
    r = rng(3)
    dk, dv = 16, 16
    bits = np.full(dk, 16, np.uint8); rho = np.ones(dk, np.float32)
    S_exact = r.standard_normal((dk, dv)) * 3
    Sq = S_exact.copy()
    bound = 0.0
    for t in range(30):
        st = oracle.fit_quantise(Sq, bits, rho, dtype=np.float64)
        Sd = oracle.dequant(bits, st["r"], st["c"], st["code"], st["piv"], dtype=np.float64)
        bound += np.linalg.norm(Sd - Sq)
        alpha = np.full(dk, r.uniform(0.5, 1.0))
        q, k = unit(r.standard_normal(dk)), unit(r.standard_normal(dk))
        v = r.standard_normal(dv); beta = r.uniform(0, 1)
        Sq, _ = oracle.update(Sd, alpha, q, k, v, beta, dtype=np.float64)
        S_exact, _ = matrix_delta_rule(S_exact, alpha, q, k, v, beta)
        assert np.linalg.norm(Sq - S_exact) <= bound * (1 + 1e-9) + 1e-12


# --------------------------------------------------------------------------
# (b) unit-norm key, beta = 1: the new state maps k exactly onto v
# --------------------------------------------------------------------------

@pytest.mark.parametrize("kda", [False, True])
def test_exact_projection_beta_one(kda):
    r = rng(4)
    dk, dv = 128, 128
    S = r.standard_normal((dk, dv))
    alpha = r.uniform(0.2, 1.0, dk) if kda else np.full(dk, 0.9)
    k = unit(r.standard_normal(dk)); q = unit(r.standard_normal(dk)); v = r.standard_normal(dv)
    Sn, o = oracle.update(S, alpha, q, k, v, 1.0, dtype=np.float64)
    np.testing.assert_allclose(Sn.T @ k, v, rtol=0, atol=1e-12 * np.abs(v).max())


# --------------------------------------------------------------------------
# (c) requantising a dequantised state with frozen scales returns its codes
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_requantise_fixed_point(dtype):
    r = rng(5)
    dk = dv = 128
    bits = r.choice([2, 3, 4, 5, 6, 7, 8], size=dk).astype(np.uint8)
    bits[r.choice(dk, 3, replace=False)] = 16
    rho = np.exp(r.standard_normal(dk)).astype(np.float32)
    S = (r.standard_normal((dk, dv)) * np.exp(r.standard_normal((dk, 1)))).astype(dtype)
    st = oracle.fit_quantise(S, bits, rho, dtype=dtype)
    Sd = oracle.dequant(bits, st["r"], st["c"], st["code"], st["piv"], dtype=dtype)
    code2, _ = oracle.quantise(Sd, bits, st["r"], st["c"], dtype=dtype)
    assert np.array_equal(code2, st["code"])


# --------------------------------------------------------------------------
# (d) generated gates have the drawn half-life
# --------------------------------------------------------------------------

@pytest.mark.parametrize("ci", [0, 2])
def test_gate_half_life(ci):
    cfg = W.CONFIGS[ci]
    h = W.half_lives(cfg)
    a64 = W.gates64(cfg)
    assert h.min() >= 1.0 and h.max() <= 4096.0
    np.testing.assert_allclose(a64 ** h, 0.5, rtol=0, atol=1e-12)
    a32 = W.gates(cfg).astype(np.float64)
    assert np.all(np.abs(a32 ** h - 0.5) <= 0.5 * h * 2.0 ** -24 * 1.01)


# --------------------------------------------------------------------------
# (e) brute-force column scales at dk = dv = 4
# --------------------------------------------------------------------------

def brute_force_column(p, w, Q, dk):
    """Exact minimum over c > 0 of sum_i w_i (p_i - c n_i(c))^2 with
    n_i(c) = clamp(rne(p_i / c)): the codes are piecewise constant in c with
    breakpoints c = |p_i| / (m + 1/2); inside a piece the error is a quadratic."""
    bps = {0.0}
    for i in range(dk):
        for m in range(Q[i]):
            if p[i] != 0:
                bps.add(abs(p[i]) / (m + 0.5))
    bps = sorted(bps) + [math.inf]
    best = math.inf
    for lo, hi in zip(bps[:-1], bps[1:]):
        mid = (lo + hi) / 2 if hi < math.inf else lo * 2 + 1
        n = np.clip(np.round(p / mid), -Q, Q)
        den = float(np.sum(w * n * n))
        cands = [mid]
        if den > 0:
            cands.append(min(max(float(np.sum(w * n * p)) / den, lo), hi if hi < math.inf else 1e300))
        for c in cands:
            if c <= 0 or c == math.inf:
                continue
            e = float(np.sum(w * (p - c * n) ** 2))
            best = min(best, e)
    return best


def test_bruteforce_column_scales_small():
    r = rng(6)
    ratios = []
    for trial in range(200):
        dk = dv = 4
        bits = r.choice([2, 3, 4], size=dk).astype(np.uint8)
        rho = np.exp(r.standard_normal(dk)).astype(np.float32)
        S = r.standard_normal((dk, dv)) * np.exp(r.standard_normal((1, dv)))
        st = oracle.fit_quantise(S, bits, rho, dtype=np.float64)
        Q = (1 << (bits.astype(int) - 1)) - 1
        w = rho.astype(np.float64) * st["r"] ** 2
        p = S / st["r"][:, None]
        for j in range(dv):
            e_fit = oracle.column_error(S, bits, rho, st["r"], st["c"][j], st["code"], j)
            e_opt = brute_force_column(p[:, j], w, Q, dk)
            assert e_fit >= e_opt - 1e-12 * max(1.0, e_opt)
            ratios.append(e_fit / e_opt if e_opt > 0 else 1.0)
    # the fixed-iteration fit is a heuristic; it must stay close to optimal on average
    assert np.median(ratios) < 1.5


# --------------------------------------------------------------------------
# the least-squares step and the final quantiser are each optimal
# --------------------------------------------------------------------------

def test_fit_stages_monotone_and_ls_optimal():
    r = rng(7)
    dk = dv = 64
    bits = r.choice([3, 4, 6, 8], size=dk).astype(np.uint8)
    rho = np.exp(1.5 * r.standard_normal(dk)).astype(np.float32)
    S = r.standard_normal((dk, dv)) * np.exp(r.standard_normal((dk, 1))) * np.exp(r.standard_normal((1, dv)))
    st0 = oracle.fit_quantise(S, bits, rho, ls_iters=0, dtype=np.float64, diag=True)
    st1 = oracle.fit_quantise(S, bits, rho, ls_iters=1, dtype=np.float64)
    np.testing.assert_array_equal(st0["r"], st1["r"])
    Q = (1 << (bits.astype(int) - 1)) - 1
    # the initial column scale maps each column's largest element to the end code
    t0 = st0["tpre"]
    assert np.all(np.abs(t0) <= Q[:, None] * (1 + 1e-12))
    np.testing.assert_allclose(np.max(np.abs(t0) / Q[:, None], axis=0), 1.0, rtol=1e-12)
    for j in range(dv):
        e_init = oracle.column_error(S, bits, rho, st0["r"], st0["c"][j], st0["code"], j)
        e_ls = oracle.column_error(S, bits, rho, st1["r"], st1["c"][j], st0["code"], j)
        e_fin = oracle.column_error(S, bits, rho, st1["r"], st1["c"][j], st1["code"], j)
        assert e_ls <= e_init * (1 + 1e-12) + 1e-300
        assert e_fin <= e_ls * (1 + 1e-12) + 1e-300
        for f in (1 - 1e-4, 1 + 1e-4, 0.9, 1.1):
            e_pert = oracle.column_error(S, bits, rho, st1["r"], st1["c"][j] * f, st0["code"], j)
            assert e_pert >= e_ls * (1 - 1e-12)
    # each final code is the nearest level of its clamped grid
    p = S / st1["r"][:, None]
    t = p / st1["c"][None, :]
    dist = np.abs(t - st1["code"])
    assert np.all(dist <= 0.5 + 1e-9) or np.all((dist <= 0.5 + 1e-9) | (np.abs(st1["code"]) == Q[:, None]))


def test_row_scale_direction_and_invariances():
    """Row scale grows with the row's magnitude and shrinks with its impact score
    ("Methodology in Plain English"); the codes do not depend on a common
    power-of-four factor on all impact weights or a power-of-two factor on the
    whole state."""
    r = rng(8)
    dk = dv = 32
    bits = np.full(dk, 6, np.uint8)
    rho = np.exp(r.standard_normal(dk)).astype(np.float32)
    S = r.standard_normal((dk, dv)).astype(np.float32)
    base = oracle.fit_quantise(S, bits, rho)
    S2 = S.copy(); S2[3] *= 3.0
    assert oracle.fit_quantise(S2, bits, rho)["r"][3] > base["r"][3]
    # four times the largest weight halves that row's scale (exactly: powers of 4)
    top = int(np.argmax(rho))
    rho2 = rho.copy(); rho2[top] *= 4.0
    assert oracle.fit_quantise(S, bits, rho2)["r"][top] == base["r"][top] / 2
    # a row already at the impact floor keeps its scale when its weight falls
    low = int(np.argmin(rho))
    assert rho[low] < rho.max() / 4
    rho3 = rho.copy(); rho3[low] *= 0.5
    np.testing.assert_array_equal(oracle.fit_quantise(S, bits, rho3)["r"], base["r"])
    # common factor 16 on the weights: r halves, c doubles, codes unchanged (exact)
    st = oracle.fit_quantise(S, bits, rho * 16)
    np.testing.assert_array_equal(st["code"], base["code"])
    np.testing.assert_array_equal(st["r"], base["r"] / 4)
    np.testing.assert_array_equal(st["c"], base["c"] * 4)
    # the whole state scaled by 8: r scales by 8, c and the codes are unchanged (exact)
    st3 = oracle.fit_quantise(S * 8, bits, rho)
    np.testing.assert_array_equal(st3["code"], base["code"])
    np.testing.assert_array_equal(st3["r"], base["r"] * 8)
    np.testing.assert_array_equal(st3["c"], base["c"])


def test_row_scale_hand_worked():
    """Row scales worked by hand on rows whose root mean square, mean absolute
    value and maximum all differ, with the impact floor binding on two rows
    and a pivot row's weight ignored ("Methodology in Plain English": the
    scale grows with the row's magnitude and shrinks with its impact score;
    the magnitude is the row's RMS, the measure "Main Findings" uses).
        row 0 = [1, -1, 2, 4]: RMS sqrt(22/4), mean |.| 2, max 4; rho 16 (the largest) -> s = 1/4
        row 1 = [0, 3, 0, -4]: RMS 5/2, mean |.| 7/4, max 4; rho 1 < 16/4 -> s = 4^-1/2 = 1/2
        row 2 = [2, 2, 2, 2]:  RMS 2; rho 1/2 -> floored, s = 1/2
        row 3: a pivot row with rho 1000, outside the fit and the floor
    r_i = RMS_i s_i / Q_i with Q = 7, 7, 31 (widths 4, 4, 6)."""
    S = np.array([[1, -1, 2, 4], [0, 3, 0, -4], [2, 2, 2, 2], [9, 9, 9, 9]], np.float64)
    bits = np.array([4, 4, 6, 16], np.uint8)
    rho = np.array([16, 1, 0.5, 1000], np.float32)
    st = oracle.fit_quantise(S, bits, rho, dtype=np.float64)
    expect = [np.sqrt(5.5) * 0.25 / 7, 2.5 * 0.5 / 7, 2.0 * 0.5 / 31, 0.0]
    np.testing.assert_allclose(st["r"], expect, rtol=1e-15, atol=0)
    # the same rows in fp32: the scales round once per operation
    st32 = oracle.fit_quantise(S, bits, rho)
    np.testing.assert_allclose(st32["r"], expect, rtol=2e-7, atol=0)


def test_higher_impact_rows_reconstruct_better():
    """Rows whose errors matter more receive finer resolution ("Key Contributions")."""
    r = rng(9)
    dk = dv = 128
    bits = np.full(dk, 4, np.uint8)
    rho = np.ones(dk, np.float32); rho[:64] = 8.0
    errs_hi, errs_lo = [], []
    for trial in range(5):
        S = r.standard_normal((dk, dv))
        st = oracle.fit_quantise(S, bits, rho, dtype=np.float64)
        Sd = oracle.dequant(bits, st["r"], st["c"], st["code"], st["piv"], dtype=np.float64)
        e = np.sum((Sd - S) ** 2, axis=1)
        errs_hi.append(e[:64].mean()); errs_lo.append(e[64:].mean())
    assert np.mean(errs_hi) < np.mean(errs_lo)


def test_single_row_is_exact():
    """With one key row every column maps its element to the end code, so the
    stored form reproduces the row up to rounding of the scales."""
    r = rng(10)
    for b in (3, 5, 8):
        S = r.standard_normal((1, 64)) * 7
        st = oracle.fit_quantise(S, np.array([b], np.uint8), np.array([2.5], np.float32), dtype=np.float64)
        Q = (1 << (b - 1)) - 1
        assert np.all(np.abs(st["code"]) == Q)
        Sd = oracle.dequant(np.array([b], np.uint8), st["r"], st["c"], st["code"], st["piv"], dtype=np.float64)
        np.testing.assert_allclose(Sd, S, rtol=1e-14)


def test_zero_state_and_degenerate_columns():
    dk = dv = 16
    bits = np.full(dk, 5, np.uint8); rho = np.ones(dk, np.float32)
    st = oracle.fit_quantise(np.zeros((dk, dv)), bits, rho)
    assert np.all(st["code"] == 0) and np.all(st["c"] == 1.0)
    np.testing.assert_allclose(st["r"], 1.0 / 15, rtol=1e-7)
    S = np.zeros((dk, dv), np.float32); S[:, 3] = 1.0
    st = oracle.fit_quantise(S, bits, rho)
    assert np.all(st["code"][:, [0, 1, 2]] == 0) and np.all(st["code"][:, 3] == 15)


# --------------------------------------------------------------------------
# packed byte format: an independent big-integer formulation of the bit stream
# --------------------------------------------------------------------------

def stream_words(fields, nwords):
    """Independent formulation of one column-group stream: a big integer with
    field m (value, width) at bit sum of the previous widths, cut into words."""
    acc, pos = 0, 0
    for val, width in fields:
        acc |= int(val) << pos
        pos += width
    return [(acc >> (32 * w)) & 0xFFFFFFFF for w in range(nwords)]


def test_storage_rows_balance_widths():
    """Every row group of a mixed-width head holds rows of nearly the same
    widths (the deal of the sorted rows), and a one-width head keeps key order."""
    assert list(W.storage_rows(np.full(128, 5, np.uint8))) == list(range(128))
    r = rng(5)
    bits = r.choice([3, 4, 5, 6, 7, 8, 16], size=128).astype(np.uint8)
    key_of = W.storage_rows(bits)
    assert sorted(key_of) == list(range(128))
    groups = bits[key_of].astype(int).reshape(8, 16)
    # row rr of every group: consecutive ranks, so widths differ by at most one step
    assert np.all(groups.max(axis=0) - groups.min(axis=0) <= 16 - 8)
    assert groups.sum(axis=1).max() - groups.sum(axis=1).min() <= 16


def test_pack_format_slab_streams():
    r = rng(11)
    dk, dv = 128, 128
    bits = r.choice([2, 3, 4, 5, 6, 7, 8, 16], size=dk).astype(np.uint8)
    code = np.zeros((dk, dv), np.int32); piv = np.zeros((dk, dv), np.float32)
    for i, b in enumerate(bits):
        if b == 16:
            piv[i] = r.standard_normal(dv).astype(np.float16).astype(np.float32)
        else:
            Q = (1 << (int(b) - 1)) - 1
            code[i] = r.integers(-Q, Q + 1, dv)
    rr = r.standard_normal(dk).astype(np.float32); cc = r.standard_normal(dv).astype(np.float32)
    item = oracle.pack_item(bits, rr, cc, code, piv)
    # storage rows: widths differ, so the key rows sorted (widest first, ties
    # by index) are dealt to the 8 row groups in turn
    ranked = sorted(range(dk), key=lambda i: (-int(bits[i]), i))
    key_of = [0] * dk
    for j, i in enumerate(ranked):
        key_of[16 * (j % 8) + j // 8] = i
    # position p of every row group stores F_p-bit fields, F_p the widest row
    # at that position; W = ceil(4 sum F_p / 32)
    F = [max(int(bits[key_of[16 * g + t]]) for g in range(8)) for t in range(16)]
    Wh = (4 * sum(F) + 31) // 32
    # the deal puts the widest row of every position in group 0, so W is also
    # the most words any group would need with fields of its rows' own widths
    assert Wh == max((4 * sum(int(bits[key_of[16 * g + t]]) for t in range(16)) + 31) // 32 for g in range(8))
    assert item.size == 4 * dk + 4 * dv + 8 * 32 * 4 * Wh
    assert bytes(item[:4 * dk]) == rr[key_of].astype("<f4").tobytes()
    assert bytes(item[4 * dk: 4 * dk + 4 * dv]) == cc.astype("<f4").tobytes()
    words = item[4 * dk + 4 * dv:].view("<u4")
    for s_ in range(8):
        slab = words[s_ * 32 * Wh:(s_ + 1) * 32 * Wh].reshape(Wh, 32)  # word m of stream l at 32 m + l
        for l in range(32):
            g, cg = l % 8, l // 8
            fields = []
            for rho_ in range(16):
                i = key_of[16 * g + rho_]
                b = int(bits[i])
                for k in range(4):
                    j = 16 * s_ + 4 * cg + k
                    if b == 16:
                        fields.append((int(np.array([piv[i, j]], "<f2").view("<u2")[0]), 16))
                    else:
                        u = code[i, j] + (1 << (F[rho_] - 1))
                        assert 1 <= u <= (1 << F[rho_]) - 1
                        fields.append((u, F[rho_]))
            assert list(slab[:, l]) == stream_words(fields, Wh), (s_, l)
    back = oracle.unpack_item(bits, item, dk, dv)
    np.testing.assert_array_equal(back["code"], code)
    np.testing.assert_array_equal(back["piv"], piv)
    np.testing.assert_array_equal(back["r"], rr)


def test_golden_pack_streams():
    """Hand-derived streams (tests/golden/pack_streams.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "pack_streams.txt")
    n = 0
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        b_s, pat, hex_s = [x.strip() for x in line.split("|")]
        b = int(b_s)
        bits = np.full(128, b, np.uint8)
        code = np.zeros((128, 128), np.int32)
        if pat.startswith("all"):
            code[:] = int(pat.split()[1])
        else:
            assert pat == "rowramp"
            code[:] = (np.arange(128) % 16 % 15 - 7)[:, None]
        item = oracle.pack_item(bits, np.zeros(128), np.zeros(128), code, np.zeros((128, 128)))
        want = [int(x, 16) for x in hex_s.split()]
        words = item[1024:].view("<u4")
        Wh = len(want)
        assert words.size == 8 * 32 * Wh
        for s_ in range(8):
            slab = words[s_ * 32 * Wh:(s_ + 1) * 32 * Wh].reshape(Wh, 32)
            for l in (0, 7, 13, 31):
                assert list(slab[:, l]) == want, (line, s_, l)
        n += 1
    assert n >= 5


# --------------------------------------------------------------------------
# the packed decode step: update-then-requantise, error recursion
# --------------------------------------------------------------------------

def test_decode_step_matches_matrix_form_and_error_recursion():
    """The packed step reconstructs, updates (matrix form), reads out from the
    unquantised new state, and requantises; so the error against an exact
    recursion obeys E_t = A_t E_(t-1) + eps_t ("Methodology in Plain English")."""
    cfg = W.with_overrides(W.CONFIGS[2], batch=2, heads=3)
    bits = W.bit_table(cfg); rho = W.rho(cfg)
    n = cfg.items
    P = oracle.SlotPool(np.arange(n) % cfg.heads, bits, rho, kda=True)
    S0 = oracle.initial_state(cfg).reshape(n, 128, 128)
    P.pack(S0)
    S_exact = P.unpack().astype(np.float64)
    for t in range(6):
        x = W.step_inputs(cfg, t)
        Sd = P.unpack().astype(np.float64)
        E_prev = Sd - S_exact
        q = x["q"].reshape(n, -1); k = x["k"].reshape(n, -1); v = x["v"].reshape(n, -1)
        al = x["alpha"].reshape(n, -1); be = x["beta"].reshape(-1)
        o, dg = P.step(q, k, v, al, be, diag=True)
        S_after = P.unpack().astype(np.float64)
        for s in range(n):
            Sm, om = matrix_delta_rule(Sd[s], al[s].astype(np.float64), q[s].astype(np.float64),
                                       k[s].astype(np.float64), v[s].astype(np.float64), float(be[s]))
            np.testing.assert_allclose(dg["S_new"][s], Sm, rtol=0, atol=2e-6 * np.abs(Sm).max())
            np.testing.assert_allclose(o[s], om, rtol=0, atol=2e-6 * np.abs(om).max())
            A = (np.eye(128) - be[s] * np.outer(k[s], k[s])) @ np.diag(al[s].astype(np.float64))
            S_exact_s, _ = matrix_delta_rule(S_exact[s], al[s].astype(np.float64), q[s].astype(np.float64),
                                             k[s].astype(np.float64), v[s].astype(np.float64), float(be[s]))
            eps = S_after[s] - dg["S_new"][s]
            E_pred = A @ E_prev[s] + eps
            E_true = S_after[s] - S_exact_s
            assert np.linalg.norm(E_true - E_pred) <= 1e-5 * np.linalg.norm(S_exact_s)
            S_exact[s] = S_exact_s


def test_more_bits_less_drift():
    cfg = W.CONFIGS[0]
    n = cfg.items
    S0 = oracle.initial_state(cfg).reshape(n, 128, 128)
    rho = W.rho(cfg)
    drift = {}
    for b in (3, 8):
        bits = np.full((cfg.heads, 128), b, np.uint8)
        P = oracle.SlotPool(np.arange(n) % cfg.heads, bits, rho)
        P.pack(S0)
        Sf = S0.copy()
        for t in range(4):
            x = W.step_inputs(cfg, t)
            args = [x[m].reshape(n, -1) for m in "qkv"] + [x["alpha"].reshape(-1), x["beta"].reshape(-1)]
            P.step(*args)
            oracle.fp32_step(Sf, *args)
        drift[b] = np.linalg.norm(P.unpack() - Sf) / np.linalg.norm(Sf)
    assert drift[8] < drift[3] / 8


def test_fp32_recursion_close_to_fp64():
    r = rng(12)
    n, dk, dv = 3, 128, 128
    S32 = r.standard_normal((n, dk, dv)).astype(np.float32)
    S64 = S32.astype(np.float64)
    for t in range(10):
        q = np.stack([unit(r.standard_normal(dk)) for _ in range(n)])
        k = np.stack([unit(r.standard_normal(dk)) for _ in range(n)])
        v = r.standard_normal((n, dv)); a = r.uniform(0.5, 1, (n, dk)); b = r.uniform(0, 1, n)
        o32 = oracle.fp32_step(S32, q, k, v, a, b, kda=True)
        o64 = oracle.fp64_step(S64, q, k, v, a, b, kda=True)
    assert np.linalg.norm(S32 - S64) / np.linalg.norm(S64) < 1e-5
    assert np.linalg.norm(o32 - o64) / np.linalg.norm(o64) < 1e-5


def test_golden_pack_streams_mixed_widths():
    """Hand-derived streams of a mixed-width head (tests/golden/pack_streams_mixed.txt):
    pins the storage-row order and the per-position field widths."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "pack_streams_mixed.txt")
    want = None
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            want = [int(x, 16) for x in line.split()]
    bits = np.array([4] * 64 + [2] * 64, np.uint8)
    code = np.zeros((128, 128), np.int32)
    key = np.arange(128)
    code[:64] = ((key[:64] // 8) % 7 - 3)[:, None]
    code[64:] = 1
    item = oracle.pack_item(bits, np.ones(128), np.ones(128), code, np.zeros((128, 128)))
    words = item[1024:].view("<u4")
    Wh = len(want)
    assert words.size == 8 * 32 * Wh
    for s_ in range(8):
        slab = words[s_ * 32 * Wh:(s_ + 1) * 32 * Wh].reshape(Wh, 32)
        for l in range(32):
            assert list(slab[:, l]) == want, (s_, l)
    back = oracle.unpack_item(bits, item, 128, 128)
    np.testing.assert_array_equal(back["code"], code)


def test_golden_pack_streams_pivot_position():
    """Hand-derived streams of a head with one pivot row
    (tests/golden/pack_streams_pivot.txt): binary16 fields and 16-bit codes
    sharing the leading position."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "pack_streams_pivot.txt")
    want = {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            g, hx = [x.strip() for x in line.split("|")]
            want[g] = [int(x, 16) for x in hx.split()]
    bits = np.full(128, 8, np.uint8); bits[5] = 16
    code = np.ones((128, 128), np.int32); code[5] = 0
    piv = np.zeros((128, 128), np.float32); piv[5] = 1.0
    item = oracle.pack_item(bits, np.ones(128), np.ones(128), code, piv)
    Wh = len(want["0"])
    words = item[1024:].view("<u4")
    assert words.size == 8 * 32 * Wh
    for s_ in range(8):
        slab = words[s_ * 32 * Wh:(s_ + 1) * 32 * Wh].reshape(Wh, 32)
        for l in range(32):
            assert list(slab[:, l]) == want["0" if l % 8 == 0 else "other"], (s_, l)
    back = oracle.unpack_item(bits, item, 128, 128)
    np.testing.assert_array_equal(back["code"], code)
    np.testing.assert_array_equal(back["piv"], piv)
