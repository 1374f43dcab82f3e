"""Calibration of the tables (impact scores, lifetime-weighted widths).

CPU: the oracle pinned to closed forms, an exact case, the allocation
stand-in it generalises and brute force; the library's host steps against the
oracle bit for bit.  GPU: the statistics, per-row error and reduction kernels
against the oracle, and the whole stepq_calibrate against the oracle's
allocation of the same sums.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from quantized_recurrent_state_sm_b200 import workload as W


def rng(seed):
    return np.random.default_rng(seed)


# ---- oracle pins (CPU) -------------------------------------------------------

def test_accumulate_closed_form():
    """Constant q and alpha: the sums are batch * q^2 and batch * log alpha."""
    B, H, dk = 5, 3, 128
    q = np.full((B, H, dk), 0.25, np.float32)
    for kda in (False, True):
        alpha = np.full((B, H, dk) if kda else (B, H), 0.5, np.float32)
        acc_q2 = np.zeros((H, dk)); acc_la = np.zeros((H, dk) if kda else (H,))
        oracle.calib_accumulate(kda, q, alpha, acc_q2, acc_la)
        oracle.calib_accumulate(kda, q, alpha, acc_q2, acc_la)
        np.testing.assert_array_equal(acc_q2, 2 * B * 0.0625)
        np.testing.assert_allclose(acc_la, 2 * B * math.log(0.5), rtol=1e-15)


def test_rho_mean_and_floor():
    acc = np.array([[8.0] * 127 + [0.0]])
    rho = oracle.calib_rho(acc, 4.0)
    assert rho[0, 0] == 2.0 and rho[0, 127] == np.float32(1e-30)


def test_weight_closed_form():
    for a in (0.5, 0.9, 0.999):
        assert abs(oracle.calib_weight(math.log(a)) - 1.0 / (1.0 - a * a)) <= 1e-9 / (1.0 - a * a)
    assert oracle.calib_weight(0.0) == 1e12  # a unit that never decays: the floor


def test_row_error_rank_one_state_is_exact():
    """S_ij = x_i s_j with s_j = +-1 and rho = 1: every row's scale puts its
    values on +-Q exactly, the column scales stay 1, and the stored form
    reproduces S up to the fp32 rounding of r (error ~ (2^-24 Q)^2 per element)."""
    r_ = rng(3)
    x = r_.lognormal(0.0, 1.0, 128).astype(np.float32)
    s = np.where(r_.random(128) < 0.5, -1.0, 1.0).astype(np.float32)
    S = (x[:, None] * s[None, :]).astype(np.float32)
    for b in (2, 3, 4, 6, 8):
        Q = (1 << (b - 1)) - 1
        r, c, err = oracle.calib_row_error(S, b, np.ones(128, np.float32))
        np.testing.assert_array_equal(c, 1.0)
        assert np.all(err <= (x.astype(np.float64) ** 2) * 128 * (Q * 2.0 ** -23) ** 2), b


def test_row_error_falls_with_width():
    """Random states: more bits, less error (every row, two widths apart)."""
    r_ = rng(4)
    S = (r_.standard_normal((128, 128)) * r_.lognormal(0, 1, (128, 1))).astype(np.float32)
    rho = r_.lognormal(0, 1, 128).astype(np.float32)
    errs = [oracle.calib_row_error(S, b, rho)[2] for b in range(2, 9)]
    for lo, hi in zip(errs[:-2], errs[2:]):
        assert np.all(hi < lo)
    # rows of one scale, rho = 1: at 8 bits the codes are fine everywhere and
    # the error is uniform rounding noise, step^2 / 12 per element
    G = r_.standard_normal((128, 128)).astype(np.float32)
    r8, c8, e8 = oracle.calib_row_error(G, 8, np.ones(128, np.float32))
    step2 = (r8[:, None].astype(np.float64) * c8[None, :]) ** 2
    ratio = e8.sum() / (step2.sum() / 12.0)
    assert 0.9 < ratio < 1.1, ratio


def test_allocate_reduces_to_the_stand_in():
    """With D_u(b) = 4^-b the calibrated allocation is the fixed-table stand-in
    (workload.allocate_bits): the risk w 4^-min orders units as their
    half-lives do, and the gains are the stand-in's."""
    for ci in (1, 2, 3, 4):
        cfg = W.CONFIGS[ci]
        hl = W.half_lives(cfg).reshape(-1)
        alpha = W.gates64(cfg).reshape(-1)
        w = np.array([oracle.calib_weight(math.log(a)) for a in alpha])
        ch = sorted(cfg.bits_choices)
        D = np.array([[4.0 ** -b for b in ch]] * hl.size)
        n_piv = int(math.ceil(cfg.pivot_frac * hl.size - 1e-9)) if cfg.pivot_frac > 0 else 0
        got = oracle.calib_allocate(w, D, ch, cfg.avg_bits, n_piv)
        order = np.lexsort((np.arange(hl.size), -hl))
        want = W.allocate_bits(w, ch, cfg.avg_bits, n_piv, order)
        np.testing.assert_array_equal(got, want, err_msg=f"config {ci}")


def test_allocate_optimal_on_convex_distortions():
    """Unit-cost upgrades of separable convex distortions: the greedy reaches
    the brute-force minimum of sum w D under the budget."""
    r_ = rng(7)
    ch = [3, 4, 5, 6]
    for trial in range(20):
        n = 4
        drops = np.sort(r_.random((n, 3)) * 10, axis=1)[:, ::-1]  # decreasing gains = convex D
        D = np.concatenate([np.full((n, 1), 40.0), 40.0 - np.cumsum(drops, axis=1)], axis=1)
        w = r_.lognormal(0, 1, n)
        avg = r_.choice([3.25, 3.5, 4.0, 4.75])
        got = oracle.calib_allocate(w, D, ch, avg, 0)
        budget = round(avg * n)
        best = min(sum(w[u] * D[u, ch.index(b[u])] for u in range(n))
                   for b in itertools.product(ch, repeat=n) if sum(b) <= budget)
        obj = sum(w[u] * D[u, ch.index(int(got[u]))] for u in range(n))
        assert int(got.sum()) <= budget
        assert abs(obj - best) <= 1e-9 * abs(best), (trial, got, obj, best)


def test_allocate_hand_example():
    """Three units, widths {3, 4, 6}, budget round(3 x 28/3) = 28 bits with
    one pivot.  The pivot is the largest w D(3): unit 1 (2 x 9 = 18 against 10
    and 8).  16 + 3 + 3 = 22 leaves 6 bits.  Gains: unit 2 3->4 is
    1 x (8 - 2) / 1 = 6 against unit 0's 1 x (10 - 7) = 3: unit 2 -> 4 (5
    left).  Unit 0's 3 against unit 2's 4->6, (2 - 1) / 2 = 0.5: unit 0 -> 4
    (4 left).  Unit 0's 4->6, (7 - 6) / 2 = 0.5, ties unit 2's 0.5: the lower
    index, unit 0 -> 6 (2 left); then unit 2 -> 6 (0 left)."""
    w = np.array([1.0, 2.0, 1.0])
    D = np.array([[10.0, 7.0, 6.0], [9.0, 1.0, 0.5], [8.0, 2.0, 1.0]])
    bits = oracle.calib_allocate(w, D, [3, 4, 6], 28.0 / 3.0, 1)
    assert list(bits) == [6, 16, 6]
    # one bit less: the last upgrade no longer fits
    assert list(oracle.calib_allocate(w, D, [3, 4, 6], 27.0 / 3.0, 1)) == [6, 16, 4]
    with pytest.raises(ValueError):
        oracle.calib_allocate(w, D, [3, 4, 6], 5.0, 1)  # 16 + 3 + 3 > 15


def test_calib_bits_units():
    """Gated-DeltaNet units are heads (D = sum_i rho_i err_i, one width per
    head); KDA units are key rows (D = rho_i err_i)."""
    r_ = rng(9)
    H, dk, ch = 3, 128, [3, 4, 6]
    rho = r_.lognormal(0, 1, (H, dk)).astype(np.float32)
    err = np.sort(r_.random((H, 3, dk)), axis=1)[:, ::-1].copy()
    acc_la = np.log(np.array([0.9, 0.99, 0.5])) * 10
    bits = oracle.calib_bits(False, acc_la, rho, err, ch, 4.0, 0.0, 10)
    assert np.all(bits == bits[:, :1])
    w = np.array([oracle.calib_weight(m) for m in acc_la / 10])
    D = (rho[:, None, :].astype(np.float64) * err).sum(axis=2)
    np.testing.assert_array_equal(bits[:, 0], oracle.calib_allocate(w, D, ch, 4.0, 0))
    acc_k = np.repeat(acc_la[:, None], dk, axis=1)
    bk = oracle.calib_bits(True, acc_k, rho, err, ch, 4.0, 0.01, 10)
    wk = np.repeat(w, dk)
    Dk = (rho[:, :, None].astype(np.float64) * err.transpose(0, 2, 1)).reshape(H * dk, 3)
    np.testing.assert_array_equal(bk.reshape(-1), oracle.calib_allocate(wk, Dk, ch, 4.0, 4))


def test_oracle_calibrate_recovers_query_weights():
    """With planted per-row query gains the impact scores follow them: rows of
    larger gain get larger rho (rank correlation over the head's rows)."""
    cfg = W.with_overrides(W.CONFIGS[1], heads=8, q_gain_sigma=1.0)
    out = oracle.calibrate(cfg, batch=2, steps=16, sample_every=8)
    g2 = W.query_gains(cfg) ** 2
    for h in range(8):
        ra = np.argsort(np.argsort(out["rho"][h])); rb = np.argsort(np.argsort(g2[h]))
        corr = np.corrcoef(ra, rb)[0, 1]
        assert corr > 0.8, corr
    assert out["bits"].shape == (8, 128)
    units = out["bits"][:, 0].astype(int)
    assert np.all(out["bits"] == out["bits"][:, :1]) and units.sum() <= round(cfg.avg_bits * 8)


def test_workload_calibration_inputs_are_separate():
    cfg = W.CONFIGS[1]
    a = W.calibration_inputs(cfg, 0, 2)
    b = W.step_inputs(cfg, 0, np.arange(2))
    assert not np.array_equal(a["q"], b["q"])
    # no query gains configured: q is the plain normalised draw
    assert W.query_gains(cfg).min() == 1.0 == W.query_gains(cfg).max()


# ---- the library's host steps against the oracle (CPU) -----------------------

def _random_sums(kda, H, nW, seed):
    r_ = rng(seed)
    dk = 128
    acc_q2 = r_.random((H, dk)) * 3
    acc_la = np.log(r_.uniform(0.5, 0.9999, (H, dk) if kda else (H,))) * 7
    err = np.sort(r_.random((H, nW, dk)), axis=1)[:, ::-1].copy() * r_.lognormal(0, 1, (H, 1, 1))
    return acc_q2, acc_la, err


@pytest.mark.parametrize("kda", [False, True])
def test_library_host_steps_match_oracle(kda):
    from quantized_recurrent_state_sm_b200 import stepq
    ch = [3, 4, 5, 6, 7, 8]
    for seed in range(4):
        H = (16 if not kda else 4) if seed < 3 else 32  # the last: a full 32-head KDA table, 4096 units
        acc_q2, acc_la, err = _random_sums(kda, H, len(ch), seed)
        rho_l = stepq.calib_rho(acc_q2, 7.0)
        rho_o = oracle.calib_rho(acc_q2, 7.0)
        np.testing.assert_array_equal(rho_l, rho_o)
        for avg, frac in ((4.0, 0.0), (6.0, 0.02), (5.5, 0.1)):
            bl = stepq.calib_bits(stepq.KDA if kda else stepq.GDN, acc_la, rho_l, err, ch, avg, frac, 7.0)
            bo = oracle.calib_bits(kda, acc_la, rho_o, err, ch, avg, frac, 7.0)
            np.testing.assert_array_equal(bl, bo)
    with pytest.raises(stepq.StepqError):
        stepq.calib_bits(stepq.GDN, acc_la[:1] if not kda else acc_la[:1, 0], rho_l[:1], err[:1], ch, 3.0, 1.0, 7.0)


# ---- GPU kernels against the oracle -----------------------------------------

def _rollout_states(cfg, batch, steps):
    """fp32 states of the calibration requests after `steps` oracle steps."""
    H, dk, dv = cfg.heads, cfg.dk, cfg.dv
    kda = cfg.variant == 1
    S = oracle.initial_state(cfg, W.calibration_requests(batch)).reshape(batch * H, dk, dv).copy()
    n = batch * H
    for t in range(steps):
        x = W.calibration_inputs(cfg, t, batch)
        oracle.fp32_step(S, x["q"].reshape(n, dk), x["k"].reshape(n, dk), x["v"].reshape(n, dv),
                         x["alpha"].reshape(n, dk) if kda else x["alpha"].reshape(n), x["beta"].reshape(n), kda=kda)
    return S.reshape(batch, H, dk, dv)


@pytest.mark.gpu
@pytest.mark.parametrize("ci", [1, 2])
def test_gpu_calib_accumulate(ci):
    import torch
    from quantized_recurrent_state_sm_b200 import stepq
    cfg = W.with_overrides(W.CONFIGS[ci], heads=8, q_gain_sigma=0.7)
    kda = cfg.variant == 1
    H = cfg.heads
    acc_q2 = torch.zeros((H, 128), dtype=torch.float64, device="cuda")
    acc_la = torch.zeros((H, 128) if kda else (H,), dtype=torch.float64, device="cuda")
    o_q2 = np.zeros((H, 128)); o_la = np.zeros((H, 128) if kda else (H,))
    for t in range(3):
        x = W.calibration_inputs(cfg, t, 6)
        stepq.calib_accumulate(cfg.variant, torch.from_numpy(x["q"]).cuda(), torch.from_numpy(x["alpha"]).cuda(),
                               acc_q2, acc_la)
        oracle.calib_accumulate(kda, x["q"], x["alpha"], o_q2, o_la)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(acc_q2.cpu().numpy(), o_q2)  # exact products, one summation order
    np.testing.assert_allclose(acc_la.cpu().numpy(), o_la, rtol=1e-14)  # log: each side's libm


@pytest.mark.gpu
@pytest.mark.parametrize("ci,ls", [(1, 1), (2, 1), (3, 2), (4, 1)])
def test_gpu_calib_row_error(ci, ls):
    """Per-row errors, r' and c of every candidate width against the oracle.
    r': relative 2e-5 (fp32 fits whose sums run in another order, and the
    GPU's approximate reciprocals).  c: the same, except a column whose
    least-squares round met a code at a rounding boundary: that code goes the
    other way on one side and moves N_j / D_j by one code's share (at most 2
    such columns of 128 per fit, each within 2e-3).  Errors: relative 5e-3 per
    row; an element whose code rounds the other way near a half-step keeps
    |p - c code| near half a step either way, and the rest moves by the scale
    differences times Q (at most 127 x 2e-5).  In a fit with a boundary
    column, that column's elements move by up to 2e-3 x Q c_j, a quarter step
    at Q = 127, against the row's ~dv / 12 squared steps: relative 3e-2."""
    import torch
    from quantized_recurrent_state_sm_b200 import stepq
    cfg = W.with_overrides(W.CONFIGS[ci], heads=4, ls_iters=ls)
    B = 3
    S = _rollout_states(cfg, B, 4)
    rho = W.rho(cfg)
    widths = [2, 3, 4, 5, 6, 7, 8]
    worst_b = 0.0
    err, rc = stepq.calib_row_error(torch.from_numpy(S).cuda(), torch.from_numpy(rho).cuda(), widths, ls)
    err = err.cpu().numpy(); rc = rc.cpu().numpy()
    worst = 0.0
    for b in range(B):
        for h in range(cfg.heads):
            for x, w in enumerate(widths):
                r, c, e = oracle.calib_row_error(S[b, h], w, rho[h], ls)
                np.testing.assert_allclose(rc[b, h, x, :128], r, rtol=2e-5)
                rc_rel = np.abs(rc[b, h, x, 128:] - c) / np.abs(c)
                assert np.sum(rc_rel > 2e-5) <= 2 and rc_rel.max() <= 2e-3, (b, h, w, rc_rel.max())
                rel = np.abs(err[b, h, x] - e) / e
                if rc_rel.max() > 2e-5:
                    worst_b = max(worst_b, rel.max())
                    assert rel.max() <= 3e-2, (b, h, w, rel.max())
                else:
                    worst = max(worst, rel.max())
    print(f"config {ci}: worst per-row relative error difference {worst:.2e} "
          f"({worst_b:.2e} in fits with a least-squares boundary column)")
    assert worst <= 5e-3


@pytest.mark.gpu
@pytest.mark.parametrize("ci", [1, 2, 4])
def test_gpu_calibrate_end_to_end(ci):
    """stepq_calibrate: rho identical to the oracle's (same exact sums); the
    widths equal the oracle's allocation of the GPU's own error sums (taken
    with the piecewise calls), and agree with the whole oracle calibration
    except where two units' gains lie within the fp32 error noise."""
    import torch
    from quantized_recurrent_state_sm_b200 import stepq
    cfg = W.with_overrides(W.CONFIGS[ci], heads=8 if ci == 1 else 2, q_gain_sigma=0.7)
    kda = cfg.variant == 1
    B, T, every = 4, 16, 8
    H = cfg.heads
    xs = [W.calibration_inputs(cfg, t, B) for t in range(T)]
    dev = {k: torch.from_numpy(np.stack([x[k] for x in xs])).cuda() for k in xs[0]}
    S0 = torch.from_numpy(oracle.initial_state(cfg, W.calibration_requests(B))).cuda()
    ch = sorted(cfg.bits_choices)
    rho, bits = stepq.calibrate(cfg.variant, S0, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], ch,
                                cfg.avg_bits, cfg.pivot_frac, every, cfg.ls_iters)
    ref = oracle.calibrate(cfg, B, T, every)
    np.testing.assert_array_equal(rho, ref["rho"])
    # the GPU's sums by the piecewise calls, allocated by the oracle
    acc_q2 = torch.zeros((H, 128), dtype=torch.float64, device="cuda")
    acc_la = torch.zeros((H, 128) if kda else (H,), dtype=torch.float64, device="cuda")
    for t in range(T):
        stepq.calib_accumulate(cfg.variant, dev["q"][t], dev["alpha"][t], acc_q2, acc_la)
    S = S0.clone()
    err_sum = torch.zeros((H, len(ch), 128), dtype=torch.float64, device="cuda")
    rho_d = torch.from_numpy(rho).cuda()
    for t in range(T):
        stepq.fp32_step(cfg.variant, S, dev["q"][t], dev["k"][t], dev["v"][t], dev["alpha"][t], dev["beta"][t])
        if (t + 1) % every == 0:
            err, _ = stepq.calib_row_error(S, rho_d, ch, cfg.ls_iters)
            stepq.calib_reduce(err, err_sum)
    torch.cuda.synchronize()
    la = acc_la.cpu().numpy(); es = err_sum.cpu().numpy()
    want = oracle.calib_bits(kda, la, rho, es, ch, cfg.avg_bits, cfg.pivot_frac, B * T)
    np.testing.assert_array_equal(bits, want)
    np.testing.assert_allclose(es, ref["err"], rtol=5e-3)
    units = bits if kda else bits[:, :1]
    agree = np.mean(units == (ref["bits"] if kda else ref["bits"][:, :1]))
    print(f"config {ci}: widths agree with the full oracle calibration on {agree:.3f} of units")
    assert agree >= 0.9
