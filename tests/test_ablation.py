"""Ablation variants of the scale fit (row scales only, column scales only,
one scale per state) next to the method's dual-axis fit.

CPU: the oracle's variants pinned to their definitions on exact cases, and
the two-axis claim on a state with outliers along both axes.  GPU: pack and
lockstep decode in every variant against the oracle, with the method's
acceptance rules (no least squares: no least-squares boundary columns).
"""
import numpy as np
import pytest

import oracle
from quantized_recurrent_state_sm_b200 import workload as W

ROW, COL, HEAD = oracle.SCALE_ROW, oracle.SCALE_COL, oracle.SCALE_HEAD


def rng(seed):
    return np.random.default_rng(seed)


def rel_err(S, f, bits):
    Sh = oracle.dequant(bits, f["r"], f["c"], f["code"], f["piv"])
    return float(np.linalg.norm(S.astype(np.float64) - Sh) / np.linalg.norm(S))


def test_row_mode_definition():
    """c = 1; r_i = max_j |S_ij| / Q_i, so each row's largest element maps to
    +-Q_i; a zero row gets r = 1 / Q_i."""
    r_ = rng(1)
    S = (r_.standard_normal((128, 128)) * r_.lognormal(0, 1, (128, 1))).astype(np.float32)
    S[5] = 0
    bits = r_.choice([3, 4, 6, 8], 128).astype(np.uint8)
    f = oracle.fit_quantise_mode(ROW, S, bits, np.ones(128, np.float32))
    Q = (1 << (bits.astype(int) - 1)) - 1
    np.testing.assert_array_equal(f["c"], 1.0)
    m = np.abs(S).max(axis=1)
    m[5] = 1.0
    np.testing.assert_array_equal(f["r"], (m / Q).astype(np.float32))
    arg = np.abs(S).argmax(axis=1)
    for i in range(128):
        if i != 5:
            assert abs(f["code"][i, arg[i]]) == Q[i]
    assert np.all(f["code"][5] == 0)


def test_col_and_head_mode_definition():
    """r_i = 1 / Q_i (rounded once); COL: c_j = the column's largest |S_ij| (up
    to the two roundings of S / r / Q); HEAD: every c_j the largest of them.
    Pivot rows are stored as binary16 and take no part."""
    r_ = rng(2)
    S = (r_.standard_normal((128, 128)) * r_.lognormal(0, 1, (1, 128))).astype(np.float32)
    bits = r_.choice([3, 5, 7, 16], 128).astype(np.uint8)
    quant = bits != 16
    Q = (1 << (bits.astype(int) - 1)) - 1
    fc = oracle.fit_quantise_mode(COL, S, bits, np.ones(128, np.float32))
    fh = oracle.fit_quantise_mode(HEAD, S, bits, np.ones(128, np.float32))
    for f in (fc, fh):
        np.testing.assert_array_equal(f["r"][quant], (1.0 / Q[quant]).astype(np.float32))
        np.testing.assert_array_equal(f["r"][~quant], 0)
        np.testing.assert_array_equal(f["piv"][~quant], S[~quant].astype(np.float16).astype(np.float32))
    cmax = np.abs(S[quant]).max(axis=0)
    np.testing.assert_allclose(fc["c"], cmax, rtol=3e-7)
    np.testing.assert_array_equal(fh["c"], fc["c"].max())
    assert np.abs(fc["code"][quant]).max() <= Q[quant].max()


def test_zero_state_in_every_variant():
    S = np.zeros((128, 128), np.float32)
    bits = np.full(128, 4, np.uint8)
    for mode in (ROW, COL, HEAD):
        f = oracle.fit_quantise_mode(mode, S, bits, np.ones(128, np.float32))
        np.testing.assert_array_equal(f["c"], 1.0)
        np.testing.assert_array_equal(f["r"], np.float32(1 / 7))
        assert np.all(f["code"] == 0)


def test_two_axis_outliers_need_both_scales():
    """A state with outliers along key rows and value columns at once (the
    pages' observation): the dual-axis fit beats row-only and column-only
    scaling, and both beat one scale per state."""
    r_ = rng(3)
    for trial in range(4):
        rg = r_.lognormal(0, 1.2, (128, 1)); cg = r_.lognormal(0, 1.2, (1, 128))
        S = (r_.standard_normal((128, 128)) * rg * cg).astype(np.float32)
        bits = np.full(128, 4, np.uint8); rho = np.ones(128, np.float32)
        e_dual = rel_err(S, oracle.fit_quantise(S, bits, rho), bits)
        e_row = rel_err(S, oracle.fit_quantise_mode(ROW, S, bits, rho), bits)
        e_col = rel_err(S, oracle.fit_quantise_mode(COL, S, bits, rho), bits)
        e_head = rel_err(S, oracle.fit_quantise_mode(HEAD, S, bits, rho), bits)
        assert e_dual < min(e_row, e_col) and max(e_row, e_col) < e_head, (e_dual, e_row, e_col, e_head)


def test_dual_mode_is_the_method():
    r_ = rng(4)
    S = r_.standard_normal((128, 128)).astype(np.float32)
    bits = r_.choice([3, 4, 6], 128).astype(np.uint8); rho = r_.lognormal(0, 1, 128).astype(np.float32)
    a = oracle.fit_quantise_mode(oracle.SCALE_DUAL, S, bits, rho)
    b = oracle.fit_quantise(S, bits, rho)
    for k in ("r", "c", "code", "piv"):
        np.testing.assert_array_equal(a[k], b[k])


# ---- GPU --------------------------------------------------------------------

def small_config(ci):
    """Config ci at batch 3 with 8 Gated-DeltaNet or 4 KDA heads (no pivot head
    at 8 heads of config 3's 4-bit budget, where a 16-bit head would not fit)."""
    cfg = W.with_overrides(W.CONFIGS[ci], batch=3, heads=8 if W.CONFIGS[ci].variant == W.GDN else 4)
    return W.with_overrides(cfg, pivot_frac=0.0) if ci == 3 else cfg


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [ROW, COL, HEAD])
@pytest.mark.parametrize("ci", [1, 2, 3, 4])
def test_gpu_pack_variants(mode, ci):
    import torch
    from tests.parity import PoolComparison
    from tests.test_gpu_parity import Setup
    cfg = small_config(ci)
    su = Setup(cfg, mode=mode)
    S0 = oracle.initial_state(cfg)
    su.gpu.pack(torch.from_numpy(S0).cuda())
    torch.cuda.synchronize()
    host = su.gpu.state.cpu().numpy()
    cmp = PoolComparison()
    for s, flat in enumerate(S0.reshape(-1, 128, 128)):
        bh = su.head(s)
        rh = su.rho[su.slots[s] % cfg.heads]
        fit = oracle.fit_quantise_mode(mode, flat, bh, rh, cfg.ls_iters)
        want = oracle.pack_item(bh, fit["r"], fit["c"], fit["code"], fit["piv"])
        cmp.item(bh, su.gpu_item(host, s), want, fit["tpre"], None, flat, where=f"slot {s}")
    cmp.check_fraction()


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [ROW, COL, HEAD])
@pytest.mark.parametrize("ci", [1, 2, 3, 4])
def test_gpu_decode_variants(mode, ci):
    from tests.test_gpu_parity import Setup, lockstep
    cfg = small_config(ci)
    cmp, worst = lockstep(Setup(cfg, mode=mode), steps=3)
    print(f"config {ci} mode {mode}: {cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")


def test_low_impact_row_is_coarsened_by_at_most_one_bit():
    """The impact floor of the row scale: however small a row's impact weight,
    its step is at most twice the step it would get at its head's largest
    weight (here 1, so the floor is 1/4 and the factor is exactly 2).  Such a
    row keeps codes up to about half its range and its reconstruction keeps the
    row's norm within 1 %.  Without the bound, a weight of 1/289 among rows of
    weight 1 put the row's values below one step of the shared column scales;
    rounding then inflated it by about 9 %, and the refit, which follows the
    row's magnitude, repeated that gain every step of a rollout."""
    r_ = rng(12)
    for rho0 in (1.0, 1.0 / 289, 1e-6):
        ratios = []
        for trial in range(20):
            S = r_.standard_normal((128, 128)).astype(np.float32)
            bits = np.full(128, 6, np.uint8)
            rho = np.ones(128, np.float32); rho[0] = rho0
            f = oracle.fit_quantise(S, bits, rho)
            ref = oracle.fit_quantise(S, bits, np.ones(128, np.float32))
            assert f["r"][0] == (ref["r"][0] if rho0 == 1.0 else 2 * ref["r"][0])
            np.testing.assert_array_equal(f["r"][1:], ref["r"][1:])
            Sh = oracle.dequant(bits, f["r"], f["c"], f["code"], f["piv"])
            ratios.append(np.linalg.norm(Sh[0]) / np.linalg.norm(S[0]))
            assert np.abs(f["code"][0]).max() >= (24 if rho0 == 1.0 else 12)
        assert 0.99 < np.mean(ratios) < 1.01, (rho0, np.mean(ratios))


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [ROW, HEAD])
def test_gpu_decode_variants_many_pivot_rows(mode):
    """The variants on the KDA kernel that checks every row position for
    pivot rows (a head with more than 8 pivot rows, so 16-bit fields at two
    positions or more), in lockstep with the oracle."""
    from tests.test_gpu_parity import Setup, lockstep
    cfg = W.with_overrides(W.CONFIGS[2], batch=3, heads=2)
    r_ = np.random.default_rng(7)
    bits = r_.choice([3, 4, 5, 6, 7, 8], size=(2, 128)).astype(np.uint8)
    bits[0, r_.choice(128, 20, replace=False)] = 16
    assert W.position_widths(bits[0])[2] == 16  # a third 16-bit position
    cmp, worst = lockstep(Setup(cfg, bits=bits, mode=mode), steps=3)
    print(f"mode {mode}, 20 pivot rows: {cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")
