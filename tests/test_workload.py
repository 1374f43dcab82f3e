"""Host logic: the seeded workload generator and the pool layout arithmetic."""
import numpy as np
import pytest

from quantized_recurrent_state_sm_b200 import workload as W


@pytest.mark.parametrize("ci", [0, 1, 2, 3, 4])
def test_bit_tables_meet_budget(ci):
    cfg = W.CONFIGS[ci]
    bits = W.bit_table(cfg)
    assert bits.shape == (cfg.heads, cfg.dk)
    units = bits[:, 0] if cfg.variant == W.GDN else bits.reshape(-1)
    if cfg.variant == W.GDN:
        assert np.all(bits == bits[:, :1])  # one width per head
    allowed = set(cfg.bits_choices) | {16}
    assert set(np.unique(units).tolist()) <= allowed
    # the nominal average counts FP16 pivots at 16 bits
    assert units.mean() == pytest.approx(cfg.avg_bits, abs=1e-12)
    n_piv = int(np.ceil(cfg.pivot_frac * units.size - 1e-9)) if cfg.pivot_frac > 0 else 0
    assert int((units == 16).sum()) == n_piv
    if n_piv:
        h = W.half_lives(cfg).reshape(-1)
        piv = np.flatnonzero(units == 16)
        assert h[piv].min() >= np.sort(h)[-n_piv]  # the longest half-lives
    # longer-lived units never get fewer bits than shorter-lived ones (non-pivots)
    h = W.half_lives(cfg).reshape(-1)
    m = units != 16
    order = np.argsort(h[m], kind="stable")
    assert np.all(np.diff(units[m][order].astype(int)) >= 0)


def test_step_inputs_deterministic_and_sliceable():
    cfg = W.CONFIGS[1]
    full = W.step_inputs(cfg, 5)
    sub = W.step_inputs(cfg, 5, [0, 17, 63])
    again = W.step_inputs(cfg, 5)
    for k in full:
        np.testing.assert_array_equal(full[k], again[k])
        np.testing.assert_array_equal(full[k][[0, 17, 63]], sub[k])
    np.testing.assert_allclose(np.linalg.norm(full["k"], axis=-1), 1.0, rtol=1e-6)
    np.testing.assert_allclose(np.linalg.norm(full["q"], axis=-1), 1.0, rtol=1e-6)
    assert np.all((full["beta"] > 0) & (full["beta"] < 1))
    assert full["alpha"].shape == (cfg.batch, cfg.heads)
    other = W.step_inputs(cfg, 6)
    assert not np.array_equal(full["v"], other["v"])


def test_normal_moments():
    z = W.normal(W.derive_key(1, 2, 3), np.arange(200000))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_kda_alpha_and_outliers():
    cfg = W.CONFIGS[4]
    x = W.step_inputs(cfg, 0, [0, 1])
    assert x["alpha"].shape == (2, cfg.heads, cfg.dk)
    np.testing.assert_array_equal(x["alpha"][0], W.gates(cfg))
    kg, vg = W.outlier_gains(cfg)
    assert np.all((kg == 30).sum(axis=1) == 3) and np.all((vg == 30).sum(axis=1) == 3)
    # outlier value channels carry ~30x the magnitude of the others
    h = 0
    big = vg[h] == 30
    ratio = np.abs(x["v"][:, h, big]).mean() / np.abs(x["v"][:, h, ~big]).mean()
    assert ratio > 5


def test_pool_layout():
    cfg = W.CONFIGS[3]
    bits = W.bit_table(cfg)
    sz = W.head_item_bytes(bits, cfg.dv)
    assert np.all(sz % 16 == 0)
    offs, total = W.item_offsets(bits, cfg.dv, cfg.batch)
    assert offs[0, 0] == 0 and offs[1, 0] == sz.sum() and offs[0, 1] == sz[0]
    assert total == cfg.batch * sz.sum()
    assert 190e6 < total < 240e6  # "about 200 MB per layer" at batch 512
