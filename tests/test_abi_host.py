"""The C-ABI library on the host: it loads, exports every declared symbol, and
validates descriptors and handles without touching a GPU."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from quantized_recurrent_state_sm_b200 import workload as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def S():
    from quantized_recurrent_state_sm_b200 import build
    build.build()
    from quantized_recurrent_state_sm_b200 import stepq
    return stepq


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"STEPQ_API\s+[\w\s\*]+?\b(stepq_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(S):
    names = declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(S.lib, n), n
    assert set(S.EXPORTS) <= names


def test_pool_bytes_matches_layout(S):
    for ci in range(5):
        cfg = W.CONFIGS[ci]
        bits, rho = W.bit_table(cfg), W.rho(cfg)
        _, total = W.item_offsets(bits, 128, cfg.batch)
        d, keep = S.make_desc(cfg.variant, cfg.batch, cfg.heads, bits, rho)
        assert S.lib.stepq_state_bytes(C.byref(d)) == total
        assert S.lib.stepq_pool_bytes(C.byref(d)) >= total


def test_descriptor_validation(S):
    cfg = W.CONFIGS[1]
    bits, rho = W.bit_table(cfg), W.rho(cfg)

    def nbytes(**kw):
        b = kw.pop("bits", bits); r = kw.pop("rho", rho)
        d, keep = S.make_desc(cfg.variant, cfg.batch, cfg.heads, b, r)
        for k, v in kw.items():
            setattr(d, k, v)
        n = S.lib.stepq_pool_bytes(C.byref(d))
        return n, S.lib.stepq_last_error().decode()

    assert nbytes()[0] > 0
    assert nbytes(variant=7) == (0, nbytes(variant=7)[1]) and "variant" in nbytes(variant=7)[1]
    assert nbytes(dk=64)[0] == 0 and "128" in nbytes(dk=64)[1]
    assert nbytes(batch=-1)[0] == 0
    assert nbytes(heads=0)[0] == 0
    assert nbytes(ls_iters=9)[0] == 0
    bad = bits.copy(); bad[0, 5] = 9
    assert nbytes(bits=bad)[0] == 0
    mixed = bits.copy(); mixed[0, 5] = 3 if mixed[0, 0] != 3 else 4
    n, msg = nbytes(bits=mixed)
    assert n == 0 and "one width per head" in msg
    r2 = rho.copy(); r2[1, 1] = 0.0
    assert nbytes(rho=r2)[0] == 0
    r3 = rho.copy(); r3[1, 1] = np.nan
    assert nbytes(rho=r3)[0] == 0
    d, keep = S.make_desc(cfg.variant, cfg.batch, cfg.heads, bits, rho)
    d.bits = None
    assert S.lib.stepq_pool_bytes(C.byref(d)) == 0
    assert S.lib.stepq_pool_bytes(None) == 0
    # the limits: batch x heads up to 2^24 items, heads up to 65535 (the
    # staging records hold a head in 16 bits)
    top = (1 << 24) // cfg.heads
    d, keep = S.make_desc(cfg.variant, top, cfg.heads, bits, rho)
    states = S.lib.stepq_state_bytes(C.byref(d))
    assert states == top * int(W.head_item_bytes(bits, cfg.dv).sum())  # ~0.2 TB: 64-bit sizes
    assert S.lib.stepq_pool_bytes(C.byref(d)) > states
    n, msg = nbytes(batch=top + 1)
    assert n == 0 and "exceeds" in msg
    H = 65536
    hb = np.full((H, 128), 6, np.uint8)
    hr = np.ones((H, 128), np.float32)
    d, keep = S.make_desc(cfg.variant, 1, H, hb, hr)
    assert S.lib.stepq_pool_bytes(C.byref(d)) == 0 and "65535" in S.lib.stepq_last_error().decode()
    d, keep = S.make_desc(cfg.variant, 1, H - 1, hb[:H - 1], hr[:H - 1])
    assert S.lib.stepq_pool_bytes(C.byref(d)) > 0


def test_null_and_dead_handles(S):
    assert S.lib.stepq_pool_destroy(None) == S.ERR_INVALID_ARG
    assert S.lib.stepq_decode_step(None, None, None, None, None, None, None) == S.ERR_INVALID_ARG
    bogus = C.c_void_p(0x1000)
    assert S.lib.stepq_pack(bogus, None) == S.ERR_STATE
    out = C.c_void_p()
    cfg = W.CONFIGS[0]
    d, keep = S.make_desc(cfg.variant, cfg.batch, cfg.heads, W.bit_table(cfg), W.rho(cfg))
    assert S.lib.stepq_pool_create(C.byref(d), None, 10 ** 9, None, C.byref(out)) == S.ERR_INVALID_ARG
    assert S.lib.stepq_pool_create(C.byref(d), C.c_void_p(16), 16, None, C.byref(out)) == S.ERR_INVALID_ARG
    assert S.lib.stepq_pool_create(C.byref(d), None, 0, None, None) == S.ERR_INVALID_ARG
    assert S.lib.stepq_status_string(3) == b"STEPQ_ERR_CUDA"


def test_calibration_descriptor_validation(S):
    """stepq_calib_scratch_bytes is 0 and stepq_calibrate returns
    STEPQ_ERR_INVALID_ARG / UNSUPPORTED for invalid calibration descriptors,
    on the host, before any device call."""
    widths = np.array([3, 4, 6], np.int32)
    wp = widths.ctypes.data_as(C.c_void_p)

    def desc(**kw):
        d = S.CalibDesc(S.GDN, 4, 8, 128, 128, 16, 8, 1, 3, wp, 4.0, 0.01)
        for k, v in kw.items():
            setattr(d, k, v)
        return d

    assert S.lib.stepq_calib_scratch_bytes(C.byref(desc())) > 0
    bad = [dict(variant=7), dict(dk=64), dict(batch=0), dict(steps=0), dict(sample_every=0),
           dict(sample_every=32), dict(ls_iters=-1), dict(n_widths=0), dict(n_widths=9),
           dict(widths=None), dict(avg_bits=0.0), dict(pivot_frac=1.5)]
    for kw in bad:
        assert S.lib.stepq_calib_scratch_bytes(C.byref(desc(**kw))) == 0, kw
    for ws in ([4, 3], [1, 4], [3, 9], [4, 4]):
        w2 = np.array(ws, np.int32)
        d = desc(n_widths=len(ws), widths=w2.ctypes.data_as(C.c_void_p))
        assert S.lib.stepq_calib_scratch_bytes(C.byref(d)) == 0, ws
    rho = np.zeros(8 * 128, np.float32); bits = np.zeros(8 * 128, np.uint8)
    st = S.lib.stepq_calibrate(C.byref(desc(dk=64)), None, None, None, None, None, None, None, 0, None,
                               rho.ctypes.data_as(C.c_void_p), bits.ctypes.data_as(C.c_void_p))
    assert st == S.ERR_UNSUPPORTED
    st = S.lib.stepq_calibrate(C.byref(desc()), None, None, None, None, None, None, None, 0, None,
                               rho.ctypes.data_as(C.c_void_p), bits.ctypes.data_as(C.c_void_p))
    assert st == S.ERR_INVALID_ARG  # scratch too small, before any pointer is touched


def test_calibration_host_steps_validate(S):
    acc = np.ones((2, 128)); rho = np.ones((2, 128), np.float32)
    with pytest.raises(S.StepqError):
        S.calib_rho(acc, 0.0)
    err = np.ones((2, 3, 128))
    with pytest.raises(S.StepqError):
        S.calib_bits(S.GDN, np.zeros(2), rho, err, [3, 4, 3], 4.0, 0.0, 10.0)  # widths not ascending
    with pytest.raises(S.StepqError):
        S.calib_bits(S.GDN, np.zeros(2), rho, err, [3, 4, 6], 2.0, 0.0, 10.0)  # budget below the narrowest


def test_scale_mode_rejects_unknown(S):
    assert S.lib.stepq_pool_set_scale_mode(None, 0) == S.ERR_INVALID_ARG


def test_layout_agrees_across_implementations(S):
    """Item sizes of random mixed-width heads (pivot rows included) agree
    between the library, the oracle and the workload's format arithmetic:
    the storage-row order and per-position field widths are written three
    times, independently."""
    import oracle
    r = np.random.default_rng(21)
    for trial in range(12):
        H = int(r.integers(1, 6))
        choices = r.choice([2, 3, 4, 5, 6, 7, 8, 16], size=int(r.integers(1, 5)), replace=False)
        bits = r.choice(choices, size=(H, 128)).astype(np.uint8)
        if trial % 3 == 0:
            bits[0] = bits[0, 0]  # one head of a single width (key order)
        rho = np.ones((H, 128), np.float32)
        per_head = [oracle.item_bytes(bits[h]) for h in range(H)]
        _, total = W.item_offsets(bits, 128, 3)
        assert total == 3 * sum(per_head), trial
        d, keep = S.make_desc(S.KDA, 3, H, bits, rho)
        assert S.lib.stepq_state_bytes(C.byref(d)) == total, trial


def test_pool_layout_regions_and_guards(S):
    """stepq_pool_layout: the packed states first, then each table, every
    region followed by its guard region, in order and without overlap; the
    total is stepq_pool_bytes and the states' extent stepq_state_bytes."""
    for ci in range(5):
        cfg = W.with_overrides(W.CONFIGS[ci], batch=3)
        bits, rho = W.bit_table(cfg), W.rho(cfg)
        d, keep = S.make_desc(cfg.variant, cfg.batch, cfg.heads, bits, rho)
        r = S.Regions()
        assert S.lib.stepq_pool_layout(C.byref(d), C.byref(r)) == S.OK
        H, n = cfg.heads, cfg.items
        assert r.states == 0 and r.state_bytes == S.lib.stepq_state_bytes(C.byref(d))
        assert r.total == S.lib.stepq_pool_bytes(C.byref(d))
        g = list(r.guards)
        sizes = [r.state_bytes, None, 8 * H, 4 * H, 4, 4 * n, 16 * n]
        starts = [r.states, r.head_records, r.head_offsets, r.item_sizes, r.status_word, r.item_order,
                  r.staging_records]
        for k in range(7):
            if sizes[k] is not None:
                assert starts[k] + sizes[k] <= g[k], (ci, k)
            assert g[k] % 16 == 0 and g[k] + r.guard_bytes <= (starts[k + 1] if k < 6 else r.total), (ci, k)
        assert starts[1] % 256 == 0 and all(x % 16 == 0 for x in starts)
    assert S.lib.stepq_pool_layout(None, C.byref(r)) == S.ERR_INVALID_ARG


def test_selftest_bounded_wait_arguments(S):
    """Argument checks of the wait self-test happen on the host."""
    assert S.lib.stepq_selftest_bounded_wait(None, 1000, 0, None) == S.ERR_INVALID_ARG
    assert S.lib.stepq_selftest_bounded_wait(C.c_void_p(16), -1, 0, None) == S.ERR_INVALID_ARG
    assert S.lib.stepq_selftest_bounded_wait(C.c_void_p(16), (1 << 34) + 1, 0, None) == S.ERR_INVALID_ARG
    assert "limit_cycles" in S.lib.stepq_last_error().decode()
