"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Every input is seeded and synthetic (quantized_recurrent_state_sm_b200.workload).
The GPU always runs the whole batch; for the large configurations the oracle
follows requests {0, 1, B/2, B-1} x all heads, whose packed bytes are copied
into the GPU pool before each lockstep step (items are independent, so this is
exact).
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_recurrent_state_sm_b200 import workload as W
from tests.parity import PoolComparison, rel_l2

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from quantized_recurrent_state_sm_b200 import stepq
else:  # pragma: no cover
    stepq = None


def to_dev(x):
    return {k: torch.from_numpy(np.array(v, copy=True)).cuda() for k, v in x.items()}


class Setup:
    """A GPU pool and the oracle's pool over the compared slots."""

    def __init__(self, cfg, requests=None, bits=None, rho=None, mode=0):
        self.cfg = cfg
        self.bits = W.bit_table(cfg) if bits is None else bits
        self.rho = W.rho(cfg) if rho is None else rho
        self.req = np.arange(cfg.batch) if requests is None else np.asarray(requests)
        H = cfg.heads
        self.slots = (self.req[:, None] * H + np.arange(H)[None, :]).reshape(-1)
        self.kda = cfg.variant == W.KDA
        self.gpu = stepq.PackedStatePool(cfg.variant, cfg.batch, H, self.bits, self.rho, cfg.ls_iters)
        if mode:
            self.gpu.set_scale_mode(mode)
        self.ref = oracle.SlotPool(self.slots % H, self.bits, self.rho, ls_iters=cfg.ls_iters, kda=self.kda,
                                   mode=mode)
        offs, total = W.item_offsets(self.bits, 128, cfg.batch)
        assert total == self.gpu.state_nbytes
        self.gpu_off = offs.reshape(-1)[self.slots]

    def slot_inputs(self, x):
        n = len(self.slots)
        sub = {k: v[self.req] for k, v in x.items()}
        return (sub["q"].reshape(n, -1), sub["k"].reshape(n, -1), sub["v"].reshape(n, -1),
                sub["alpha"].reshape(n, -1) if self.kda else sub["alpha"].reshape(-1),
                sub["beta"].reshape(-1))

    def push_oracle_bytes(self):
        """Overwrite the compared GPU items with the oracle's bytes."""
        st = self.gpu.state
        for s in range(len(self.slots)):
            o, n = int(self.gpu_off[s]), int(self.ref.sizes[s])
            st[o:o + n].copy_(torch.from_numpy(self.ref.item(s).copy()))

    def gpu_item(self, host_state, s):
        o, n = int(self.gpu_off[s]), int(self.ref.sizes[s])
        return host_state[o:o + n]

    def head(self, s):
        return self.bits[self.slots[s] % self.cfg.heads]


def lockstep(setup, steps, t0=0, full_inputs=True, step=None, S0=None, ref_bytes=None):
    """`steps` steps from step t0 with the oracle's bytes pushed before each;
    the oracle's pool starts from S0 packed (default: the initial state) or
    from ref_bytes[(request, head)]."""
    cfg = setup.cfg
    cmp = PoolComparison()
    if ref_bytes is not None:
        for s, slot in enumerate(setup.slots):
            setup.ref.set_item(s, ref_bytes[(int(slot // cfg.heads), int(slot % cfg.heads))])
    else:
        if S0 is None:
            S0 = oracle.initial_state(cfg, setup.req)
        setup.ref.pack(S0.reshape(-1, 128, 128))
    worst = 0.0
    for t in range(t0, t0 + steps):
        setup.push_oracle_bytes()
        x = W.step_inputs(cfg, t) if full_inputs else None
        d = to_dev(x)
        if step is None:
            out = setup.gpu.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        else:
            out = step(setup.gpu, d)
        torch.cuda.synchronize()
        o_ref, dg = setup.ref.step(*setup.slot_inputs(x), diag=True)
        o = out.cpu().numpy()[setup.req].reshape(len(setup.slots), -1)
        e = rel_l2(o, o_ref)
        worst = max(worst, e)
        assert e <= 1e-4, f"step {t}: readout rel L2 {e:.3e}"
        host = setup.gpu.state.cpu().numpy()
        for s in range(len(setup.slots)):
            cmp.item(setup.head(s), setup.gpu_item(host, s), setup.ref.item(s), dg["tpre"][s],
                     dg["lsgap"][s], dg["S_new"][s], where=f"step {t} slot {s}")
    cmp.check_fraction()
    setup.gpu.check()  # no kernel reported an error
    return cmp, worst


def test_unpack_is_exact():
    cfg = W.with_overrides(W.CONFIGS[1], batch=3)
    su = Setup(cfg)
    S0 = oracle.initial_state(cfg)
    su.ref.pack(S0.reshape(-1, 128, 128))
    su.push_oracle_bytes()
    got = su.gpu.unpack().cpu().numpy().reshape(-1, 128, 128)
    np.testing.assert_array_equal(got, su.ref.unpack())


@pytest.mark.parametrize("ci", [0, 1, 2, 4])
def test_pack_matches_oracle(ci):
    cfg = W.with_overrides(W.CONFIGS[ci], batch=min(W.CONFIGS[ci].batch, 4))
    su = Setup(cfg)
    S0 = oracle.initial_state(cfg)
    su.gpu.pack(torch.from_numpy(S0).cuda())
    torch.cuda.synchronize()
    host = su.gpu.state.cpu().numpy()
    cmp = PoolComparison()
    for s, flat in enumerate(S0.reshape(-1, 128, 128)):
        bh = su.head(s)
        rh = su.rho[su.slots[s] % cfg.heads]
        fit = oracle.fit_quantise(flat, bh, rh, cfg.ls_iters, diag=True)
        want = oracle.pack_item(bh, fit["r"], fit["c"], fit["code"], fit["piv"])
        cmp.item(bh, su.gpu_item(host, s), want, fit["tpre"], fit["lsgap"], flat, where=f"slot {s}")
    cmp.check_fraction()


def test_lockstep_config0_full():
    cmp, worst = lockstep(Setup(W.CONFIGS[0]), steps=16)
    print(f"config 0: {cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")


@pytest.mark.parametrize("ci,steps", [(1, 3), (2, 3), (4, 2)])
def test_lockstep_subsampled_full_batch(ci, steps):
    cfg = W.CONFIGS[ci]
    cmp, worst = lockstep(Setup(cfg, W.parity_requests(cfg)), steps=steps, t0=100)
    print(f"config {ci}: {cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")


def test_lockstep_config3_full_size_sampled():
    """The serving-scale launch (512 x 48 items) on the oracle's sampled requests."""
    cfg = W.CONFIGS[3]
    cmp, worst = lockstep(Setup(cfg, W.parity_requests(cfg)), steps=2, t0=500)
    print(f"config 3: {cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")


def long_rollout_state(cfg, requests, steps):
    """The oracle's unquantised fp32 recursion from the initial state over the
    first `steps` steps, for the given requests: [R, H, dk, dv]."""
    S = oracle.initial_state(cfg, requests)
    R, H = S.shape[:2]
    Sf = np.ascontiguousarray(S.reshape(R * H, 128, 128))
    kda = cfg.variant == W.KDA
    for t in range(steps):
        x = W.step_inputs(cfg, t, requests)
        oracle.fp32_step(Sf, x["q"].reshape(R * H, -1), x["k"].reshape(R * H, -1), x["v"].reshape(R * H, -1),
                         x["alpha"].reshape(R * H, -1) if kda else x["alpha"].reshape(-1), x["beta"].reshape(-1),
                         kda=kda)
    return Sf.reshape(R, H, 128, 128)


@pytest.mark.parametrize("ci", [0, 1, 2, 3, 4])
def test_lockstep_from_long_rollout_state(ci):
    """Lockstep from the state of each configuration's full-length unquantised
    rollout (64 steps for config 0, 256 for configs 1 and 2, 1024 for config
    3, 2048 for config 4, where the 30x key and value channels have grown
    their outlier rows and columns), 8 steps, on the full batch with the
    oracle on requests {0, 1, B/2, B-1}: the parity rules hold at the
    magnitudes and clip rates of a long rollout."""
    cfg = W.CONFIGS[ci]
    req = W.parity_requests(cfg)
    S_T = long_rollout_state(cfg, req, cfg.steps)
    su = Setup(cfg, req)
    cmp, worst = lockstep(su, steps=8, t0=cfg.steps, S0=S_T)
    rms = np.sqrt(np.mean(S_T.astype(np.float64) ** 2, axis=3))  # row RMS, [R, H, dk]
    print(f"config {ci} after {cfg.steps} steps: row RMS max/median {np.median(rms.max(-1) / np.median(rms, -1)):.1f}; "
          f"{cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")


@pytest.mark.parametrize("ci", [0, 1, 2, 3, 4])
def test_lockstep_from_packed_rollout_state(ci):
    """Lockstep from the oracle's own packed state after each configuration's
    full-length requantised rollout (every step fitted, rounded and packed, so
    the codes carry the accumulated requantisation structure), 8 steps, on the
    full batch with the oracle on requests {0, 1, B/2, B-1}."""
    from tests.drift import oracle_rollout_bytes
    cfg = W.CONFIGS[ci]
    req = W.parity_requests(cfg)
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    S0 = oracle.initial_state(cfg, req)
    s0 = {}
    for a, r in enumerate(req):
        for h in range(cfg.heads):
            f = oracle.fit_quantise(S0[a, h], bits[h], rho[h], cfg.ls_iters)
            s0[(int(r), h)] = oracle.pack_item(bits[h], f["r"], f["c"], f["code"], f["piv"])
    final = oracle_rollout_bytes(ci, [int(r) for r in req], bits, rho, s0, cfg.steps)
    cmp, worst = lockstep(Setup(cfg, req), steps=8, t0=cfg.steps, ref_bytes=final)
    print(f"config {ci} from the packed state after {cfg.steps} steps: {cmp.diff}/{cmp.codes} codes differ, "
          f"worst readout {worst:.2e}")


def test_every_width_and_pivot_rows_kda():
    cfg = W.with_overrides(W.CONFIGS[2], batch=3, heads=2)
    r = np.random.default_rng(0)
    bits = r.choice([2, 3, 4, 5, 6, 7, 8, 16], size=(2, 128)).astype(np.uint8)
    lockstep(Setup(cfg, bits=bits), steps=4)


def test_kda_position_layouts():
    """Row-wise heads whose 16-bit field positions number at most one (the
    kernel that checks only position 0 for pivots): mixed widths without
    pivots, exactly 8 pivot rows (position 0 all pivots), one pivot row (a
    16-bit position shared with 8-bit codes) and a single width."""
    cfg = W.with_overrides(W.CONFIGS[2], batch=3, heads=4)
    r = np.random.default_rng(1)
    bits = np.empty((4, 128), np.uint8)
    bits[0] = r.choice([3, 4, 5, 6, 7, 8], size=128)
    bits[1] = r.choice([2, 5, 8], size=128)
    bits[1, r.choice(128, 8, replace=False)] = 16
    bits[2] = r.choice([4, 6], size=128)
    bits[2, 77] = 16
    bits[3] = 5
    assert max(int(W.position_widths(b)[1]) for b in bits) < 16  # no head has a second 16-bit position
    lockstep(Setup(cfg, bits=bits), steps=4)


@pytest.mark.parametrize("ci", [0, 2])
def test_fp32_baseline_matches_oracle(ci):
    cfg = W.with_overrides(W.CONFIGS[ci], batch=2)
    n = cfg.items
    S0 = oracle.initial_state(cfg)
    S_gpu = torch.from_numpy(S0).cuda()
    S_or = S0.reshape(n, 128, 128).copy()
    kda = cfg.variant == W.KDA
    for t in range(8):
        x = W.step_inputs(cfg, t)
        d = to_dev(x)
        o = stepq.fp32_step(cfg.variant, S_gpu, d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        o_ref = oracle.fp32_step(S_or, x["q"].reshape(n, -1), x["k"].reshape(n, -1), x["v"].reshape(n, -1),
                                 x["alpha"].reshape(n, -1) if kda else x["alpha"].reshape(-1), x["beta"].reshape(-1), kda=kda)
        assert rel_l2(o.cpu().numpy().reshape(n, -1), o_ref) < 1e-5
    assert rel_l2(S_gpu.cpu().numpy().reshape(n, 128, 128), S_or) < 1e-5


def test_zero_state_and_identity_update():
    cfg = W.with_overrides(W.CONFIGS[1], batch=2, heads=8)
    su = Setup(cfg)
    n = cfg.items
    su.gpu.pack(torch.zeros((cfg.batch, cfg.heads, 128, 128), device="cuda"))
    su.ref.pack(np.zeros((n, 128, 128), np.float32))
    torch.cuda.synchronize()
    host = su.gpu.state.cpu().numpy()
    cmp = PoolComparison()
    for s in range(n):
        # every code is zero and every column scale is 1; row scales s_i / Q_i
        cmp.item(su.head(s), su.gpu_item(host, s), su.ref.item(s), where=f"slot {s}")
    assert cmp.diff == 0
    # alpha = 1, beta = 0: the update is the identity and out = S^T q
    x = W.step_inputs(cfg, 0)
    x["alpha"][:] = 1.0
    x["beta"][:] = 0.0
    S0 = oracle.initial_state(cfg)
    su.ref.pack(S0.reshape(n, 128, 128))
    su.push_oracle_bytes()
    Sd = su.ref.unpack()
    d = to_dev(x)
    out = su.gpu.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"]).cpu().numpy().reshape(n, -1)
    want = np.einsum("nij,ni->nj", Sd.astype(np.float64), x["q"].reshape(n, -1).astype(np.float64))
    assert rel_l2(out, want) < 1e-6


def test_empty_batch_is_a_noop():
    cfg = W.with_overrides(W.CONFIGS[0], batch=0)
    pool = stepq.PackedStatePool(cfg.variant, 0, cfg.heads, W.bit_table(cfg), W.rho(cfg))
    assert pool.state_nbytes == 0
    e = torch.empty((0, cfg.heads, 128), device="cuda")
    pool.decode_step(e, e, e, torch.empty((0, cfg.heads), device="cuda"), torch.empty((0, cfg.heads), device="cuda"))
    pool.pack(torch.empty((0, cfg.heads, 128, 128), device="cuda"))
    pool.close()


def test_invalid_arguments_are_rejected_on_the_host():
    cfg = W.with_overrides(W.CONFIGS[0], batch=2)
    pool = stepq.PackedStatePool(cfg.variant, cfg.batch, cfg.heads, W.bit_table(cfg), W.rho(cfg))
    d = to_dev(W.step_inputs(cfg, 0))
    import ctypes as C
    L = stepq.lib
    h = pool._h
    host = np.zeros(cfg.items * 128, np.float32)
    P = lambda t: C.c_void_p(t.data_ptr())
    # host memory where device memory is required
    st = L.stepq_decode_step(h, host.ctypes.data_as(C.c_void_p), P(d["k"]), P(d["v"]), P(d["alpha"]), P(d["beta"]), P(d["v"]))
    assert st == stepq.ERR_INVALID_ARG
    # misaligned tensor
    big = torch.zeros(cfg.items * 128 + 1, device="cuda")
    st = L.stepq_decode_step(h, C.c_void_p(big.data_ptr() + 4), P(d["k"]), P(d["v"]), P(d["alpha"]), P(d["beta"]),
                             P(torch.empty_like(d["v"])))
    assert st == stepq.ERR_INVALID_ARG
    # output aliasing an input
    st = L.stepq_decode_step(h, P(d["q"]), P(d["k"]), P(d["v"]), P(d["alpha"]), P(d["beta"]), P(d["v"]))
    assert st == stepq.ERR_INVALID_ARG
    # shape checks in the binding
    with pytest.raises(ValueError):
        pool.decode_step(d["q"][:1], d["k"], d["v"], d["alpha"], d["beta"])
    pool.close()
    # a destroyed handle
    st = L.stepq_decode_step(h, P(d["q"]), P(d["k"]), P(d["v"]), P(d["alpha"]), P(d["beta"]), P(torch.empty_like(d["v"])))
    assert st == stepq.ERR_STATE
    torch.cuda.synchronize()  # the context is still healthy


@pytest.mark.parametrize("ci,ls", [(1, 0), (1, 2), (3, 3), (2, 0), (2, 3)])
def test_least_squares_round_counts(ci, ls):
    """0 rounds (maximum-based column scales), and several rounds (later
    rounds clip to the row's range)."""
    cfg = W.with_overrides(W.CONFIGS[ci], batch=2, ls_iters=ls)
    lockstep(Setup(cfg), steps=2, t0=7)


def test_every_width_gdn():
    """Gated-DeltaNet heads of every width 2..8 (one instantiation of the
    fused kernel per width) and an all-pivot head in one pool, lockstep."""
    widths = [2, 3, 4, 5, 6, 7, 8, 16]
    cfg = W.with_overrides(W.CONFIGS[1], batch=3, heads=len(widths))
    bits = np.repeat(np.array(widths, np.uint8)[:, None], 128, axis=1)
    cmp, worst = lockstep(Setup(cfg, bits=bits), steps=4, t0=3)
    print(f"widths {widths}: {cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")


@pytest.mark.parametrize("ci,batch,heads", [(0, 1, 1), (1, 5, 3), (2, 1, 1), (2, 7, 5), (4, 3, 33)])
def test_odd_shapes(ci, batch, heads):
    """One request of one head, and item counts that fill the persistent grid
    unevenly (the configuration's generators at that head count; no pivot
    head where a 16-bit unit would not fit the bit budget of so few heads)."""
    cfg = W.with_overrides(W.CONFIGS[ci], batch=batch, heads=heads)
    if cfg.variant == W.GDN and heads < 8:
        cfg = W.with_overrides(cfg, pivot_frac=0.0)
    lockstep(Setup(cfg), steps=3, t0=11)
