"""Decode over an active subset of the pool's requests (stepq_pool_set_active),
the slot-indexed pool of a serving runtime: the active requests' items match
the oracle's pool over exactly those slots (lockstep, the parity rules of the
full step), the inactive requests' input rows are never read, their output
rows never written and their states left untouched; the subset step also
equals the full step bit for bit on the active items."""
import numpy as np
import pytest
import torch

from quantized_recurrent_state_sm_b200 import workload as W

pytestmark = pytest.mark.gpu


def _pool(stepq, cfg):
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    return stepq.PackedStatePool(cfg.variant, cfg.batch, cfg.heads, bits, rho, cfg.ls_iters)


@pytest.mark.parametrize("ci", [1, 2, 3, 4])
def test_active_subset_matches_oracle(ci):
    from tests.test_gpu_parity import Setup, lockstep
    cfg = W.with_overrides(W.CONFIGS[ci], batch=6)
    active = [4, 0, 3]
    inactive = [1, 2, 5]
    su = Setup(cfg, requests=active)  # the oracle follows exactly the active slots
    g = torch.Generator(device="cuda").manual_seed(ci)
    su.gpu.pack(torch.randn((cfg.batch, cfg.heads, 128, 128), device="cuda", generator=g) * 0.2)
    su.gpu.set_active(active)
    offs, total = W.item_offsets(su.bits, 128, cfg.batch)
    per_req = int(np.asarray(offs).reshape(cfg.batch, cfg.heads)[1, 0])

    def step(gpu, d):
        before = gpu.state.clone()
        xp = {k: v.clone() for k, v in d.items()}
        for k in xp:
            xp[k][inactive] = float("nan")  # never read
        out = torch.full((cfg.batch, cfg.heads, 128), -7.0, device="cuda")
        gpu.decode_step(xp["q"], xp["k"], xp["v"], xp["alpha"], xp["beta"], out)
        torch.cuda.synchronize()
        assert bool((out[inactive] == -7.0).all())  # never written
        for b in inactive:
            seg = slice(b * per_req, (b + 1) * per_req)
            assert torch.equal(gpu.state[seg], before[seg]), b
        return out

    cmp, worst = lockstep(su, steps=3, t0=50, step=step)
    print(f"config {ci}, active {active}: {cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")


@pytest.mark.parametrize("ci", [1, 2])
def test_active_subset_matches_full_step(ci):
    from quantized_recurrent_state_sm_b200 import stepq
    cfg = W.with_overrides(W.CONFIGS[ci], batch=6)
    full, part = _pool(stepq, cfg), _pool(stepq, cfg)
    g = torch.Generator(device="cuda").manual_seed(ci)
    S0 = torch.randn((cfg.batch, cfg.heads, 128, 128), device="cuda", generator=g) * 0.2
    full.pack(S0)
    part.pack(S0)
    active = [4, 0, 3]
    part.set_active(active)
    offs, total = W.item_offsets(W.bit_table(cfg), 128, cfg.batch)
    per_req = int(offs[1, 0])
    for t in range(3):
        part.state.copy_(full.state)
        before = part.state.clone()
        x = {k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, t).items()}
        # inactive rows of the inputs may hold anything: they are not read
        xp = {k: v.clone() for k, v in x.items()}
        for k in xp:
            xp[k][[1, 2, 5]] = float("nan")
        o_full = full.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        o_part = torch.full_like(o_full, -7.0)
        part.decode_step(xp["q"], xp["k"], xp["v"], xp["alpha"], xp["beta"], o_part)
        torch.cuda.synchronize()
        part.check()
        # same kernel, same per-item arithmetic: identical results
        assert torch.equal(o_part[active], o_full[active])
        assert bool((o_part[[1, 2, 5]] == -7.0).all())  # inactive rows of out untouched
        for b in range(cfg.batch):
            seg = slice(b * per_req, (b + 1) * per_req)
            want = full.state[seg] if b in active else before[seg]
            assert torch.equal(part.state[seg], want), (t, b)


def test_active_set_validation_and_reset():
    from quantized_recurrent_state_sm_b200 import stepq
    cfg = W.with_overrides(W.CONFIGS[1], batch=4)
    pool = _pool(stepq, cfg)
    for bad in ([0, 0], [4], [-1]):
        with pytest.raises(stepq.StepqError):
            pool.set_active(bad)
    pool.set_active([])  # an empty step is a no-op
    z = torch.zeros((cfg.batch, cfg.heads, 128), device="cuda")
    zb = torch.zeros((cfg.batch, cfg.heads), device="cuda")
    before = pool.state.clone()
    pool.decode_step(z, z, z, zb, zb)
    torch.cuda.synchronize()
    assert torch.equal(pool.state, before)
    pool.set_active(None)
    assert pool.n_active == cfg.batch
