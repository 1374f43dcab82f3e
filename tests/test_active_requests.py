"""Decode over an active subset of the pool's requests (stepq_pool_set_active):
the active requests' items come out exactly as in a full step over the same
states, and the inactive requests' states stay untouched."""
import numpy as np
import pytest
import torch

from quantized_recurrent_state_sm_b200 import workload as W

pytestmark = pytest.mark.gpu


def _pool(stepq, cfg):
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    return stepq.PackedStatePool(cfg.variant, cfg.batch, cfg.heads, bits, rho, cfg.ls_iters)


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
