"""Guard words after every region of a pool buffer (stepq_pool_check_guards):
every kernel that works on a pool -- pack, the fused decode step, the split
pipeline, the active request set, the ablation fits, unpack -- leaves them
intact on every configuration's layout, and a changed guard word is reported.
This is the memory-safety evidence that replaces a sanitizer run: a write
past the packed states or past any table of the pool buffer lands in a
guard region."""
import numpy as np
import pytest
import torch

import oracle
from quantized_recurrent_state_sm_b200 import workload as W

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from quantized_recurrent_state_sm_b200 import stepq
else:  # pragma: no cover
    stepq = None


def _inputs(cfg, t):
    return {k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, t).items()}


@pytest.mark.parametrize("ci", [0, 1, 2, 3, 4])
def test_guards_hold_through_every_kernel(ci):
    cfg = W.with_overrides(W.CONFIGS[ci], batch=min(W.CONFIGS[ci].batch, 5))
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    B, H = cfg.batch, cfg.heads
    pool = stepq.PackedStatePool(cfg.variant, B, H, bits, rho, cfg.ls_iters)
    pool.check_guards()
    S0 = torch.from_numpy(oracle.initial_state(cfg)).cuda()
    pool.pack(S0)
    pool.check_guards()
    for t in range(3):
        x = _inputs(cfg, t)
        pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        pool.check()
        pool.check_guards()
    work = torch.empty((B, H, 128, 128), device="cuda")
    x = _inputs(cfg, 3)
    pool.decode_step_split(x["q"], x["k"], x["v"], x["alpha"], x["beta"], work, side_stream=torch.cuda.Stream())
    pool.check_guards()
    pool.set_active([B - 1, 0])
    x = _inputs(cfg, 4)
    pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    pool.check_guards()
    pool.set_active(None)
    for mode in (stepq.SCALE_ROW, stepq.SCALE_COL, stepq.SCALE_HEAD):
        pool.set_scale_mode(mode)
        pool.pack(S0)
        pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        pool.check_guards()
    pool.set_scale_mode(stepq.SCALE_DUAL)
    pool.unpack()
    pool.check()
    pool.check_guards()


def test_changed_guard_word_is_reported():
    cfg = W.with_overrides(W.CONFIGS[1], batch=2)
    pool = stepq.PackedStatePool(cfg.variant, cfg.batch, cfg.heads, W.bit_table(cfg), W.rho(cfg))
    regions = pool.regions
    for g, name in ((0, "packed states"), (6, "staging records")):
        at = regions["guards"][g] + 4 * 5
        keep = pool.buffer[at].clone()
        pool.buffer[at] ^= 0xFF
        with pytest.raises(stepq.StepqError) as e:
            pool.check_guards()
        assert "guard word 5 after the " + name in str(e.value)
        pool.buffer[at] = keep
        pool.check_guards()
