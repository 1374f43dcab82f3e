"""Cases for the checking build (libstepq_check.so, selected by STEPQ_CHECK=1):
run by tests/test_check_build.py in a process of its own, so that the binding
loads the checking library.  On valid tables the checking build computes
exactly what the oracle computes (lockstep parity on every configuration's
layout) and keeps every guard word; a staging record that does not match the
pool's layout -- here an item size one kilobyte short, which stays inside the
buffer -- is rejected before any kernel touches memory, and reported by
stepq_pool_check."""
import os

import numpy as np
import torch

import oracle
from quantized_recurrent_state_sm_b200 import stepq, workload as W
from tests.test_gpu_parity import Setup, lockstep


def test_the_checking_library_is_loaded():
    assert stepq.CHECK_BUILD and os.path.basename(stepq.LIB_PATH) == "libstepq_check.so"


def test_lockstep_parity_and_guards_every_config():
    for ci in range(5):
        cfg = W.with_overrides(W.CONFIGS[ci], batch=min(W.CONFIGS[ci].batch, 3))
        su = Setup(cfg)
        cmp, worst = lockstep(su, steps=2, t0=7)
        su.gpu.check_guards()
        print(f"checking build, config {ci}: {cmp.diff}/{cmp.codes} codes differ, worst readout {worst:.2e}")


def test_inconsistent_staging_record_is_rejected():
    cfg = W.with_overrides(W.CONFIGS[1], batch=4)
    pool = stepq.PackedStatePool(cfg.variant, cfg.batch, cfg.heads, W.bit_table(cfg), W.rho(cfg))
    pool.pack(torch.from_numpy(oracle.initial_state(cfg)).cuda())
    x = {k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, 0).items()}
    at = pool.regions["staging_records"] + 16 * 9 + 4  # record 9: item bytes | head << 16
    rec = pool.buffer[at:at + 4].clone()
    field = int(rec.cpu().numpy().view(np.int32)[0])
    bad = np.array([(field & ~0xFFFF) | ((field & 0xFFFF) - 1024)], np.int32).view(np.uint8)
    pool.buffer[at:at + 4] = torch.from_numpy(bad).cuda()
    before = pool.state.clone()
    out = torch.full((cfg.batch, cfg.heads, 128), -3.0, device="cuda")
    pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
    torch.cuda.synchronize()
    try:
        pool.check()
        raise AssertionError("the inconsistent record was not reported")
    except stepq.StepqError as e:
        assert "checking build" in str(e)
    assert torch.equal(pool.state, before) and bool((out == -3.0).all())  # nothing was touched
    pool.buffer[at:at + 4] = rec
    pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
    pool.check()  # the status word was cleared; the restored tables pass
    pool.check_guards()
    assert not torch.equal(pool.state, before)


def test_inconsistent_position_offset_is_rejected():
    """A KDA head record whose stored bit offset of a row position disagrees
    with the position widths is rejected before any kernel reads a stream."""
    cfg = W.with_overrides(W.CONFIGS[2], batch=2)
    bits = W.bit_table(cfg)
    pool = stepq.PackedStatePool(cfg.variant, cfg.batch, cfg.heads, bits, W.rho(cfg))
    pool.pack(torch.from_numpy(oracle.initial_state(cfg)).cuda())
    x = {k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, 0).items()}
    F = W.position_widths(bits[0])
    offs = np.concatenate([[0], np.cumsum(4 * F[:-1])]).astype("<u2")
    r0 = pool.regions["head_records"]
    head0 = pool.buffer[r0:r0 + 4096].cpu().numpy().tobytes()  # the first head's record lies in here
    at = head0.find(offs.tobytes())
    assert at >= 0 and head0.find(offs.tobytes(), at + 1) < 0  # the offsets, found once
    at = r0 + at + 2 * 5  # position 5
    saved = pool.buffer[at:at + 2].clone()
    bad = offs.copy()
    bad[5] += 4
    pool.buffer[at:at + 2] = torch.from_numpy(bad[5:6].view(np.uint8).copy()).cuda()
    before = pool.state.clone()
    out = torch.full((cfg.batch, cfg.heads, 128), -3.0, device="cuda")
    pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
    torch.cuda.synchronize()
    try:
        pool.check()
        raise AssertionError("the inconsistent position offset was not reported")
    except stepq.StepqError as e:
        assert "checking build" in str(e)
    assert torch.equal(pool.state, before) and bool((out == -3.0).all())
    pool.buffer[at:at + 2] = saved
    pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
    pool.check()
    pool.check_guards()
