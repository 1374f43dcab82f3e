"""The oracle's recursion stays bounded over each workload's full length on its
prescribed tables (stand-in bit widths, pivots and LogNormal impact weights).

The pages report that the packed state at a nominal 6 bits tracks FP32 states
and that 4 bits still does better than uniform INT8 (ai.info summary, "Main
Findings"); a reading of the row scale whose rollouts run away on these tables
cannot be that method.  Each case runs the oracle's packed recursion and the
unquantised fp32 recursion side by side from the same initial state over the
configuration's whole step count, on request 0's first eight heads, and checks
at every 64th step that the relative state drift ||unpack - S_fp32|| /
||S_fp32|| is finite, below a bound, and not still growing in the second half
(the drift at the end is within 25 % of the drift at the midpoint).  The
bounds sit above the measured values (0.165 after configuration 0's 64 steps;
plateaus of at most 0.09, 0.12, 0.80 and 0.15 for configurations 1-4).  The
uniform 6-bit widths of configuration 0 drift more than configuration 1's
lifetime-allocated 6-bit average, whose longest-lived heads get 8 bits; the
4-bit average of configuration 3 puts most of its heads at 3 or 4 bits.
"""
import numpy as np
import pytest

import oracle
from quantized_recurrent_state_sm_b200 import workload as W

BOUND = {0: 0.25, 1: 0.15, 2: 0.2, 3: 1.0, 4: 0.25}


@pytest.mark.parametrize("ci", [0, 1, 2, 3, 4])
def test_rollout_drift_bounded_over_full_length(ci):
    cfg = W.CONFIGS[ci]
    kda = cfg.variant == W.KDA
    heads = np.arange(min(8, cfg.heads))
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    S0 = oracle.initial_state(cfg, [0])[0][heads]
    pool = oracle.SlotPool(heads, bits, rho, kda=kda, ls_iters=cfg.ls_iters)
    pool.pack(S0)
    Sf = np.ascontiguousarray(S0.copy())
    drift = []
    for t in range(cfg.steps):
        x = W.step_inputs(cfg, t, [0])
        q, k, v = x["q"][0][heads], x["k"][0][heads], x["v"][0][heads]
        a, b = x["alpha"][0][heads], x["beta"][0][heads]
        pool.step(q, k, v, a, b)
        oracle.fp32_step(Sf, q, k, v, a, b, kda=kda)
        if (t + 1) % 64 == 0:
            Sq = pool.unpack()
            d = float(np.linalg.norm(Sq - Sf) / np.linalg.norm(Sf))
            assert np.isfinite(d) and d <= BOUND[ci], (ci, t + 1, d)
            drift.append(d)
    print(f"config {ci}: drift every 64 steps " + " ".join(f"{d:.3f}" for d in drift))
    if len(drift) >= 4:
        assert drift[-1] <= 1.25 * drift[len(drift) // 2 - 1], drift
