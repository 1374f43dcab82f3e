"""Free-running drift of the oracle's packed recursion against its own fp32
recursion, over a sample of (request, head) items, in worker processes.

Used by the GPU drift-parity tests (the GPU side runs in the test process).
Items are independent, so the sample splits into groups of heads of one
request, each group run in its own spawned process over every step of the
rollout.  A group returns, every `every` steps, the sums over its items of
||unpack(pool) - S_fp32||_F^2 and ||S_fp32||_F^2; the drift over the sample is
sqrt(sum of the first / sum of the second).  With `perturb`, the group also runs
a copy of the packed pool in which one code of every item starts one step away
(a rollout whose rounding decisions are decorrelated from the first), which
measures how far two equally valid rollouts' drifts lie apart.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np


def _perturb(pool, bits, seed):
    import oracle
    r = np.random.default_rng(seed)
    for s in range(pool.n):
        bh = bits[pool.slot_head[s]]
        it = oracle.unpack_item(bh, pool.item(s), 128, 128)
        rows = np.flatnonzero(bh != 16)
        if rows.size == 0:
            continue
        i, j = int(r.choice(rows)), int(r.integers(128))
        Q = (1 << (int(bh[i]) - 1)) - 1
        it["code"][i, j] += 1 if it["code"][i, j] < Q else -1
        pool.set_item(s, oracle.pack_item(bh, it["r"], it["c"], it["code"], it["piv"]))


def _group(args):
    """One request's heads `heads` over steps 0 .. steps-1 from the packed S0."""
    ci, overrides, req, heads, steps, every, perturb, bits, rho, s0_bytes = args
    import oracle
    from quantized_recurrent_state_sm_b200 import workload as W
    cfg = W.with_overrides(W.CONFIGS[ci], **overrides) if overrides else W.CONFIGS[ci]
    kda = cfg.variant == W.KDA
    heads = np.asarray(heads)
    pool = oracle.SlotPool(heads, bits, rho, ls_iters=cfg.ls_iters, kda=kda)
    pool.pool[:] = s0_bytes
    # the fp32 recursion starts from the same full-precision state as the GPU's, S0
    Sf = np.ascontiguousarray(oracle.initial_state(cfg, [req])[0][heads])
    pools = [pool]
    if perturb:
        P = oracle.SlotPool(heads, bits, rho, ls_iters=cfg.ls_iters, kda=kda)
        P.pool[:] = pool.pool
        _perturb(P, bits, seed=1000 * req + int(heads[0]))
        pools.append(P)
    rows = []
    for t in range(steps):
        x = W.step_inputs(cfg, t, [req])
        q, k, v = x["q"][0][heads], x["k"][0][heads], x["v"][0][heads]
        a, b = x["alpha"][0][heads], x["beta"][0][heads]
        for P in pools:
            P.step(q, k, v, a, b)
        oracle.fp32_step(Sf, q, k, v, a, b, kda=kda)
        if (t + 1) % every == 0 or t + 1 == steps:
            ref = float(np.sum(Sf.astype(np.float64) ** 2))
            errs = [float(np.sum((P.unpack().astype(np.float64) - Sf) ** 2)) for P in pools]
            rows.append((t + 1, ref, *errs))
    return rows


def oracle_drift(ci, requests, bits, rho, s0_items, steps, every=64, perturb=True, overrides=None,
                 heads_per_group=None, workers=None):
    """Drift of the oracle over requests x all heads.

    s0_items[(req, h)] -> packed bytes of that item's initial state (the same
    bytes the GPU pool starts from).  Returns (steps_list, D_or, D_pert), the
    drift over the whole sample at each checkpoint (D_pert None without
    perturb).
    """
    from quantized_recurrent_state_sm_b200 import workload as W
    cfg = W.with_overrides(W.CONFIGS[ci], **overrides) if overrides else W.CONFIGS[ci]
    H = cfg.heads
    workers = workers or max(1, min(32, os.cpu_count() or 1))
    if heads_per_group is None:
        groups_per_req = max(1, -(-workers // len(requests)))
        heads_per_group = max(1, -(-H // groups_per_req))
    jobs = []
    for req in requests:
        for h0 in range(0, H, heads_per_group):
            hs = list(range(h0, min(H, h0 + heads_per_group)))
            s0 = np.concatenate([s0_items[(req, h)] for h in hs])
            jobs.append((ci, overrides, int(req), hs, steps, every, perturb, bits, rho, s0))
    ctx = mp.get_context("spawn")
    with ctx.Pool(min(workers, len(jobs))) as pool:
        res = pool.map(_group, jobs)
    T = [r[0] for r in res[0]]
    ref = np.sum([[r[1] for r in g] for g in res], axis=0)
    err = np.sum([[r[2] for r in g] for g in res], axis=0)
    D_or = np.sqrt(err / ref)
    D_p = None
    if perturb:
        errp = np.sum([[r[3] for r in g] for g in res], axis=0)
        D_p = np.sqrt(errp / ref)
    return T, D_or, D_p


def _group_bytes(args):
    """One request's heads `heads` over steps 0 .. steps-1 of the packed
    recursion from the packed S0: the final packed bytes of each item."""
    ci, overrides, req, heads, steps, bits, rho, s0_bytes = args
    import oracle
    from quantized_recurrent_state_sm_b200 import workload as W
    cfg = W.with_overrides(W.CONFIGS[ci], **overrides) if overrides else W.CONFIGS[ci]
    kda = cfg.variant == W.KDA
    heads = np.asarray(heads)
    pool = oracle.SlotPool(heads, bits, rho, ls_iters=cfg.ls_iters, kda=kda)
    pool.pool[:] = s0_bytes
    for t in range(steps):
        x = W.step_inputs(cfg, t, [req])
        pool.step(x["q"][0][heads], x["k"][0][heads], x["v"][0][heads], x["alpha"][0][heads],
                  x["beta"][0][heads])
    return [(req, int(h), pool.item(s).copy()) for s, h in enumerate(heads)]


def oracle_rollout_bytes(ci, requests, bits, rho, s0_items, steps, overrides=None, workers=None):
    """The oracle's packed recursion over requests x all heads from the packed
    bytes s0_items[(req, h)]: {(req, h): packed bytes after `steps` steps}."""
    from quantized_recurrent_state_sm_b200 import workload as W
    cfg = W.with_overrides(W.CONFIGS[ci], **overrides) if overrides else W.CONFIGS[ci]
    H = cfg.heads
    workers = workers or max(1, min(32, os.cpu_count() or 1))
    per = max(1, -(-H // max(1, -(-workers // len(requests)))))
    jobs = []
    for req in requests:
        for h0 in range(0, H, per):
            hs = list(range(h0, min(H, h0 + per)))
            s0 = np.concatenate([s0_items[(req, h)] for h in hs])
            jobs.append((ci, overrides, int(req), hs, steps, bits, rho, s0))
    with mp.get_context("spawn").Pool(min(workers, len(jobs))) as pool:
        res = pool.map(_group_bytes, jobs)
    return {(r, h): b for group in res for (r, h, b) in group}
