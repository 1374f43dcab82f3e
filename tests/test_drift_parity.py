"""Free-running drift parity of the CUDA path with the oracle, at each
configuration's full step count.

The drift of a packed rollout is D_t = ||unpack(pool_t) - S_fp32_t||_F /
||S_fp32_t||_F, each side against its own unquantised fp32 recursion from the
same initial state (the GPU's stepq_fp32_step, the oracle's scalar loops).
The GPU runs the whole batch in the launch configuration the benchmark times;
the oracle follows 16 requests (among them 0, 1, B/2 and B-1) x every head, in
spawned worker processes (items are independent).  The sampled requests get the
workload's exact inputs and their items start from the oracle's packed bytes;
the other requests run on random inputs of the same distribution (they are
only there to fill the launch).  Every 64 steps and at the end the drift over
the sampled items is compared with the oracle's: within 1e-3 relative (the
stated tolerance) wherever the oracle meets that against itself, and within
the oracle's own spread everywhere.

Requantising every step is chaotic: the fp32 sums run in a different order on
the two sides, so a rounding decision at a boundary sometimes differs, and the
item's later rounding noise decorrelates from the oracle's.  The drift over
hundreds of items is an average that such differences barely move.  The
oracle also runs a copy of the sample in which one code of every item starts
one step away; the printed spread |D_pert - D_or| / D_or is how far two
equally valid rollouts of the same sample lie apart.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from quantized_recurrent_state_sm_b200 import workload as W
from tests.drift import oracle_drift

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from quantized_recurrent_state_sm_b200 import stepq
else:  # pragma: no cover
    stepq = None

TOL = 1e-3
EVERY = 64


def drift_requests(cfg, n=16):
    B = cfg.batch
    even = np.linspace(0, B - 1, min(n, B)).round().astype(int).tolist()
    return sorted(set(even) | set(W.parity_requests(cfg)))


def oracle_bytes(cfg, req, S0, bits, rho):
    out = {}
    for a, r in enumerate(req):
        for h in range(cfg.heads):
            f = oracle.fit_quantise(S0[a, h], bits[h], rho[h], cfg.ls_iters)
            out[(r, h)] = oracle.pack_item(bits[h], f["r"], f["c"], f["code"], f["piv"])
    return out


def gpu_drift(cfg, req, S0, s0_bytes, bits, rho, steps):
    B, H = cfg.batch, cfg.heads
    dev = torch.device("cuda")
    kda = cfg.variant == W.KDA
    pool = stepq.PackedStatePool(cfg.variant, B, H, bits, rho, cfg.ls_iters)
    idx = np.arange(B) % len(req)
    idx[req] = np.arange(len(req))
    S0_dev = torch.from_numpy(S0).to(dev)
    Sf = S0_dev[torch.from_numpy(idx).to(dev)].contiguous()  # [B, H, dk, dv]
    pool.pack(Sf)
    offs, total = W.item_offsets(bits, 128, B)
    offs = np.asarray(offs).reshape(B, H)
    state = pool.state
    for r in req:
        for h in range(H):
            b = s0_bytes[(r, h)]
            o = int(offs[r, h])
            state[o:o + len(b)].copy_(torch.from_numpy(np.ascontiguousarray(b)))
    ridx = torch.tensor(req, device=dev)
    g = torch.Generator(device=dev).manual_seed(0x51DE + cfg.index)
    gate = torch.from_numpy(W.gates(cfg)).to(dev)
    alpha = (gate[None].expand(B, H, 128) if kda else gate[None].expand(B, H)).contiguous()

    def unit(x):
        return x / x.norm(dim=-1, keepdim=True)

    T, D = [], []
    for t in range(steps):
        x = W.step_inputs(cfg, t, req)
        q = unit(torch.randn(B, H, 128, device=dev, generator=g))
        k = unit(torch.randn(B, H, 128, device=dev, generator=g))
        v = torch.randn(B, H, 128, device=dev, generator=g)
        beta = torch.sigmoid(torch.randn(B, H, device=dev, generator=g))
        q[ridx] = torch.from_numpy(x["q"]).to(dev)
        k[ridx] = torch.from_numpy(x["k"]).to(dev)
        v[ridx] = torch.from_numpy(x["v"]).to(dev)
        beta[ridx] = torch.from_numpy(x["beta"]).to(dev)
        a = alpha.clone()
        a[ridx] = torch.from_numpy(x["alpha"]).to(dev)
        pool.decode_step(q, k, v, a, beta)
        stepq.fp32_step(cfg.variant, Sf, q, k, v, a, beta)
        if (t + 1) % EVERY == 0 or t + 1 == steps:
            U = pool.unpack()[ridx].double()
            ref = Sf[ridx].double()
            D.append(float(torch.sqrt(((U - ref) ** 2).sum() / (ref ** 2).sum())))
            T.append(t + 1)
            del U, ref
    torch.cuda.synchronize()
    pool.check()
    return T, np.array(D)


@pytest.fixture(scope="module", params=[0, 1, 2, 3, 4])
def drift(request):
    """One free-running rollout per configuration, shared by the tests below."""
    ci = request.param
    cfg = W.CONFIGS[ci]
    req = drift_requests(cfg)
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    S0 = oracle.initial_state(cfg, req)
    s0_bytes = oracle_bytes(cfg, req, S0, bits, rho)
    res = {}

    def run_oracle():
        res["or"] = oracle_drift(ci, req, bits, rho, s0_bytes, cfg.steps, every=EVERY, perturb=True)

    th = threading.Thread(target=run_oracle)
    th.start()
    T, D_gpu = gpu_drift(cfg, req, S0, s0_bytes, bits, rho, cfg.steps)
    th.join()
    T_or, D_or, D_p = res["or"]
    assert list(T) == list(T_or)
    gap = np.abs(D_gpu - D_or) / D_or
    spread = np.abs(D_p - D_or) / D_or
    print(f"\nconfig {ci}: {len(req)} requests x {cfg.heads} heads, {cfg.steps} steps")
    for t, dg, do, g_, s_ in zip(T, D_gpu, D_or, gap, spread):
        print(f"  step {t:5d}: drift gpu {dg:.6f} oracle {do:.6f}  gap {g_:.2e}  spread {s_:.2e}")
    assert np.all(np.isfinite(D_gpu)) and np.all(np.isfinite(D_or))
    return {"ci": ci, "T": T, "gpu": D_gpu, "oracle": D_or, "gap": gap, "spread": spread}


def test_drift_within_stated_tolerance(drift):
    """The stated drift tolerance, |D_gpu - D_or| <= 1e-3 D_or at every checkpoint,
    wherever the oracle meets it against itself.  Where two equally valid
    oracle rollouts of the sample (one code of every item nudged by one step
    at the start) already differ by more than 1e-3 at some checkpoint, no
    reordering of the fp32 sums can be held to it: the case is an expected
    failure with the measured figures."""
    gap, spread = drift["gap"], drift["spread"]
    if spread.max() > TOL:
        pytest.xfail(f"config {drift['ci']}: the oracle's own spread reaches {spread.max():.2e} > {TOL:g} "
                     f"(GPU gap max {gap.max():.2e})")
    assert np.all(gap <= TOL), f"drift gap above {TOL:g}: max {gap.max():.2e} (spread max {spread.max():.2e})"


def test_drift_within_oracle_spread(drift):
    """The GPU's drift lies within the oracle's own envelope: every gap is at
    most 1e-3 or four times the root mean square, over the checkpoints, of
    the spread between two equally valid oracle rollouts (the gap and the
    spread are both the difference of two rollouts whose rounding decisions
    have decorrelated)."""
    gap, spread = drift["gap"], drift["spread"]
    bound = max(TOL, 4.0 * float(np.sqrt(np.mean(spread ** 2))))
    assert np.all(gap <= bound), f"drift gap {gap.max():.2e} above {bound:.2e}"
