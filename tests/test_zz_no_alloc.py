"""The decode step without a pool (stepq_decode_step_noalloc) against the pool
entry point.  Collected last on purpose: it must pass after every other test
as well as alone, since its scratch tables live in a library-owned device array
that persists across calls."""
import numpy as np
import pytest

from quantized_recurrent_state_sm_b200 import workload as W


@pytest.fixture(scope="module")
def S():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from quantized_recurrent_state_sm_b200 import stepq
    return stepq


def _inputs(cfg, t):
    import torch
    return {k: torch.from_numpy(v).cuda() for k, v in W.step_inputs(cfg, t).items()}


@pytest.mark.gpu
@pytest.mark.parametrize("ci,batch", [(1, 8), (2, 4)])
def test_noalloc_matches_pool_on_two_calls(S, ci, batch):
    import torch
    cfg = W.with_overrides(W.CONFIGS[ci], batch=batch)
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    pool = S.PackedStatePool(cfg.variant, cfg.batch, cfg.heads, bits, rho, cfg.ls_iters)
    g = torch.Generator(device="cuda").manual_seed(ci)
    pool.pack(torch.randn((cfg.batch, cfg.heads, 128, 128), device="cuda", generator=g) * 0.2)
    states = pool.state.clone()  # the same packed states, in memory the caller owns
    for t in range(2):  # two calls in a row
        x = _inputs(cfg, t)
        o_pool = pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        o_free = S.decode_step_noalloc(cfg.variant, bits, rho, states, x["q"], x["k"], x["v"], x["alpha"],
                                       x["beta"], ls_iters=cfg.ls_iters)
        torch.cuda.synchronize()
        pool.check()
        # the same kernel on the same bytes and inputs, in the same item order:
        # identical results, bit for bit
        assert torch.equal(o_free, o_pool), f"readout differs at call {t}"
        diff = int((states != pool.state).sum())
        assert diff == 0, f"{diff} packed bytes differ at call {t}"


@pytest.mark.gpu
def test_noalloc_rejects_tables_beyond_its_scratch(S):
    import torch
    cfg = W.with_overrides(W.CONFIGS[1], batch=4096)  # 131 072 items: far beyond the fixed scratch
    bits, rho = W.bit_table(cfg), W.rho(cfg)
    B, H = 1, cfg.heads
    tiny = torch.zeros(16, dtype=torch.uint8, device="cuda")
    q = torch.zeros((cfg.batch, H, 128), device="cuda")
    with pytest.raises(S.StepqError) as e:
        S.decode_step_noalloc(cfg.variant, bits, rho, tiny, q, q, q, torch.zeros((cfg.batch, H), device="cuda"),
                              torch.zeros((cfg.batch, H), device="cuda"))
    assert "scratch" in str(e.value)


def test_noalloc_host_checks_without_gpu():
    """Descriptor and size checks happen on the host before any CUDA call."""
    import ctypes as C
    from quantized_recurrent_state_sm_b200 import build
    build.build()
    from quantized_recurrent_state_sm_b200 import stepq
    big = W.with_overrides(W.CONFIGS[1], batch=4096)
    d, keep = stepq.make_desc(big.variant, big.batch, big.heads, W.bit_table(big), W.rho(big))
    assert stepq.lib.stepq_decode_step_noalloc(C.byref(d), None, 0, None, None, None, None, None, None,
                                               None) == stepq.ERR_UNSUPPORTED
    assert "scratch" in stepq.lib.stepq_last_error().decode()
    small = W.with_overrides(W.CONFIGS[1], batch=8)
    d, keep = stepq.make_desc(small.variant, small.batch, small.heads, W.bit_table(small), W.rho(small))
    assert stepq.lib.stepq_decode_step_noalloc(C.byref(d), None, 16, None, None, None, None, None, None,
                                               None) == stepq.ERR_INVALID_ARG
    assert "states holds 16 bytes" in stepq.lib.stepq_last_error().decode()
