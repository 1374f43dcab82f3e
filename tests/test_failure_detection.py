"""Failure detection without a GPU fault: the bounded barrier wait that the
fused decode kernel uses for its staged copies gives up after its limit on a
barrier nothing arrives at, reports the decode kernel's timeout status, and
leaves the context usable (a decode step afterwards still matches the
oracle).  No fault, trap or endless wait is involved."""
import pytest

from quantized_recurrent_state_sm_b200 import workload as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from quantized_recurrent_state_sm_b200 import stepq
    return stepq


def test_wait_completes_when_the_arrival_comes(S):
    status, cycles = S.selftest_bounded_wait(10 ** 6, arrive=True)
    assert status == 0 and 0 <= cycles < 10 ** 6


def test_wait_gives_up_after_its_limit_and_the_context_stays_usable(S):
    limit = 2_000_000  # about a millisecond of SM clock
    status, cycles = S.selftest_bounded_wait(limit, arrive=False)
    assert status == 1  # the decode kernel's "gave up waiting" status
    assert limit <= cycles < 20 * limit
    from tests.test_gpu_parity import Setup, lockstep
    cfg = W.with_overrides(W.CONFIGS[1], batch=2)
    lockstep(Setup(cfg), steps=1, t0=3)
    status, _ = S.selftest_bounded_wait(limit, arrive=True)
    assert status == 0
