"""Failure detection on the device, in the one form that faults nothing: a bounded wait that
nothing will ever complete runs out.

rod_test_expire_waits arms the next tensor-core recurrence prefill so that its TMA producers
issue no copies and every bounded wait gives up after a short probe limit. The consumers then
wait on input barriers that never complete; each kernel must give up, raise its abort flag, let
every role leave its loop, drain its MMAs, free tensor memory and return. The host sees
ROD_ERR_TIMEOUT from rod_check, the CUDA context stays usable, and the very next call (not
armed) must match the oracle again. Nothing here traps, asserts or touches memory out of
bounds.
"""
import pytest
import torch

import oracle
import sliding_window_attention_chunked_b200 as rod
from sliding_window_attention_chunked_b200 import workloads as wl

from .parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIMEOUT = -7


@pytest.mark.parametrize("B,H,T", [(1, 2, 5000), (2, 3, 300)])
def test_expired_wait_reports_timeout_then_recovers(B, H, T):
    q, k, v, g = wl.gla_inputs(B, H, T, 128, 128, dist="l2", seed=T)
    qd, kd, vd, gd = [t.to(DEV) for t in (q, k, v, g)]
    rod.check()  # nothing pending from earlier tests
    # armed call: every wait of its kernels expires after 4096 probes
    rod.test_expire_waits(4096)
    S = torch.zeros(B, H, 128, 128, device=DEV)
    rod.gla_prefill(qd, kd, vd, gd, S, chunk=64)
    with pytest.raises(rod.RodError) as err:
        rod.check()
    assert err.value.status == TIMEOUT
    # the flag was read and cleared; the context is usable; the next call is correct
    rod.check()
    o_ref, S_ref = oracle.gla_prefill(q, k, v, g)
    S = torch.zeros(B, H, 128, 128, device=DEV)
    o = rod.gla_prefill(qd, kd, vd, gd, S, chunk=64)
    rod.check()
    compare(o, o_ref, "bf16", "o after a timed-out call")
    compare(S, S_ref, "bf16", "state after a timed-out call")


def test_disarmed_call_runs_normally():
    q, k, v, g = wl.gla_inputs(1, 2, 700, 128, 128, dist="l2", seed=3)
    rod.test_expire_waits(4096)
    rod.test_expire_waits(0)  # disarm
    o_ref, S_ref = oracle.gla_prefill(q, k, v, g)
    S = torch.zeros(1, 2, 128, 128, device=DEV)
    o = rod.gla_prefill(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), S, chunk=64)
    rod.check()
    compare(o, o_ref, "bf16", "o")
    compare(S, S_ref, "bf16", "state")
