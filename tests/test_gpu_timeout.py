"""The prefill kernel's bounded waits, made to run out on purpose.

attn_debug_prefill_timeout shortens the producer's and MMA issuers' pipeline
wait limit to 1 ms and makes the producer leave out one K/V ring step (its copy
is never issued and its barrier never armed). The MMA issuer's wait for that
step runs out: the CTA records ATTN_ERR_TIMEOUT, lets its copies in flight
land, drains its tensor-core work, releases its tensor memory and returns; the
softmax warps give up on their own (full) limit. Nothing faults or hangs: every
wait in the kernel is bounded. The next normal call on the same context must be
exact again.
"""

import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen
from oracle import attn_oracle as orc
from parity_util import compare_output

pytestmark = pytest.mark.gpu

TIMEOUT = 5


@pytest.mark.parametrize("withhold", [3, 0])
def test_prefill_wait_runs_out_and_the_context_stays_usable(cuda_device, withhold):
    q, k, v = gen.prefill_inputs(1, 2, 1, 512, 128, seed=6100)
    qd, kd, vd = q.to(cuda_device), k.to(cuda_device), v.to(cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ab.binding.debug_prefill_timeout(qd, kd, vd, wait_limit_ns=1_000_000, withhold_step=withhold,
                                     device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == TIMEOUT

    o, lse = ab.prefill(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = orc.prefill(q, k, v, True, gen.attn_scale(128))
    compare_output(o, o_ref, lse, lse_ref, label="after a timeout")


def test_prefill_short_limit_without_a_withheld_step_completes(cuda_device):
    q, k, v = gen.prefill_inputs(1, 2, 1, 512, 128, seed=6101)
    qd, kd, vd = q.to(cuda_device), k.to(cuda_device), v.to(cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o, lse = ab.binding.debug_prefill_timeout(qd, kd, vd, wait_limit_ns=50_000_000, withhold_step=-1,
                                              device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o_ref, lse_ref = orc.prefill(q, k, v, True, gen.attn_scale(128))
    compare_output(o, o_ref, lse, lse_ref, label="short limit, nothing withheld")
