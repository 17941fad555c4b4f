"""Bounded waits: a pipeline wait that runs out is reported, and the library
recovers.

Every wait inside the kernels (a consumer waiting for its data, a producer for
a free buffer slot) gives up after a time limit, lets the copies and MMAs its
kernel already issued complete, records a timeout in the device status word
and lets the kernel return.  sgqa_set_wait_limit_ns() lowers that limit; at
1 ns the waits of the tcgen05 index and attention kernels and of the decode
gather cannot be met, so the calls end early, and sgqa_check() must report
SGQA_ERR_TIMEOUT.  With the default limit restored, the same calls must give
the same outputs as before the failure, bit for bit (the kernels are
deterministic).  No GPU fault is involved: a timed-out kernel returns.
"""
import dataclasses

import pytest
import torch

from sparse_long_context_sgqa_b200 import inputs as I
from tests import _harness as Hn

pytestmark = pytest.mark.gpu

PREFILL = dataclasses.replace(I.WORKLOADS["prefill8k"], name="timeout_prefill", seq_len=4096, chunk=2048)
DECODE = dataclasses.replace(I.WORKLOADS["prefill8k"], name="timeout_decode", seq_len=8192, num_seqs=2,
                             q_start=8191, n_queries=1, chunk=1)


def test_timeout_is_reported_and_later_calls_succeed(cuda_device):
    from sparse_long_context_sgqa_b200 import binding as Bd
    inputs = {wl.name: Hn.make_inputs(wl, cuda_device) for wl in (PREFILL, DECODE)}
    first = {wl.name: Hn.run_forward(wl, cuda_device, *inputs[wl.name]) for wl in (PREFILL, DECODE)}
    for wl in (PREFILL, DECODE):
        try:
            Bd.sgqa_set_wait_limit_ns(1)
            with pytest.raises(Bd.SgqaError) as err:
                Hn.run_forward(wl, cuda_device, *inputs[wl.name])  # ends with sgqa_check()
        finally:
            Bd.sgqa_set_wait_limit_ns(0)
        assert err.value.code == 5, err.value  # SGQA_ERR_TIMEOUT
        Bd.sgqa_check()  # the status word was cleared
        again = Hn.run_forward(wl, cuda_device, *inputs[wl.name])
        assert torch.equal(again.out, first[wl.name].out), wl.name
        assert torch.equal(again.sel, first[wl.name].sel), wl.name
        assert torch.equal(again.store, first[wl.name].store), wl.name

