"""The device-side time limit of the kernels' waits, made to run out.

Every mbarrier wait in the library's kernels gives up after a time limit,
sets the device error word and lets its kernel return, so that a lost
arrival never hangs the GPU. mla_selftest_wait_timeout runs that wait (the
same helper) with a 1 ms limit on a barrier that nothing arrives at. The
test checks that the wait gave up, that the host then reads
MLA_ERR_DEVICE_TIMEOUT, that the next check is clean, and that the context
still runs a prefill that matches the oracle. No GPU fault is involved.
"""

import pytest
import torch

from decode_latent_rmsnorm_b200 import mla
from decode_latent_rmsnorm_b200 import workloads as W
from _parity import compare, f64, oracle_prefill, run_prefill

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_context_survives(gpu_lib):
    mla.mla_check_device_status()                       # start from a clean error word
    flag = mla.mla_selftest_wait_timeout(1000)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_check_device_status()
    assert e.value.status == 5                          # MLA_ERR_DEVICE_TIMEOUT
    assert int(flag.item()) == 1                        # the wait gave up
    mla.mla_check_device_status()                       # the word was cleared
    wl = W.scaled(W.KIMI, seqlens=(300, 129), seed=47)
    inp = W.prefill_inputs(wl)
    got = run_prefill(wl, inp)
    compare(f64(got), oracle_prefill(wl, inp), "bf16", "prefill after the timeout self-test")


def test_selftest_rejects_bad_limit(gpu_lib):
    with pytest.raises(mla.MlaError) as e:
        mla.mla_selftest_wait_timeout(0)
    assert e.value.status == 1
