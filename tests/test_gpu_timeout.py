"""A bounded device wait that runs out, on the GPU, without a fault.

dsa_debug_stall makes a kernel's MMA-issuing thread wait on an mbarrier that
nothing arrives at. The wait gives up after its limit (1 s), the kernel
records DSA_ERR_TIMEOUT and every CTA leaves through its give-up path
(copies in flight drained, tensor memory freed); the kernels launched after
it in the same call return at once. The call must come back, the error word
must read DSA_ERR_TIMEOUT, and the next call, with the knob cleared, must give
the oracle's results: the context is still usable.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from test_gpu_parity import assert_mla_close, cuda, lse_atol, no_device_error

pytestmark = pytest.mark.gpu

DSA_ERR_TIMEOUT = -5


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_02_b200 as d
    return d


@pytest.fixture(scope="module")
def small():
    inp = W.make_prefill(W.CONFIGS[1], L=384)           # rows 256.. take the sparse path
    rows = np.array([0, 255, 256, 383])
    return inp, rows, oracle.forward(inp, rows=rows)


@pytest.mark.parametrize("mask", [1, 2, 3], ids=["indexer", "sparse_mla", "both"])
def test_stalled_wait_times_out_and_the_next_call_is_clean(dsa, small, mask):
    inp, rows, ref = small
    g = cuda(inp)
    args = (g["q8"], None, g["k8"], None, g["w"], g["q"], g["kv"], inp["k"], inp["scale"],
            inp["sm_scale"])
    no_device_error(dsa)
    dsa.debug_stall(mask)
    try:
        t0 = time.perf_counter()
        dsa.forward(*args, chunk=128)
        st = dsa.get_device_error()                     # synchronises the stream
        took = time.perf_counter() - t0
    finally:
        dsa.debug_stall(0)
    assert st == DSA_ERR_TIMEOUT, dsa.STATUS.get(st, st)
    assert took < 60, took                              # limited waits, not a hang
    out, lse, idx = dsa.forward(*args, chunk=128)
    no_device_error(dsa)
    got = idx[rows].cpu().numpy()
    for i, r in enumerate(rows):
        assert set(got[i][got[i] >= 0]) == set(ref["idx"][i][ref["idx"][i] >= 0]), r
    assert_mla_close(out[rows], ref["out"], lse[rows], ref["lse"],
                     lse_atol(inp["q"][rows], inp["kv"], inp["sm_scale"], ref["lse"], inp["k"]))


def test_debug_stall_rejects_unknown_bits(dsa):
    with pytest.raises(dsa.DSAError):
        dsa.debug_stall(4)
