"""Bounded waits on the GPU.

Every wait inside the library's kernels (rendezvous counters, grid barriers,
pipeline mbarriers) gives up after a time limit and reports a timeout instead
of hanging.  Here the same wait primitives run against a counter that nothing
increments and an mbarrier that nothing arrives on, with a 50 ms limit: the
host must read SPEC_ERR_TIMEOUT, both waits must have given up, and the CUDA
context must still work afterwards (a prefill and a verification step that
match brute-force greedy decoding by the float64 oracle).
"""

import ctypes
import time

import numpy as np
import pytest
import torch

import synth
from oracle import oracle_greedy_ar
from speculative_decoding_06_b200 import spec as S
from gpu_common import make_pair

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_survives():
    scratch = torch.zeros(4, dtype=torch.int32, device="cuda")
    expired = ctypes.c_int32(-1)
    t0 = time.perf_counter()
    rc = S.lib().spec_wait_selftest(ctypes.c_void_p(scratch.data_ptr()), 50_000, ctypes.byref(expired))
    dt = time.perf_counter() - t0
    assert rc == S.SPEC_ERR_TIMEOUT
    assert expired.value == 2
    assert dt >= 0.1  # both waits ran to their 50 ms limit
    # bad arguments are refused before any GPU work
    assert S.lib().spec_wait_selftest(None, 50_000, ctypes.byref(expired)) == S.SPEC_ERR_ARG
    assert S.lib().spec_wait_selftest(ctypes.c_void_p(scratch.data_ptr()), 0, ctypes.byref(expired)) == S.SPEC_ERR_ARG

    # the context is intact: a prefill and one verification step
    eng, om = make_pair(synth.TINY, max_batch=1, max_seq=256, max_nodes=16)
    try:
        prompt = synth.prefix_tokens(om.d.vocab, 32, seed=4)
        greedy = oracle_greedy_ar(om, prompt, 5)
        assert eng.prefill(0, prompt) == greedy[0]
        shape = synth.chain(3)  # root (the pending token) + the true next three tokens
        a, acc, bonus = eng.verify(0, np.array(greedy[:4], np.int32), shape.parents)
        assert a == 3 and acc == greedy[1:4] and bonus == greedy[4]
    finally:
        eng.close()
