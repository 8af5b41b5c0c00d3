"""The allocation-free LM-head entry point, checked against the verification path.

Callers that may not call cudaMalloc (inside a CUDA-graph capture, in runtimes
that own all device buffers, in plug-in hosts that forbid allocation after
start-up) use spec_lm_head_argmax_noalloc, whose scratch is a fixed array
inside the library.  This file runs last so that a failure here never hides
the rest of the suite; it passes alone and after the other tests.
"""

import numpy as np
import pytest
import torch

import synth
from speculative_decoding_06_b200 import spec as S
from gpu_common import DECISIVE, TOL

pytestmark = pytest.mark.gpu


def test_noalloc_lm_head_matches_the_verification_step():
    from speculative_decoding_06_b200.engine import SpecEngine
    dims = synth.MINI_BF16
    w = synth.model_weights(dims, seed=0, device="cuda")
    # with every decoder matrix zero each layer adds nothing to the residual
    # stream, so the final hidden row of a tree node is its token's embedding
    for lw in w["layers"]:
        for k in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"):
            lw[k].zero_()
    eng = SpecEngine(dims, w, max_batch=1, max_seq=256, max_nodes=64)
    pend = eng.prefill(0, synth.prefix_tokens(dims.vocab, 16))
    stream = torch.cuda.current_stream()
    for call in range(2):  # two calls in a row share the scratch
        shape = synth.tree_from_widths((5, 8, 10, 12, 10, 8, 6, 2), stream=call)
        toks = synth.plant_draws(shape.n, dims.vocab, stream=40 + call).rand_tok.copy()
        toks[0] = pend
        amax_ref, t1_ref, t2_ref, _ = eng.score([0], [(toks, shape.parents)])
        M = shape.n
        hidden = w["embed"][torch.as_tensor(toks, device="cuda").long()].float().contiguous()
        amax = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        t1 = torch.zeros(M, dtype=torch.float32, device="cuda")
        t2 = torch.zeros(M, dtype=torch.float32, device="cuda")
        rc = S.spec_lm_head_argmax_noalloc(hidden.data_ptr(), w["final_norm"].data_ptr(), w["lm_head"].data_ptr(),
                                           M, dims.hidden, dims.vocab, dims.rms_eps, amax.data_ptr(),
                                           t1.data_ptr(), t2.data_ptr(), stream.cuda_stream)
        assert rc == S.SPEC_OK
        torch.cuda.synchronize()
        a, v1, v2 = amax.cpu().numpy(), t1.cpu().numpy(), t2.cpu().numpy()
        err = float(np.max(np.abs(v1 - t1_ref)))
        assert err <= TOL["bf16"]
        assert float(np.max(np.abs(v2 - t2_ref))) <= TOL["bf16"]
        sure = (t1_ref - t2_ref) > min(DECISIVE, max(2.5 * err, 1e-6))
        assert np.array_equal(a[sure], amax_ref[sure])
        assert np.all((a >= 0) & (a < dims.vocab))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    dims = synth.MINI_BF16
    dummy = torch.zeros(16, device="cuda")
    p = dummy.data_ptr()
    assert S.spec_lm_head_argmax_noalloc(p, p, p, 65, dims.hidden, dims.vocab, 1e-5, p, p, p, None) == \
        S.SPEC_ERR_CAPACITY
    assert S.spec_lm_head_argmax_noalloc(p, p, p, 8, 16384, dims.vocab, 1e-5, p, p, p, None) == S.SPEC_ERR_CAPACITY
    assert S.spec_lm_head_argmax_noalloc(p, p, p, 8, 100, dims.vocab, 1e-5, p, p, p, None) == S.SPEC_ERR_CAPACITY
