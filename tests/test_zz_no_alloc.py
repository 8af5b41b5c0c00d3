"""The allocation-free LM-head entry point, checked against the verification path
and against the float64 oracle's LM head.

Callers that may not call cudaMalloc (inside a CUDA-graph capture, in runtimes
that own all device buffers, in plug-in hosts that forbid allocation after
start-up) use spec_lm_head_argmax_noalloc, whose scratch is a fixed array
inside the library.  This file runs last so that a failure here never hides
the rest of the suite; it passes alone and after the other tests.
"""

import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import OracleModel, top2_margin
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
    assert S.spec_lm_head_argmax_noalloc(p, p, p, 8, dims.hidden, 262145, 1e-5, p, p, p, None) == \
        S.SPEC_ERR_CAPACITY


def _noalloc(hidden, norm, lm, M, d, V, eps, stream):
    amax = torch.full((M,), -7, dtype=torch.int32, device="cuda")
    t1 = torch.zeros(M, dtype=torch.float32, device="cuda")
    t2 = torch.zeros(M, dtype=torch.float32, device="cuda")
    stream.wait_stream(torch.cuda.current_stream())  # inputs and outputs were written on torch's stream
    rc = S.spec_lm_head_argmax_noalloc(hidden.data_ptr(), norm.data_ptr(), lm.data_ptr(), M, d, V, eps,
                                       amax.data_ptr(), t1.data_ptr(), t2.data_ptr(), stream.cuda_stream)
    assert rc == S.SPEC_OK
    stream.synchronize()
    return amax.cpu().numpy(), t1.cpu().numpy(), t2.cpu().numpy()


@pytest.mark.parametrize("d,V,M", [(512, 2048, 61), (512, 2000, 64), (8192, 262144, 64)])
def test_noalloc_lm_head_matches_the_oracle(d, V, M):
    """Seeded hidden rows through the final RMSNorm and the LM head, against the float64 oracle: a vocabulary
    that ends in a partial 128-row tile (2000), the full 64-row tile, and d and V at the scratch's limits."""
    dims = dataclasses.replace(synth.MINI_BF16, n_layers=0, hidden=d, vocab=V)
    g = torch.Generator().manual_seed(d + V)
    lm = (torch.randn(V, d, generator=g) * 0.02).to(torch.bfloat16)
    norm = (1.0 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16)
    host = {"embed": np.zeros((1, d), np.uint16), "lm_head": synth.tensor_to_host(lm),
            "final_norm": synth.tensor_to_host(norm), "layers": []}
    om = OracleModel(dims, host)
    lm_d, norm_d = lm.cuda(), norm.cuda()
    stream = torch.cuda.Stream()
    for call in range(2):  # two calls in a row share the scratch
        hid = torch.randn(M, d, generator=g, dtype=torch.float32)
        ref = om.lm_logits(hid.numpy().astype(np.float64))
        amax, t1, t2 = _noalloc(hid.cuda(), norm_d, lm_d, M, d, V, dims.rms_eps, stream)
        assert np.all(amax >= 0), "the call reported a device-side failure"
        part = np.sort(ref, axis=1)
        err1 = float(np.max(np.abs(t1 - part[:, -1])))
        err2 = float(np.max(np.abs(t2 - part[:, -2])))
        assert err1 <= TOL["bf16"] and err2 <= TOL["bf16"], (err1, err2)
        # the argmax is the oracle's wherever its margin leaves no doubt, and otherwise a value within tolerance
        thr = min(DECISIVE, max(2.5 * max(err1, err2), 1e-6))
        sure = top2_margin(ref) > thr
        assert sure.sum() >= M // 2
        assert np.array_equal(amax[sure], np.argmax(ref, axis=1)[sure])
        assert np.all(ref[np.arange(M), amax] >= part[:, -1] - 2 * TOL["bf16"])
