"""GPU parity of the EAGLE-3 draft-head step against the float64 oracle.

The draft head (summary of "EAGLE-3: Scaling up Inference Acceleration of
Large Language Models via Training-Time Test", draft-stage section) fuses the
target's low, mid and high features with one FC layer, appends the embedding
of the token one step ahead, reduces with a second FC layer, runs one decoder
layer over its own prefix K/V and the tree's ancestors, and scores with the
target's LM head.  Checked here through the C ABI: the draft layer's K/V after
a prefill, the draft logits at every node (2e-2 absolute, the bf16 tolerance),
and the top-10 candidate lists (index by rank wherever the oracle's gap to the
neighbouring ranks leaves no doubt, the set wherever the gap after rank 10
does, values within the logit tolerance).
"""

import numpy as np
import pytest
import torch

import synth
from oracle import OracleDraftHead
from oracle.draft import top_k_rows
from gpu_common import TOL, kv_close

pytestmark = pytest.mark.gpu

K = 10


def _host(t):
    return synth.tensor_to_host(t)


def _draft_host(dw):
    return {"fc_fuse": _host(dw["fc_fuse"]), "fc_in": _host(dw["fc_in"]), "final_norm": _host(dw["final_norm"]),
            "layer": {k: _host(v) for k, v in dw["layer"].items()}}


_pairs = {}


def _pair(which):
    if which in _pairs:
        return _pairs[which]
    from speculative_decoding_06_b200.engine import SpecEngine
    dims = {"small": synth.SMALL_BF16, "wide": synth.WIDE_BF16}[which]
    wdev = synth.model_weights(dims, seed=0, device="cuda")
    dwdev = synth.draft_head_weights(dims, seed=6, device="cuda")
    host = synth.weights_to_host(wdev)
    eng = SpecEngine(dims, wdev, max_batch=4, max_seq=1024, max_nodes=128, draft=dwdev)
    oh = OracleDraftHead(dims, host, _draft_host(dwdev))
    _pairs[which] = (eng, oh, dims)
    return _pairs[which]


def _feats(rows, d, seed):
    return synth.draft_features(rows, d, seed=seed, device="cuda")


def _tokens(n, vocab, seed):
    return np.random.default_rng([7, seed]).integers(0, vocab, size=n).astype(np.int32)


def _check_topk(gi, gv, logits64, err):
    """GPU top-k lists [n][K] against the oracle's logits [n][V]."""
    oi, ov = top_k_rows(logits64, K + 1)
    thr = max(2.5 * err, 1e-6)
    for r in range(logits64.shape[0]):
        # values: the GPU's candidates carry their own logits
        np.testing.assert_allclose(gv[r], logits64[r, gi[r]], atol=TOL["bf16"])
        # rank by rank where the oracle's neighbours are clearly apart
        for j in range(K):
            lo_gap = ov[r, j] - ov[r, j + 1]
            hi_gap = ov[r, j - 1] - ov[r, j] if j > 0 else np.inf
            if lo_gap > thr and hi_gap > thr:
                assert gi[r, j] == oi[r, j], "row %d rank %d" % (r, j)
        # the set, where rank 10 is clearly ahead of rank 11
        if ov[r, K - 1] - ov[r, K] > thr:
            assert set(gi[r].tolist()) == set(oi[r, :K].tolist()), "row %d set" % r
        # order: non-increasing values, ties by index
        for j in range(K - 1):
            assert gv[r, j] > gv[r, j + 1] or (gv[r, j] == gv[r, j + 1] and gi[r, j] < gi[r, j + 1])


@pytest.mark.parametrize("which", ["small", "wide"])
def test_draft_prefill_kv(which):
    """The draft layer's K/V over a 300-row prefix (three chunks) against the oracle's."""
    eng, oh, d = _pair(which)
    T = 300
    f = _feats(T, d.hidden, seed=11)
    toks = _tokens(T, d.vocab, 11)
    eng.draft_prefill(0, f, toks)
    assert eng.draft_len(0) == T
    ref = oh.prefill(_host(f.cpu()), toks)
    kv = eng.kv_view()[d.n_layers, :, 0, :, :T, :].to(torch.float64).cpu().numpy()
    gk = np.transpose(kv[0], (1, 0, 2))
    gv = np.transpose(kv[1], (1, 0, 2))
    assert kv_close(gk, ref.k, 2e-2) <= 2e-2
    assert kv_close(gv, ref.v, 2e-2) <= 2e-2


@pytest.mark.parametrize("which", ["small", "wide"])
def test_draft_step_topk(which):
    """Three sequences (draft prefixes 300, 77, 130) with a 61-node tree, a chain and a small tree."""
    eng, oh, d = _pair(which)
    Ps = [300, 77, 130]
    shapes = [synth.tree_from_widths(synth.TREE60_WIDTHS, stream=0), synth.chain(5), synth.tiny_tree()]
    seqs = []
    for i, P in enumerate(Ps):
        f = _feats(P, d.hidden, seed=20 + i)
        toks = _tokens(P, d.vocab, 20 + i)
        eng.draft_prefill(i, f, toks)
        seqs.append(oh.prefill(_host(f.cpu()), toks))
    trees = [(_tokens(sh.n, d.vocab, 40 + i), sh.parents) for i, sh in enumerate(shapes)]
    M = sum(sh.n for sh in shapes)
    fn = _feats(M, d.hidden, seed=30)
    gi, gv, off = eng.draft_step([0, 1, 2], fn, trees, flags=2)
    logits = eng.debug_logits(M)
    fh = _host(fn.cpu())
    for i, (seq, (toks, par)) in enumerate(zip(seqs, trees)):
        lo, hi = int(off[i]), int(off[i + 1])
        ref = oh.step_logits(seq, fh[lo:hi], toks, par)
        err = float(np.max(np.abs(logits[lo:hi] - ref)))
        assert err <= TOL["bf16"], "sequence %d: max |logit error| %.3g" % (i, err)
        _check_topk(gi[lo:hi], gv[lo:hi], ref, err)
    # the step leaves the draft prefixes as they were
    assert [eng.draft_len(i) for i in range(3)] == Ps


def test_draft_step_many_token_tiles():
    """Eight 61-node trees (488 rows): four 128-token tiles in every GEMM of the draft step."""
    from speculative_decoding_06_b200.engine import SpecEngine
    _, oh, d = _pair("small")
    eng = SpecEngine(d, synth.model_weights(d, seed=0, device="cuda"), max_batch=8, max_seq=512, max_nodes=64,
                     draft=synth.draft_head_weights(d, seed=6, device="cuda"))
    try:
        B = 8
        seqs = []
        for i in range(B):
            P = 90 + 17 * i
            f = _feats(P, d.hidden, seed=60 + i)
            toks = _tokens(P, d.vocab, 60 + i)
            eng.draft_prefill(i, f, toks)
            seqs.append(oh.prefill(_host(f.cpu()), toks))
        shapes = [synth.tree_from_widths(synth.TREE60_WIDTHS, stream=i) for i in range(B)]
        trees = [(_tokens(sh.n, d.vocab, 80 + i), sh.parents) for i, sh in enumerate(shapes)]
        M = sum(sh.n for sh in shapes)
        assert "bn128 tiles" in eng.info(B, 61, 300) and "x4 " in eng.info(B, 61, 300)
        fn = _feats(M, d.hidden, seed=70)
        gi, gv, off = eng.draft_step(list(range(B)), fn, trees, flags=2)
        logits = eng.debug_logits(M)
        fh = _host(fn.cpu())
        for i, (seq, (toks, par)) in enumerate(zip(seqs, trees)):
            lo, hi = int(off[i]), int(off[i + 1])
            ref = oh.step_logits(seq, fh[lo:hi], toks, par)
            err = float(np.max(np.abs(logits[lo:hi] - ref)))
            assert err <= TOL["bf16"], "sequence %d: max |logit error| %.3g" % (i, err)
            _check_topk(gi[lo:hi], gv[lo:hi], ref, err)
    finally:
        eng.close()


def test_draft_errors():
    eng, oh, d = _pair("small")
    f = _feats(8, d.hidden, seed=1)
    sh = synth.chain(3)
    toks = _tokens(sh.n, d.vocab, 1)
    with pytest.raises(Exception):  # no draft prefix for sequence 3
        eng.draft_step([3], f[: sh.n], [(toks, sh.parents)])
    bad = sh.parents.copy()
    bad[2] = 2
    eng.draft_prefill(3, f, _tokens(8, d.vocab, 2))
    with pytest.raises(Exception):  # malformed tree
        eng.draft_step([3], f[: sh.n], [(toks, bad)])
