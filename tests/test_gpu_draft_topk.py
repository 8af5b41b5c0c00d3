"""Ties in the draft head's top-10 (value desc, index asc), through the C ABI.

The draft LM head keeps, per 128-row vocabulary tile and row, the candidates
at or above the 10th largest of the tile's 32 per-lane maxima, and falls back
to an exact selection when more values than its candidate slots tie there.
These cases pin both paths with logits whose order is known without an
oracle: a reduced draft vocabulary whose LM-head rows are all zero (every
logit exactly 0: the 10 lowest token ids win), and one where 40 rows that
straddle a tile boundary share one vector (their logits tie exactly: the 10
lowest of them win when the shared logit is positive, the zero rows'
10 lowest ids when it is negative).
"""

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

K = 10
VD = 1500
DUP = np.arange(100, 140)  # local rows 100..139: 28 in vocabulary tile 0, 12 in tile 1


def _engine(d, wdev, lm_rows, ids):
    from speculative_decoding_06_b200.engine import SpecEngine
    dw = synth.draft_head_weights(d, seed=6, device="cuda")
    dw["vocab_ids"] = torch.as_tensor(ids, device="cuda")
    dw["lm_head"] = lm_rows
    return SpecEngine(d, wdev, max_batch=2, max_seq=256, max_nodes=64, draft=dw)


def _step(eng, d, seed):
    rng = np.random.default_rng([29, seed])
    P = 90
    f = synth.draft_features(P, d.hidden, seed=seed, device="cuda")
    eng.draft_prefill(0, f, rng.integers(0, d.vocab, size=P).astype(np.int32))
    sh = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=3)
    trees = [(synth.prefix_tokens(d.vocab, sh.n, stream=seed), sh.parents)]
    fn = synth.draft_features(sh.n, d.hidden, seed=seed + 1, device="cuda")
    gi, gv, _ = eng.draft_step([0], fn, trees, flags=2)
    return gi, gv, eng.debug_logits(sh.n, VD)


@pytest.fixture(scope="module")
def target():
    d = synth.SMALL_BF16
    return d, synth.model_weights(d, seed=0, device="cuda"), synth.draft_vocab_ids(d.vocab, VD)


def test_all_logits_tie(target):
    d, wdev, ids = target
    eng = _engine(d, wdev, torch.zeros(VD, d.hidden, dtype=torch.bfloat16, device="cuda"), ids)
    try:
        gi, gv, lg = _step(eng, d, 500)
        assert np.all(lg == 0.0)
        assert np.array_equal(gi, np.tile(ids[:K], (gi.shape[0], 1)))
        assert np.all(gv == 0.0)
    finally:
        eng.close()


def test_tied_rows_across_a_tile_boundary(target):
    d, wdev, ids = target
    lm = torch.zeros(VD, d.hidden, dtype=torch.bfloat16, device="cuda")
    g = torch.Generator(device="cpu").manual_seed(77)
    lm[torch.as_tensor(DUP, device="cuda")] = (torch.randn(d.hidden, generator=g) * 0.05).to(torch.bfloat16).cuda()
    eng = _engine(d, wdev, lm, ids)
    try:
        gi, gv, lg = _step(eng, d, 520)
        rest = np.setdiff1d(np.arange(VD), DUP)
        pos = neg = 0
        for r in range(gi.shape[0]):
            s = lg[r, DUP]
            assert np.all(s == s[0])  # identical rows give identical logits
            assert np.all(lg[r, rest] == 0.0)
            if s[0] > 0:
                pos += 1
                assert np.array_equal(gi[r], ids[DUP[:K]])
                assert np.all(gv[r] == s[0])
            elif s[0] < 0:
                neg += 1
                assert np.array_equal(gi[r], ids[rest[:K]])
                assert np.all(gv[r] == 0.0)
        assert pos > 0 and neg > 0
    finally:
        eng.close()
