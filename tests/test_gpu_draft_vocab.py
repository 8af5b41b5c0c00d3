"""The draft head over a reduced vocabulary (spec_config.draft_vocab) against the
float64 oracle: VocabTrim / FR-Spec / SpecVocab in the aitangshan.cn walkthrough
(sections 1 and 3.2) shrink the draft head's output to a subset of tokens.  The
draft LM head is the target's rows of the kept token ids, the draft softmax
covers that subset, and every drafted token is one of them.

Checked through the C ABI on a seeded subset of 1500 of the 8320 tokens:
the draft step's logits over the subset (2e-2), its top-10 candidates as token
ids (by rank where the oracle's gaps leave no doubt, as a set where rank 10
leads rank 11), and the dynamic draft tree (values within the per-step
tolerance of the oracle's path values over the subset, every token in the
subset, and the oracle's tree node for node where its selections are decided).
"""

import numpy as np
import pytest
import torch

import synth
from oracle.draft import OracleDraftHead, build_draft_tree, log_softmax_rows, top_k_rows
from gpu_common import TOL

pytestmark = pytest.mark.gpu

K = 10
VD = 1500


def _host(t):
    return synth.tensor_to_host(t)


@pytest.fixture(scope="module")
def pair():
    from speculative_decoding_06_b200.engine import SpecEngine
    d = synth.SMALL_BF16
    wdev = synth.model_weights(d, seed=0, device="cuda")
    dw = synth.draft_head_weights(d, seed=6, device="cuda")
    ids = synth.draft_vocab_ids(d.vocab, VD)
    dw["vocab_ids"] = torch.as_tensor(ids, device="cuda")
    dw["lm_head"] = wdev["lm_head"][dw["vocab_ids"].long()].contiguous()
    eng = SpecEngine(d, wdev, max_batch=3, max_seq=512, max_nodes=128, draft=dw)
    oh = OracleDraftHead(d, synth.weights_to_host(wdev),
                         {"fc_fuse": _host(dw["fc_fuse"]), "fc_in": _host(dw["fc_in"]),
                          "final_norm": _host(dw["final_norm"]),
                          "layer": {k: _host(v) for k, v in dw["layer"].items()}}, vocab_ids=ids)
    yield eng, oh, d, ids
    eng.close()


def _prefill(eng, oh, d, B, seed):
    rng = np.random.default_rng([13, seed])
    seqs = []
    for b in range(B):
        P = 70 + 31 * b
        f = synth.draft_features(P, d.hidden, seed=seed + b, device="cuda")
        toks = rng.integers(0, d.vocab, size=P).astype(np.int32)
        eng.draft_prefill(b, f, toks)
        seqs.append(oh.prefill(_host(f.cpu()), toks))
    return seqs


def test_reduced_vocab_draft_step(pair):
    eng, oh, d, ids = pair
    seqs = _prefill(eng, oh, d, 2, 400)
    shapes = [synth.tree_from_widths(synth.TREE60_WIDTHS, stream=7), synth.tree_from_widths((4, 3, 2), stream=8)]
    trees = [(synth.prefix_tokens(d.vocab, sh.n, stream=90 + i), sh.parents) for i, sh in enumerate(shapes)]
    M = sum(sh.n for sh in shapes)
    fn = synth.draft_features(M, d.hidden, seed=410, device="cuda")
    gi, gv, off = eng.draft_step([0, 1], fn, trees, flags=2)
    logits = eng.debug_logits(M, VD)
    fh = _host(fn.cpu())
    pos = {int(t): j for j, t in enumerate(ids)}
    assert np.all(np.isin(gi, ids))
    for i, (seq, (toks, par)) in enumerate(zip(seqs, trees)):
        lo, hi = int(off[i]), int(off[i + 1])
        ref = oh.step_logits(seq, fh[lo:hi], toks, par)  # [n][VD]
        err = float(np.max(np.abs(logits[lo:hi] - ref)))
        assert err <= TOL["bf16"], "sequence %d: max |logit error| %.3g" % (i, err)
        oi, ov = top_k_rows(ref, K + 1)
        thr = max(2.5 * err, 1e-6)
        for r in range(hi - lo):
            g = gi[lo + r]
            np.testing.assert_allclose(gv[lo + r], ref[r, [pos[int(t)] for t in g]], atol=TOL["bf16"])
            for j in range(K):
                lo_gap = ov[r, j] - ov[r, j + 1]
                hi_gap = ov[r, j - 1] - ov[r, j] if j > 0 else np.inf
                if lo_gap > thr and hi_gap > thr:
                    assert g[j] == ids[oi[r, j]], "row %d rank %d" % (r, j)
            if ov[r, K - 1] - ov[r, K] > thr:
                assert set(g.tolist()) == set(ids[oi[r, :K]].tolist())


def _path_value(oh, seq, g_root, root, toks, pos):
    P = seq.length
    rows_t, gs, total = [root], [g_root], 0.0
    for t in toks:
        T = len(rows_t)
        x = oh.rows_from_g(np.stack(gs), rows_t)
        a, _, _ = oh.layer_model.layer_forward(0, x, P + np.arange(T), seq.k, seq.v, np.tril(np.ones((T, T), bool)))
        lp, _ = log_softmax_rows(oh.layer_model.lm_logits(a[-1:]))
        total += lp[0, pos[int(t)]]
        rows_t.append(int(t))
        gs.append(a[-1])
    return total


def test_reduced_vocab_draft_tree(pair):
    eng, oh, d, ids = pair
    B, steps, topk, total = 2, 3, 4, 8
    seqs = _prefill(eng, oh, d, B, 500)
    rf = synth.draft_features(B, d.hidden, seed=510, device="cuda")
    roots = np.array([17, 4321], np.int32)
    tok, par, val = eng.draft_tree(list(range(B)), rf, roots, steps=steps, topk=topk, total=total)
    rfh = _host(rf.cpu())
    pos = {int(t): j for j, t in enumerate(ids)}
    tol = 2.5 * TOL["bf16"]
    matched = 0
    for b in range(B):
        assert tok[b, 0] == roots[b] and np.all(np.isin(tok[b, 1:], ids))
        g_root = oh.fuse(rfh[b:b + 1])[0]
        for i in range(1, total + 1):
            path, j = [], i
            while j > 0:
                path.append(int(tok[b, j]))
                j = int(par[b, j])
            path.reverse()
            ref = _path_value(oh, seqs[b], g_root, int(roots[b]), path, pos)
            assert abs(val[b, i] - ref) <= tol * len(path)
        ot = build_draft_tree(oh, seqs[b], g_root, int(roots[b]), steps=steps, topk=topk, total=total)
        vals = sorted((c[0] for c in ot.offered), reverse=True)
        if vals[total - 1] - vals[total] > 1e-3:
            assert list(tok[b]) == list(ot.tokens) and list(par[b]) == list(ot.parents)
            matched += 1
    print("reduced-vocabulary trees compared node for node: %d of %d" % (matched, B))
