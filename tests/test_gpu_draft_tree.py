"""The dynamic draft tree (spec_draft_tree) against the float64 oracle's tree builder.

Multi-step drafting ("EAGLE-3: Scaling up Inference Acceleration of Large
Language Models via Training-Time Test", draft-stage description): from the
second step on the draft's own output a of the parent replaces the target
feature.  The tree's shape follows the draft's confidence (its account of
EAGLE-2); the steps the pages leave open are read as in the oracle
(oracle/draft.py, build_draft_tree).

Checks: every output tree is well formed and rooted at the pending token; each
node's value (sum of draft log-probabilities along its path) matches the
oracle's value of the same path within the logit tolerance per step; and where
every selection the oracle makes is decided by a margin above that tolerance,
the GPU tree is the oracle's tree node for node.
"""

import numpy as np
import pytest
import torch

import synth
from oracle.draft import OracleDraftHead, build_draft_tree, log_softmax_rows
from gpu_common import TOL

pytestmark = pytest.mark.gpu


def _host(t):
    return synth.tensor_to_host(t)


def _path_value(oh, seq, g_root, root, toks):
    """Oracle value of a root path, by causal recompute with the draft's own outputs as features."""
    P = seq.length
    rows_t, gs, total = [root], [g_root], 0.0
    for t in toks:
        T = len(rows_t)
        x = oh.rows_from_g(np.stack(gs), rows_t)
        a, _, _ = oh.layer_model.layer_forward(0, x, P + np.arange(T), seq.k, seq.v, np.tril(np.ones((T, T), bool)))
        lp, _ = log_softmax_rows(oh.layer_model.lm_logits(a[-1:]))
        total += lp[0, t]
        rows_t.append(int(t))
        gs.append(a[-1])
    return total


def _decisive(tree, steps, topk, total, tol):
    """True when every selection in the oracle's build is decided by more than `tol`."""
    off = tree.offered
    per = [off[:topk]] + [off[topk + s * topk * topk: topk + (s + 1) * topk * topk] for s in range(steps - 1)]
    for grp in per[1:]:
        v = sorted((c[0] for c in grp), reverse=True)
        if len(v) > topk and v[topk - 1] - v[topk] <= tol:
            return False
    v = sorted((c[0] for c in off), reverse=True)
    return not (len(v) > total and v[total - 1] - v[total] <= tol)


@pytest.mark.parametrize("steps,topk,total", [(3, 4, 8), (2, 8, 12), (8, 10, 60)])
def test_draft_tree_matches_oracle(steps, topk, total):
    """(8, 10, 60) is the pages' evaluated setting: 8 drafting steps, top-10, 60 draft tokens."""
    from speculative_decoding_06_b200.engine import SpecEngine
    d = synth.SMALL_BF16
    wdev = synth.model_weights(d, seed=0, device="cuda")
    dwdev = synth.draft_head_weights(d, seed=6, device="cuda")
    eng = SpecEngine(d, wdev, max_batch=3, max_seq=512, max_nodes=128, draft=dwdev)
    oh = OracleDraftHead(d, synth.weights_to_host(wdev),
                         {"fc_fuse": _host(dwdev["fc_fuse"]), "fc_in": _host(dwdev["fc_in"]),
                          "final_norm": _host(dwdev["final_norm"]),
                          "layer": {k: _host(v) for k, v in dwdev["layer"].items()}})
    try:
        B = 3
        rng = np.random.default_rng([11, steps])
        seqs = []
        for b in range(B):
            P = 60 + 23 * b
            f = synth.draft_features(P, d.hidden, seed=200 + b, device="cuda")
            toks = rng.integers(0, d.vocab, size=P).astype(np.int32)
            eng.draft_prefill(b, f, toks)
            seqs.append(oh.prefill(_host(f.cpu()), toks))
        root_feats = synth.draft_features(B, d.hidden, seed=300 + steps, device="cuda")
        roots = rng.integers(0, d.vocab, size=B).astype(np.int32)
        tok, par, val = eng.draft_tree(list(range(B)), root_feats, roots, steps=steps, topk=topk, total=total)
        rf = _host(root_feats.cpu())
        tol = 2.5 * TOL["bf16"]  # one logit and one log-sum-exp per step along a path
        err_step = 1e-6  # the largest value error per drafting step seen in these trees
        g_roots = []
        for b in range(B):
            assert tok[b, 0] == roots[b] and par[b, 0] == -1
            assert all(0 <= par[b, i] < i for i in range(1, total + 1))
            g_root = oh.fuse(rf[b:b + 1])[0]
            g_roots.append(g_root)
            for i in range(1, total + 1):
                path, j = [], i
                while j > 0:
                    path.append(int(tok[b, j]))
                    j = int(par[b, j])
                path.reverse()
                ref = _path_value(oh, seqs[b], g_root, int(roots[b]), path)
                err = abs(val[b, i] - ref)
                assert err <= tol * len(path), "tree %d node %d: value %.4f vs %.4f" % (b, i, val[b, i], ref)
                err_step = max(err_step, err / len(path))
        # where every selection of the oracle's build is decided by more than the error two
        # compared values can carry, the GPU tree is the oracle's, node for node
        matched = 0
        for b in range(B):
            ot = build_draft_tree(oh, seqs[b], g_roots[b], int(roots[b]), steps=steps, topk=topk, total=total)
            if _decisive(ot, steps, topk, total, 2.5 * err_step * steps):
                assert list(tok[b]) == list(ot.tokens) and list(par[b]) == list(ot.parents), "tree %d" % b
                matched += 1
        print("value error per step %.2g; decisive trees compared node for node: %d of %d" % (err_step, matched, B))
        # the draft prefixes are unchanged
        assert [eng.draft_len(b) for b in range(B)] == [60, 83, 106]
    finally:
        eng.close()


def test_draft_tree_limits():
    from speculative_decoding_06_b200.engine import SpecEngine
    from speculative_decoding_06_b200 import spec as S
    d = synth.SMALL_BF16
    eng = SpecEngine(d, synth.model_weights(d, seed=0, device="cuda"), max_batch=1, max_seq=256, max_nodes=32,
                     draft=synth.draft_head_weights(d, seed=6, device="cuda"))
    try:
        rf = synth.draft_features(1, d.hidden, seed=1, device="cuda")
        with pytest.raises(S.SpecError):  # no draft prefix yet
            eng.draft_tree([0], rf, [5], steps=2, topk=4, total=4)
        eng.draft_prefill(0, synth.draft_features(10, d.hidden, seed=2, device="cuda"),
                          np.arange(10, dtype=np.int32))
        with pytest.raises(S.SpecError):  # topk 5 is not a supported list length
            eng.draft_tree([0], rf, [5], steps=2, topk=5, total=4)
        with pytest.raises(S.SpecError):  # 1 + 7 * 10 rows exceed max_nodes 32
            eng.draft_tree([0], rf, [5], steps=8, topk=10, total=20)
        tok, par, _ = eng.draft_tree([0], rf, [5], steps=1, topk=4, total=4)
        assert list(par[0]) == [-1, 0, 0, 0, 0]  # one step: the root's top-4
    finally:
        eng.close()
