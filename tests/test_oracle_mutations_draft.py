"""Plant plausible mistakes in the oracle's feature tap and draft-tree builder and
check that their pins catch each one (mutations on the CPU oracle only, with
monkeypatch; the CUDA path is never touched).

* a feature tapped one layer early, or after the final norm -> the Hugging Face
  hidden-state pin fails;
* a draft node fed its own output a instead of its parent's -> the greedy-chain
  pin (the worked example's step 2 / step 3 feeding) fails;
* node values from raw logits instead of log-probabilities -> the brute-force
  selection pin fails (or the builder's own ancestor-closure check does).
"""

import numpy as np
import pytest
import torch

import oracle.draft as draft_mod
import oracle.model as model_mod
import synth
from oracle.draft import build_draft_tree, greedy_draft_chain
from oracle.model import causal_features
from test_oracle_features import GQA3, gqa3  # noqa: F401  (fixture)
from test_oracle_pins import HF_ATOL, HF_RTOL, hf_model
from test_oracle_draft_tree import DIMS, _path_logprob, head  # noqa: F401  (fixture)


def _hf_features_ok(w, om):
    m = hf_model(GQA3, w)
    toks = synth.prefix_tokens(GQA3.vocab, 21, stream=9)
    feats = causal_features(om, toks, (1, 2))
    with torch.no_grad():
        hs = m(torch.tensor([list(toks)]), output_hidden_states=True).hidden_states
    return all(np.allclose(feats[:, f], hs[j][0].numpy(), rtol=HF_RTOL, atol=HF_ATOL) for f, j in enumerate((1, 2)))


def test_unmutated_features_pass(gqa3):  # noqa: F811
    assert _hf_features_ok(*gqa3)


def test_tap_one_layer_early_is_caught(gqa3, monkeypatch):  # noqa: F811
    w, om = gqa3
    orig = model_mod.OracleModel.forward_features

    def early(self, tokens, pos, past, vis_new, taps):
        return orig(self, tokens, pos, past, vis_new, [max(1, j - 1) for j in taps])

    monkeypatch.setattr(model_mod.OracleModel, "forward_features", early)
    assert not _hf_features_ok(w, om)


def test_tap_after_the_final_norm_is_caught(gqa3, monkeypatch):  # noqa: F811
    w, om = gqa3
    orig = model_mod.OracleModel.forward_features

    def normed(self, tokens, pos, past, vis_new, taps):
        logits, kv, feats = orig(self, tokens, pos, past, vis_new, taps)
        fw = model_mod.to_f64(self.w["final_norm"])
        return logits, kv, np.stack([model_mod.rms_norm(feats[:, f], fw, self.d.rms_eps)
                                     for f in range(feats.shape[1])], axis=1)

    monkeypatch.setattr(model_mod.OracleModel, "forward_features", normed)
    assert not _hf_features_ok(w, om)


def test_own_output_instead_of_parents_is_caught(head, monkeypatch):  # noqa: F811
    h, seq, g_root = head
    chain = greedy_draft_chain(h, seq, g_root, 5, 6)
    orig = draft_mod.OracleDraftHead.step_g

    def own_a(self, seq_, g, tokens, parents):
        # feed each non-root node the first-step output of itself (its own row) instead of its parent's
        logits, a = orig(self, seq_, g, tokens, parents)
        g2 = g.copy()
        for i in range(1, len(tokens)):
            g2[i] = a[i]
        return orig(self, seq_, g2, tokens, parents)

    monkeypatch.setattr(draft_mod.OracleDraftHead, "step_g", own_a)
    tree = build_draft_tree(h, seq, g_root, 5, steps=6, topk=1, total=6)
    assert list(tree.tokens[1:]) != chain


def test_raw_logit_values_are_caught(head, monkeypatch):  # noqa: F811
    h, seq, g_root = head
    monkeypatch.setattr(draft_mod, "log_softmax_rows", lambda logits: (logits, np.zeros(len(logits))))
    V = DIMS.vocab
    try:
        tree = build_draft_tree(h, seq, g_root, 3, steps=2, topk=V, total=20)
    except AssertionError:
        return  # caught by the builder's own closure check: values no longer fall along paths
    paths = [(a,) for a in range(V)] + [(a, b) for a in range(V) for b in range(V)]
    monkeypatch.undo()
    vals = {p: _path_logprob(h, seq, g_root, 3, p) for p in paths}
    chosen = set()
    for i in range(1, len(tree.tokens)):
        p, j = [], i
        while j > 0:
            p.append(int(tree.tokens[j]))
            j = int(tree.parents[j])
        chosen.add(tuple(reversed(p)))
    ranked = sorted(paths, key=lambda p: (-vals[p], len(p)))
    assert chosen != set(ranked[:20])
