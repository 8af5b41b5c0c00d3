"""Plant plausible mistakes in the oracle and check that its pins catch each one.

Every mutation is applied to the oracle on the CPU with monkeypatch, never to
the CUDA path.  Each case reruns the pin that must fail and asserts that it does.
"""

import numpy as np
import pytest
import torch

import oracle.model as om_mod
import oracle.tree as tree_mod
from oracle import OracleModel, accept_walk, causal_logits, oracle_prefill, oracle_tree_logits, root_paths
import synth

from test_oracle_pins import GQA_TINY, HF_ATOL, hf_logits, hf_model


@pytest.fixture(scope="module")
def gqa_setup():
    w = synth.model_weights(GQA_TINY, seed=0)
    return w, hf_model(GQA_TINY, w)


def _causal_ok(w, m):
    om = OracleModel(GQA_TINY, synth.weights_to_host(w))
    toks = synth.prefix_tokens(GQA_TINY.vocab, 19, stream=3)
    return np.allclose(causal_logits(om, toks), hf_logits(m, toks), rtol=1e-5, atol=HF_ATOL)


def _tree_ok(w, m):
    om = OracleModel(GQA_TINY, synth.weights_to_host(w))
    prompt = synth.prefix_tokens(GQA_TINY.vocab, 9, stream=4)
    seq, _ = oracle_prefill(om, prompt)
    shape = synth.tree_from_widths((3, 3, 2), stream=1)
    rng = np.random.default_rng(5)
    tokens = rng.integers(0, GQA_TINY.vocab, size=shape.n)
    tokens[0] = seq.pending
    logits, _ = oracle_tree_logits(om, seq, tokens, shape.parents)
    for i, path in enumerate(root_paths(shape.parents)):
        ref = hf_logits(m, list(prompt) + [int(tokens[j]) for j in path])[-1]
        if not np.allclose(logits[i], ref, rtol=1e-5, atol=HF_ATOL):
            return False
    return True


def test_unmutated_passes(gqa_setup):
    assert _causal_ok(*gqa_setup) and _tree_ok(*gqa_setup)


def _interleaved_rope(x, pos, theta):
    hd = x.shape[-1]
    inv = theta ** (-(np.arange(hd // 2) * 2.0) / hd)
    ang = np.asarray(pos, float)[:, None] * inv[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _modulo_gqa(q, k, v, visible):
    T, Hq, hd = q.shape
    Hkv = k.shape[1]
    out = np.empty_like(q)
    for h in range(Hq):
        kh = h % Hkv
        s = (q[:, h] @ k[:, kh].T) / np.sqrt(hd)
        s = np.where(visible, s, -np.inf)
        p = np.exp(s - s.max(1, keepdims=True))
        out[:, h] = (p / p.sum(1, keepdims=True)) @ v[:, kh]
    return out


def _norm_without_eps_in_root(x, w, eps):
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * w * 1.001


def _silu_as_sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


@pytest.mark.parametrize("name,attr,fn", [
    ("interleaved rotary pairing", "rope", _interleaved_rope),
    ("query head mapped modulo", "attention", _modulo_gqa),
    ("norm scaled wrongly", "rms_norm", _norm_without_eps_in_root),
    ("silu replaced by sigmoid", "silu", _silu_as_sigmoid),
])
def test_decoder_mutations_fail_the_library_pin(gqa_setup, monkeypatch, name, attr, fn):
    monkeypatch.setattr(om_mod, attr, fn)
    assert not _causal_ok(*gqa_setup), name


def test_positions_by_index_instead_of_depth_fail_tree_pin(gqa_setup, monkeypatch):
    real = tree_mod.tree_meta

    def by_index(parents):
        depth, anc = real(parents)
        return np.arange(len(depth)), anc
    monkeypatch.setattr(om_mod, "tree_meta", by_index)
    assert not _tree_ok(*gqa_setup)


def test_dropping_the_ancestor_mask_fails_tree_pin(gqa_setup, monkeypatch):
    monkeypatch.setattr(om_mod, "ancestor_matrix", lambda parents: np.tril(np.ones((len(parents),) * 2, bool)))
    assert not _tree_ok(*gqa_setup)


def test_walk_taking_highest_index_child_fails_duplicate_pin():
    parents = [-1, 0, 0, 1, 2]
    tokens = [5, 3, 3, 9, 9]
    amax = [3, 9, 0, 0, 0]

    def walk_highest(tokens, parents, argmax):
        p = list(parents)
        cur, acc = 0, []
        while True:
            kids = [c for c in range(1, len(p)) if p[c] == cur and tokens[c] == argmax[cur]]
            if not kids:
                return acc, int(argmax[cur])
            cur = kids[-1]
            acc.append(cur)

    assert accept_walk(tokens, parents, amax) == ([1, 3], 0)
    assert walk_highest(tokens, parents, amax) != ([1, 3], 0)
