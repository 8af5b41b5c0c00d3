"""Pins of the float64 oracle against facts fixed outside the oracle itself.

* the chain example and the acceptance rule printed on the course page
  ("EAGLE-3投机解码：树验证器方法", sections 问题 and 验证-接受语义), from
  tests/golden/chain_example.json;
* the four-path tree of section 树draft vs 链draft (tests/golden/tree_example.json);
* the Llama decoder as implemented by an independent library (Hugging Face
  transformers, float64, eager attention) for the causal forward, the K/V it
  caches, and -- via the tree = chain equivalence -- ancestor-only attention;
* library routines for RMSNorm and masked attention, a closed form for the
  rotary embedding;
* brute force: greedy decoding with a full recompute per token (losslessness),
  enumeration of fully matched root paths (the walk);
* the closed-form expectation of emitted tokens for planted trees.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import (OracleModel, accept_walk, causal_logits, oracle_greedy_ar, oracle_prefill,
                    oracle_tree_logits, oracle_verify, root_paths, tree_meta, argmax_fn_for_planting)
from oracle.model import attention, rms_norm, rope
from oracle.tree import TreeError
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

GQA_TINY = synth.ModelDims(2, 128, 8, 2, 16, 200, 300, 1e-5, 10000.0, "f32")


# ---------------------------------------------------------------------------
# fixtures
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny():
    w = synth.model_weights(synth.TINY, seed=0)
    return w, OracleModel(synth.TINY, synth.weights_to_host(w))


@pytest.fixture(scope="module")
def gqa():
    w = synth.model_weights(GQA_TINY, seed=0)
    return w, OracleModel(GQA_TINY, synth.weights_to_host(w))


def hf_model(d, w):
    from transformers import LlamaConfig, LlamaForCausalLM
    cfg = LlamaConfig(hidden_size=d.hidden, intermediate_size=d.ffn, num_hidden_layers=d.n_layers,
                      num_attention_heads=d.n_q_heads, num_key_value_heads=d.n_kv_heads,
                      head_dim=d.head_dim, vocab_size=d.vocab, rms_norm_eps=d.rms_eps,
                      rope_theta=d.rope_theta, tie_word_embeddings=False, attention_bias=False,
                      mlp_bias=False, max_position_embeddings=4096, attn_implementation="eager")
    m = LlamaForCausalLM(cfg).double().eval()
    sd = {"model.embed_tokens.weight": w["embed"], "lm_head.weight": w["lm_head"],
          "model.norm.weight": w["final_norm"]}
    names = {"wq": "self_attn.q_proj", "wk": "self_attn.k_proj", "wv": "self_attn.v_proj",
             "wo": "self_attn.o_proj", "w_gate": "mlp.gate_proj", "w_up": "mlp.up_proj",
             "w_down": "mlp.down_proj", "attn_norm": "input_layernorm", "mlp_norm": "post_attention_layernorm"}
    for l, lw in enumerate(w["layers"]):
        for k, hn in names.items():
            sd["model.layers.%d.%s.weight" % (l, hn)] = lw[k]
    sd = {k: v.to(torch.float64) for k, v in sd.items()}
    missing, unexpected = m.load_state_dict(sd, strict=False)
    assert not unexpected and all("rotary" in k for k in missing), (missing, unexpected)
    return m


# The library keeps RMSNorm statistics, the softmax and the rotary tables in
# float32 even in a float64 model, so agreement is at the 1e-7 level; a
# structural mistake (pairing, head mapping, a dropped term) shows up at 1e-2.
HF_ATOL = 5e-6
HF_RTOL = 1e-5


def hf_logits(m, tokens):
    with torch.no_grad():
        return m(torch.tensor([list(tokens)])).logits[0].numpy()


# ---------------------------------------------------------------------------
# the page's chain example and acceptance rule
# ---------------------------------------------------------------------------

def _chain_case(K, correct):
    """Chain root + K drafts whose first `correct` drafts equal the target's choice."""
    rng = np.random.default_rng(K * 10 + correct)
    amax = rng.integers(0, 1000, size=K + 1)
    tokens = np.zeros(K + 1, np.int64)
    tokens[0] = 7
    for j in range(1, K + 1):
        tokens[j] = amax[j - 1] if j <= correct else (amax[j - 1] + 1) % 1000
    return tokens, np.arange(-1, K), amax


def test_chain_example_from_page():
    g = json.load(open(os.path.join(GOLDEN, "chain_example.json")))
    for case in g["cases"]:
        tokens, parents, amax = _chain_case(g["K"], case["correct"])
        acc, bonus = accept_walk(tokens, parents, amax)
        assert len(acc) + 1 == case["emitted"]
        assert bonus == amax[len(acc)]
        assert acc == list(range(1, case["correct"] + 1))


def test_chain_all_correct_gives_k_plus_one():
    tokens, parents, amax = _chain_case(5, 5)
    acc, bonus = accept_walk(tokens, parents, amax)
    assert len(acc) == 5 and bonus == amax[5]


def test_walk_stops_at_first_mismatch_even_if_later_drafts_match():
    # d_3 wrong: d_4 and d_5 are never checked (course page, section 树draft vs 链draft)
    tokens, parents, amax = _chain_case(5, 2)
    tokens[4] = amax[3]
    tokens[5] = amax[4]
    acc, _ = accept_walk(tokens, parents, amax)
    assert acc == [1, 2]


def test_chain_example_on_model(tiny):
    """End to end: a chain whose first k drafts follow greedy decoding emits k+1 greedy tokens."""
    _, om = tiny
    prompt = synth.prefix_tokens(synth.TINY.vocab, 16, stream=7)
    greedy = oracle_greedy_ar(om, prompt, 7)
    g = json.load(open(os.path.join(GOLDEN, "chain_example.json")))
    for case in g["cases"] + [{"correct": 5, "emitted": 6}]:
        k = case["correct"]
        seq, _ = oracle_prefill(om, prompt)
        assert seq.pending == greedy[0]
        drafts = list(greedy[1:1 + k]) + [(greedy[1 + k] + 1) % synth.TINY.vocab] * (5 - k)
        r = oracle_verify(om, seq, [seq.pending] + drafts, list(range(-1, 5)))
        emitted = r["accepted_tokens"] + [r["bonus"]]
        assert len(emitted) == case["emitted"]
        assert emitted == greedy[1:1 + len(emitted)]


def test_tree_example_has_four_paths():
    g = json.load(open(os.path.join(GOLDEN, "tree_example.json")))
    parents = g["parents"]
    depth, anc = tree_meta(parents)
    leaves = [i for i in range(len(parents)) if i not in parents]
    assert len(leaves) == g["paths"]
    for leaf in leaves:
        assert len(anc[leaf]) == 4 and anc[leaf][0] == 0 and depth[leaf] == 3


def test_walk_equals_deepest_fully_matched_path():
    """Brute force: with distinct sibling tokens, the walk ends at the deepest node whose whole root path matches."""
    rng = np.random.default_rng(11)
    for trial in range(300):
        n = int(rng.integers(1, 40))
        parents = [-1] + [int(rng.integers(0, i)) for i in range(1, n)]
        tokens = np.zeros(n, np.int64)
        for i in range(1, n):
            sib_tokens = {tokens[j] for j in range(1, i) if parents[j] == parents[i]}
            t = int(rng.integers(0, 6))
            while t in sib_tokens:
                t += 1
            tokens[i] = t
        amax = rng.integers(0, 6, size=n)
        paths = root_paths(parents)
        full = [i for i in range(n) if all(tokens[c] == amax[parents[c]] for c in paths[i][1:])]
        deepest = max(full, key=lambda i: len(paths[i]))
        assert sum(len(paths[i]) == len(paths[deepest]) for i in full) == 1
        acc, bonus = accept_walk(tokens, parents, amax)
        assert acc == paths[deepest][1:]
        assert bonus == amax[deepest]


def test_duplicate_siblings_take_lowest_index():
    parents = [-1, 0, 0, 1, 2]
    tokens = [5, 3, 3, 9, 9]
    amax = [3, 9, 9, 0, 0]
    acc, bonus = accept_walk(tokens, parents, amax)
    assert acc == [1, 3] and bonus == 0


@pytest.mark.parametrize("parents", [[0], [-1, 1], [-1, 0, 3, 1], [-1, -1], [-1, 0, 2]])
def test_malformed_parents_rejected(parents):
    with pytest.raises(TreeError):
        tree_meta(parents)


# ---------------------------------------------------------------------------
# decoder pieces against library routines and closed forms
# ---------------------------------------------------------------------------

def test_rms_norm_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(5, 64))
    w = rng.normal(size=64)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (64,), torch.tensor(w), eps=1e-5).numpy()
    np.testing.assert_allclose(rms_norm(x, w, 1e-5), ref, rtol=1e-13, atol=1e-13)


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(1)
    T, S, Hq, Hkv, hd = 6, 11, 8, 2, 16
    q = rng.normal(size=(T, Hq, hd))
    k = rng.normal(size=(S, Hkv, hd))
    v = rng.normal(size=(S, Hkv, hd))
    vis = rng.random((T, S)) < 0.6
    vis[:, 0] = True
    ours = attention(q, k, v, vis)
    qt = torch.tensor(q).transpose(0, 1)
    kt = torch.tensor(k).transpose(0, 1).repeat_interleave(Hq // Hkv, dim=0)
    vt = torch.tensor(v).transpose(0, 1).repeat_interleave(Hq // Hkv, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.tensor(vis))
    np.testing.assert_allclose(ours, ref.transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)


def test_rope_closed_form_and_relative_position():
    # head_dim 4, theta 100: frequencies 1 and 0.1; pairs are (0, 2) and (1, 3)
    x = np.array([[[1.0, 0.0, 0.0, 2.0]]])
    y = rope(x, np.array([3]), 100.0)[0, 0]
    np.testing.assert_allclose(y, [math.cos(3), -2 * math.sin(0.3), math.sin(3), 2 * math.cos(0.3)], atol=1e-15)
    rng = np.random.default_rng(2)
    q = rng.normal(size=(1, 1, 64))
    k = rng.normal(size=(1, 1, 64))
    d1 = np.sum(rope(q, np.array([10]), 1e4) * rope(k, np.array([3]), 1e4))
    d2 = np.sum(rope(q, np.array([1010]), 1e4) * rope(k, np.array([1003]), 1e4))
    assert abs(d1 - d2) < 1e-10
    np.testing.assert_allclose(np.linalg.norm(rope(q, np.array([77]), 1e4)), np.linalg.norm(q), rtol=1e-14)


# ---------------------------------------------------------------------------
# the whole decoder against an independent implementation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("which", ["tiny", "gqa"])
def test_causal_forward_matches_hf_llama(which, tiny, gqa):
    w, om = tiny if which == "tiny" else gqa
    d = om.d
    m = hf_model(d, w)
    toks = synth.prefix_tokens(d.vocab, 37, stream=3)
    np.testing.assert_allclose(causal_logits(om, toks), hf_logits(m, toks), rtol=HF_RTOL, atol=HF_ATOL)


def test_tree_node_equals_chain_over_its_root_path(gqa):
    """Ancestor-only attention: node i's logits equal a causal forward over prefix + root path of i."""
    w, om = gqa
    d = om.d
    m = hf_model(d, w)
    prompt = synth.prefix_tokens(d.vocab, 20, stream=4)
    seq, _ = oracle_prefill(om, prompt)
    shape = synth.tree_from_widths((3, 4, 3, 2), stream=1)
    rng = np.random.default_rng(5)
    tokens = rng.integers(0, d.vocab, size=shape.n)
    tokens[0] = seq.pending
    logits, _ = oracle_tree_logits(om, seq, tokens, shape.parents)
    for i, path in enumerate(root_paths(shape.parents)):
        ref = hf_logits(m, list(prompt) + [int(tokens[j]) for j in path])[-1]
        np.testing.assert_allclose(logits[i], ref, rtol=HF_RTOL, atol=HF_ATOL)


def test_non_ancestor_tokens_do_not_change_a_node(tiny):
    _, om = tiny
    prompt = synth.prefix_tokens(synth.TINY.vocab, 24, stream=5)
    seq, _ = oracle_prefill(om, prompt)
    shape = synth.tree_from_widths((3, 3, 2), stream=2)
    rng = np.random.default_rng(6)
    tokens = rng.integers(0, synth.TINY.vocab, size=shape.n)
    tokens[0] = seq.pending
    base, _ = oracle_tree_logits(om, seq, tokens, shape.parents)
    _, anc = tree_meta(shape.parents)
    for j in range(1, shape.n):
        t2 = tokens.copy()
        t2[j] = (t2[j] + 17) % synth.TINY.vocab
        pert, _ = oracle_tree_logits(om, seq, t2, shape.parents)
        for i in range(shape.n):
            if j not in anc[i]:
                assert np.array_equal(pert[i], base[i])
            elif i == j:
                assert not np.array_equal(pert[i], base[i])


def test_root_only_tree_is_one_greedy_step(tiny):
    _, om = tiny
    prompt = synth.prefix_tokens(synth.TINY.vocab, 30, stream=6)
    greedy = oracle_greedy_ar(om, prompt, 2)
    seq, _ = oracle_prefill(om, prompt)
    r = oracle_verify(om, seq, [seq.pending], [-1])
    assert r["accepted_len"] == 0 and r["bonus"] == greedy[1]
    assert seq.length == len(prompt) + 1 and seq.tokens[-1] == greedy[0]


# ---------------------------------------------------------------------------
# losslessness and KV compaction
# ---------------------------------------------------------------------------

def _decode_with_trees(om, prompt, n_tokens, tree_fn, p, stream):
    seq, _ = oracle_prefill(om, prompt)
    emitted = [seq.pending]
    step = 0
    taus = []
    while len(emitted) < n_tokens + 1:
        shape = tree_fn(step)
        draws = synth.plant_draws(shape.n, om.d.vocab, stream=stream * 1000 + step)
        toks = synth.plant_tree(shape, seq.pending, p, draws, argmax_fn_for_planting(om, seq))
        r = oracle_verify(om, seq, toks, shape.parents)
        emitted += r["accepted_tokens"] + [r["bonus"]]
        taus.append(r["accepted_len"] + 1)
        step += 1
    return seq, emitted, taus


def test_losslessness_against_brute_force_greedy(tiny):
    """Repeated verify steps over planted and random trees emit exactly the greedy tokens."""
    _, om = tiny
    prompt = synth.prefix_tokens(synth.TINY.vocab, 64, seed=1)
    n = 200
    greedy = oracle_greedy_ar(om, prompt, n + 1)

    def tree_fn(step):
        kind = step % 4
        if kind == 0:
            return synth.tiny_tree()
        if kind == 1:
            return synth.tree_from_widths((4, 4, 3, 2, 2), stream=step)
        if kind == 2:
            return synth.chain(1 + step % 7)
        return synth.tree_from_widths((2, 2), stream=step)

    for p, stream in ((0.8, 1), (0.0, 2)):
        seq, emitted, taus = _decode_with_trees(om, prompt, n, tree_fn, p, stream)
        m = min(len(emitted), len(greedy))
        assert emitted[:m] == greedy[:m]
        if p > 0:
            assert np.mean(taus) > 1.5


def test_compacted_cache_matches_hf_cache(gqa):
    """After several verify steps the cache equals the K/V a causal forward over the emitted tokens writes."""
    w, om = gqa
    d = om.d
    prompt = synth.prefix_tokens(d.vocab, 12, stream=8)
    seq, emitted, taus = _decode_with_trees(om, prompt, 25, lambda s: synth.tree_from_widths((3, 3, 2, 2), stream=s),
                                            0.8, 3)
    assert seq.tokens == list(prompt) + emitted[:-1]
    m = hf_model(d, w)
    with torch.no_grad():
        cache = m(torch.tensor([seq.tokens]), use_cache=True).past_key_values
    for l in range(d.n_layers):
        hk = cache.layers[l].keys[0].transpose(0, 1).numpy()
        hv = cache.layers[l].values[0].transpose(0, 1).numpy()
        np.testing.assert_allclose(seq.k[l], hk, rtol=HF_RTOL, atol=HF_ATOL)
        np.testing.assert_allclose(seq.v[l], hv, rtol=HF_RTOL, atol=HF_ATOL)


# ---------------------------------------------------------------------------
# planted acceptance: closed-form expectation
# ---------------------------------------------------------------------------

def expected_emitted(parents, p):
    """1 + f(root) with f(v) = sum_j (1-p)^(j-1) p (1 + f(c_j)) over v's children in index order."""
    n = len(parents)
    children = [[] for _ in range(n)]
    for i in range(1, n):
        children[parents[i]].append(i)
    f = np.zeros(n)
    second = np.zeros(n)  # E[(count from v)^2] for the variance
    for v in range(n - 1, -1, -1):
        ev, ev2 = 0.0, 0.0
        for j, c in enumerate(children[v]):
            w_ = (1 - p) ** j * p
            ev += w_ * (1 + f[c])
            ev2 += w_ * (1 + 2 * f[c] + second[c])
        f[v], second[v] = ev, ev2
    return 1 + f[0], second[0] - f[0] ** 2


def test_expected_emitted_closed_form_for_chains():
    for gamma, want in ((5, 4.152), (8, 5.123)):
        e, _ = expected_emitted(list(range(-1, gamma)), 0.85)
        assert abs(e - want) < 1e-3
        assert abs(e - (1 - 0.85 ** (gamma + 1)) / 0.15) < 1e-12


@pytest.mark.parametrize("kind", ["chain5", "tree60"])
def test_planted_acceptance_matches_expectation(tiny, kind):
    _, om = tiny
    prompt = synth.prefix_tokens(synth.TINY.vocab, 32, stream=9)
    seq, _ = oracle_prefill(om, prompt)
    shape = synth.chain(5) if kind == "chain5" else synth.tree_from_widths(synth.TREE60_WIDTHS, stream=0)
    p = 0.85 if kind == "chain5" else 0.8
    mean, var = expected_emitted(list(shape.parents), p)
    fn = argmax_fn_for_planting(om, seq)
    samples = 200 if kind == "chain5" else 120
    got = []
    for s in range(samples):
        draws = synth.plant_draws(shape.n, synth.TINY.vocab, stream=100 + s)
        toks = synth.plant_tree(shape, seq.pending, p, draws, fn)
        logits, _ = oracle_tree_logits(om, seq, toks, shape.parents)
        acc, _ = accept_walk(toks, shape.parents, np.argmax(logits, axis=1))
        got.append(len(acc) + 1)
    assert abs(np.mean(got) - mean) < 3 * math.sqrt(var / samples) + 0.02
