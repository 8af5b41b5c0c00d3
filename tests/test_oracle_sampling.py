"""Pins of the oracle's stochastic (temperature) tree verification.

The reading (oracle/sampling.py): every draft token is a point-mass proposal in
Leviathan et al.'s speculative sampling (cited by "EAGLE-3投机解码：树验证器方法",
section 参考); each node's token is one temperature-T draw from the target
(Gumbel-max, noise from Philox4x32-10 keyed by seed, sequence, position and
vocabulary index), the walk accepts the first child that holds it, and the
output distribution is the target's ("lossless": kuma.akvtc.cn summary,
introduction).  Pinned here by:

* the generator's published known-answer vectors;
* a chi-squared test of the Gumbel-max draw against softmax(l / T);
* the acceptance probabilities of a node with several candidates, against the
  closed form p(x_1), p(x_2), ... and against Leviathan et al.'s rule carried
  out step by step (accept with p'(x), remove x on a rejection);
* T -> 0 giving the greedy step;
* brute force: the stream emitted by stochastic verification steps over
  planted trees equals autoregressive sampling with the same noise;
* mutations (noise keyed by node instead of position, or shared by every
  position) that break one of these.
"""

import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import OracleModel, oracle_prefill, oracle_verify, top2_margin
from oracle import sampling as SM
from oracle.model import causal_logits

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _chi2_crit(dof, alpha=1e-3):
    """Upper alpha quantile of chi-squared (Wilson-Hilferty), accurate to a few percent for dof >= 3."""
    z = {1e-3: 3.0902, 1e-2: 2.3263}[alpha]
    return dof * (1 - 2 / (9 * dof) + z * math.sqrt(2 / (9 * dof))) ** 3


def _chi2(counts, probs, min_expected=5.0):
    """Chi-squared statistic and degrees of freedom, pooling cells with small expected counts."""
    n = counts.sum()
    exp = probs * n
    big = exp >= min_expected
    obs = list(counts[big]) + [counts[~big].sum()]
    ex = list(exp[big]) + [exp[~big].sum()]
    obs, ex = np.array(obs, float), np.array(ex, float)
    keep = ex > 0
    return float(np.sum((obs[keep] - ex[keep]) ** 2 / ex[keep])), int(keep.sum() - 1)


@pytest.fixture(scope="module")
def tiny():
    return OracleModel(synth.TINY, synth.weights_to_host(synth.model_weights(synth.TINY, seed=0)))


def test_philox_known_answers():
    kat = json.load(open(os.path.join(GOLD, "philox4x32_10_kat.json")))
    for v in kat["vectors"]:
        ctr = [np.array([int(x, 16)], np.uint64) for x in v["ctr"]]
        out = SM.philox4x32_10(ctr, [int(x, 16) for x in v["key"]])
        assert ["%08x" % int(o[0]) for o in out] == v["out"]


def test_uniforms_grid_and_moments():
    u = SM.uniforms(seed=12345, seq=3, pos=77, n=200000)
    assert np.all((u > 0) & (u < 1))
    k = u * (1 << 24)
    assert np.array_equal(k, np.round(k)) and np.all(k % 2 == 1)  # odd multiples of 2^-24
    assert abs(u.mean() - 0.5) < 4 * math.sqrt(1 / 12 / u.size)
    g = SM.gumbel_noise(12345, 3, 77, 200000)
    assert abs(g.mean() - 0.5772156649) < 4 * (math.pi / math.sqrt(6)) / math.sqrt(g.size)  # Euler-Mascheroni


def test_gumbel_max_draws_follow_softmax(tiny):
    """20000 draws (positions 0..19999 of one seed) of the root token of a tiny-model prefix at T = 0.8."""
    lg = causal_logits(tiny, synth.prefix_tokens(1024, 32))[-1]
    T, N = 0.8, 20000
    p = SM.softmax_t(lg, T)
    y = np.array([int(np.argmax(lg / T + SM.gumbel_noise(7, 0, pos, lg.size))) for pos in range(N)])
    stat, dof = _chi2(np.bincount(y, minlength=lg.size).astype(float), p)
    assert dof >= 10
    assert stat < _chi2_crit(dof), (stat, dof)


def test_several_candidates_accept_with_their_probabilities():
    """A node whose children hold tokens x1, x2, x1 (a duplicate), x3: the single-draw walk accepts child j
    with probability p(x_j) for the first holder of each token (0 for the duplicate) and emits a bonus
    otherwise; Leviathan et al.'s rule step by step gives the same distribution."""
    rng = np.random.default_rng(5)
    V = 40
    lg = rng.normal(0, 1.5, V)
    T = 1.0
    p = SM.softmax_t(lg, T)
    kids = [int(np.argsort(-p)[0]), int(np.argsort(-p)[3]), int(np.argsort(-p)[0]), int(np.argsort(-p)[9])]
    toks = [0] + kids
    parents = [-1, 0, 0, 0, 0]
    N = 30000
    walk = np.zeros(len(kids) + 1)
    seqr = np.zeros(len(kids) + 1)
    for pos in range(N):
        y = int(np.argmax(lg / T + SM.gumbel_noise(11, 0, pos, V)))
        a = [y] + [0] * len(kids)
        nodes, bonus = SM.accept_walk(toks, parents, a)
        walk[nodes[0] - 1 if nodes else len(kids)] += 1
        j, _ = SM.sequential_rejection(p, kids, rng.random(len(kids)), rng.random())
        seqr[j if j >= 0 else len(kids)] += 1
    want = np.array([p[kids[0]], p[kids[1]], 0.0, p[kids[3]], 1 - p[kids[0]] - p[kids[1]] - p[kids[3]]])
    for counts in (walk, seqr):
        assert counts[2] == 0
        sel = want > 0
        stat, dof = _chi2(counts[sel], want[sel] / want[sel].sum(), min_expected=0)
        assert stat < _chi2_crit(max(dof, 3)), (counts, want * N)


def _plant_sampled(om, seq, shape, p, stream, T, seed, sid):
    """Plant a tree: with prob p a node copies the token the target samples at its parent."""
    def fn(tokens, parents):
        r = SM.oracle_sample_verify(om, _copy(seq), tokens, parents, T, seed, sid, check_root=False)
        return r["sampled"]
    return synth.plant_tree(shape, seq.pending, p, synth.plant_draws(shape.n, om.d.vocab, stream=stream), fn)


def _copy(seq):
    import copy
    c = copy.copy(seq)
    c.k, c.v, c.tokens = list(seq.k), list(seq.v), list(seq.tokens)
    return c


def test_zero_temperature_limit_is_greedy(tiny):
    prompt = synth.prefix_tokens(1024, 48, stream=3)
    seq, lg = oracle_prefill(tiny, prompt)
    checked = 0
    for s in range(6):
        shape = synth.tree_from_widths((3, 3, 2, 2), stream=s)
        toks = synth.plant_tree(shape, seq.pending, 0.8, synth.plant_draws(shape.n, 1024, stream=s),
                                lambda t, p_: np.argmax(oracle_verify(tiny, _copy(seq), t, p_)["logits"], axis=1))
        g = oracle_verify(tiny, _copy(seq), toks, shape.parents)
        if np.min(g["margin"]) < 1e-4:
            continue
        r = SM.oracle_sample_verify(tiny, _copy(seq), toks, shape.parents, 1e-9, 99, 0)
        assert np.array_equal(r["sampled"], g["argmax"])
        assert (r["accepted_len"], r["accepted_tokens"], r["bonus"]) == (g["accepted_len"], g["accepted_tokens"],
                                                                         g["bonus"])
        checked += 1
    assert checked >= 4


def _stochastic_stream(om, prompt, n, T, seed, sid, p=0.8, verify=SM.oracle_sample_verify):
    """Tokens emitted by prefill + stochastic verification steps over planted trees."""
    seq, lg = oracle_prefill(om, prompt)
    seq.pending = SM.sampled_pending(lg[-1], T, seed, sid, len(prompt))
    out = [seq.pending]
    step = 0
    while len(out) < n:
        shape = synth.tree_from_widths((3, 2, 2, 1), stream=step) if step % 2 else synth.chain(3)
        toks = _plant_sampled(om, seq, shape, p, step, T, seed, sid)
        r = verify(om, seq, toks, shape.parents, T, seed, sid)
        out += r["accepted_tokens"] + [r["bonus"]]
        step += 1
    return out[:n], step


def test_stochastic_steps_equal_autoregressive_sampling(tiny):
    """Brute force: 40 tokens from stochastic verification steps equal autoregressive sampling (a full
    recompute per token) with the same noise, at T = 0.7 and T = 1.2, and the steps accepted drafts."""
    prompt = synth.prefix_tokens(1024, 40, stream=9)
    for T, seed in ((0.7, 1), (1.2, 2)):
        ar = SM.oracle_sample_ar(tiny, prompt, 40, T, seed, 5)
        got, steps = _stochastic_stream(tiny, prompt, 40, T, seed, 5)
        assert got == ar
        assert steps < 30


def test_mutations_are_caught(tiny):
    """Noise keyed by the node's index instead of its position, or one noise vector for every position,
    breaks one of the pins above."""
    prompt = synth.prefix_tokens(1024, 40, stream=9)
    T, seed = 0.7, 1
    ar = SM.oracle_sample_ar(tiny, prompt, 30, T, seed, 5)
    orig = SM.perturbed_scores

    def by_node(logits, temperature, seed_, seq_, pos):
        return orig(logits, temperature, seed_, seq_, np.arange(len(pos)))
    SM.perturbed_scores = by_node
    try:
        got, _ = _stochastic_stream(tiny, prompt, 30, T, seed, 5)
    finally:
        SM.perturbed_scores = orig
    assert got != ar
    # one noise vector for all positions: consecutive draws are no longer independent
    lg = np.zeros(8)
    g_fixed = SM.gumbel_noise(3, 0, 0, 8)
    ys = [int(np.argmax(lg + g_fixed)) for _ in range(200)]
    stat, dof = _chi2(np.bincount(ys, minlength=8).astype(float), np.full(8, 1 / 8))
    assert stat > _chi2_crit(dof)
