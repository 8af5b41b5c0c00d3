"""GPU behaviour of the library beyond single-step parity: losslessness over
many steps, error paths that must leave the cache untouched, asynchronous
(device-output) steps, rollback, determinism and ancestor isolation."""

import numpy as np
import pytest

import synth
from oracle import oracle_greedy_ar, oracle_prefill, top2_margin, causal_logits
from speculative_decoding_06_b200 import spec as S
from gpu_common import DECIDED_SMALL, TOL, decisive_prefix, make_pair, planted_tree

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    return make_pair(synth.TINY, max_batch=2, max_seq=600, max_nodes=64)


@pytest.fixture(scope="module")
def mini():
    return make_pair(synth.MINI_BF16, max_batch=3, max_seq=700, max_nodes=128)


def _tree_for(step, vocab):
    kind = step % 3
    if kind == 0:
        return synth.tiny_tree()
    if kind == 1:
        return synth.tree_from_widths((4, 4, 3, 2, 2), stream=step)
    return synth.chain(1 + step % 6)


def test_lossless_decode_fp32(tiny):
    """Repeated GPU verify steps emit exactly the oracle's brute-force greedy tokens (>= 200)."""
    eng, om = tiny
    prompt = synth.prefix_tokens(om.d.vocab, 64, seed=1)
    n = 200
    greedy = oracle_greedy_ar(om, prompt, n + 1)
    # the greedy stream must be decisive at fp32 tolerance
    pend = eng.prefill(0, prompt)
    emitted = [pend]
    seq, _ = oracle_prefill(om, prompt)
    step = 0
    rng = np.random.default_rng(3)
    while len(emitted) < n + 1:
        shape = _tree_for(step, om.d.vocab)
        # plant from the greedy stream itself (no GPU-derived inputs): a node copies
        # the true continuation along the lowest-index path with prob 0.8
        toks = np.zeros(shape.n, np.int32)
        toks[0] = emitted[-1]
        pos = len(emitted)
        first_child = {}
        for i in range(1, shape.n):
            first_child.setdefault(int(shape.parents[i]), i)
        main = {0}
        for i in range(1, shape.n):
            par = int(shape.parents[i])
            on_main = par in main and first_child[par] == i
            if on_main:
                main.add(i)
            lvl = int(shape.level[i])
            want = greedy[pos + lvl - 1] if pos + lvl - 1 < len(greedy) else 0
            toks[i] = want if (on_main and rng.random() < 0.8) else rng.integers(0, om.d.vocab)
        a, acc, bonus = eng.verify(0, toks, shape.parents)
        emitted += acc + [bonus]
        step += 1
    m = min(len(emitted), len(greedy))
    assert emitted[:m] == greedy[:m]
    assert step < n  # speculation accepted something


def _greedy_run(om, prompt, n, min_margin):
    """Greedy continuation of `prompt` by the oracle and the number of leading tokens whose margin exceeds
    min_margin (every one of them is decided)."""
    seqt = list(prompt)
    greedy, margins = [], []
    for _ in range(n + 1):
        lg = causal_logits(om, seqt)[-1]
        greedy.append(int(np.argmax(lg)))
        margins.append(float(top2_margin(lg)))
        seqt.append(greedy[-1])
    return greedy, next((i for i, mg in enumerate(margins) if mg <= min_margin), n + 1)


def test_lossless_decode_bf16_until_near_tie(mini):
    """bf16: the GPU stream equals greedy decoding for at least 24 tokens, every one of them decided.

    The prompt is the first seeded one whose greedy continuation keeps the oracle's top-1 / top-2 margin above
    DECIDED_SMALL for 24 tokens (with vocabulary 2048 a margin above 0.05 holds for ~65 % of tokens, so runs of
    that length do not occur at 0.05); the search starts at the first such stream, 27."""
    eng, om = mini
    n, need = 40, 24
    for stream in range(27, 200):
        prompt = synth.prefix_tokens(om.d.vocab, 48, seed=1, stream=stream)
        greedy, safe = _greedy_run(om, prompt, n, DECIDED_SMALL)
        if safe >= need:
            break
    assert safe >= need, "no seeded prompt with a decided run of %d tokens" % need
    pend = eng.prefill(1, prompt)
    emitted = [pend]
    step = 0
    while len(emitted) < safe:
        pos = len(emitted)
        shape = synth.chain(4)
        toks = [emitted[-1]] + [greedy[pos + j] if pos + j < len(greedy) else 0 for j in range(4)]
        if step % 2:
            toks[3] = (toks[3] + 1) % om.d.vocab
        a, acc, bonus = eng.verify(1, toks, shape.parents)
        emitted += acc + [bonus]
        step += 1
    m = min(len(emitted), safe)
    assert m >= need
    assert emitted[:m] == greedy[:m]


def test_errors_leave_state_unchanged(mini):
    eng, om = mini
    prompt = synth.prefix_tokens(om.d.vocab, 40, stream=11)
    pend = eng.prefill(0, prompt)
    ln0 = eng.seq_len(0)
    with pytest.raises(S.SpecError) as e:
        eng.verify(0, [pend, 1, 2], [-1, 0, 2])
    assert e.value.code == S.SPEC_ERR_TREE
    with pytest.raises(S.SpecError) as e:
        eng.verify(0, [(pend + 1) % om.d.vocab, 1], [-1, 0])
    assert e.value.code == S.SPEC_ERR_ROOT
    with pytest.raises(S.SpecError) as e:
        eng.verify(0, [pend, om.d.vocab], [-1, 0])
    assert e.value.code == S.SPEC_ERR_TOKEN
    with pytest.raises(S.SpecError) as e:
        eng.verify(2, [pend], [-1])  # never prefilled
    assert e.value.code == S.SPEC_ERR_STATE
    with pytest.raises(S.SpecError) as e:
        eng.verify(5, [pend], [-1])  # no such sequence
    assert e.value.code == S.SPEC_ERR_ARG
    with pytest.raises(S.SpecError) as e:
        eng.verify(0, [pend] * 129, [-1] + list(range(128)))
    assert e.value.code == S.SPEC_ERR_CAPACITY
    assert eng.seq_len(0) == ln0
    a, acc, bonus = eng.verify(0, [pend], [-1])
    assert a == 0 and eng.seq_len(0) == (ln0[0] + 1, bonus)


def test_device_outputs_truncate_and_determinism(mini):
    """Async steps then sync give the sync result; rollback replays bit-identically."""
    import torch
    eng, om = mini
    prompt = synth.prefix_tokens(om.d.vocab, 200, stream=12)
    pend = eng.prefill(0, prompt)
    shape = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=2)
    rng = np.random.default_rng(1)
    toks = rng.integers(0, om.d.vocab, size=shape.n).astype(np.int32)
    toks[0] = pend
    _, _, _, _ = eng.score([0], [(toks, shape.parents)], flags=2)
    l1 = eng.debug_logits(shape.n).copy()
    r1 = eng.verify_batch([0], [(toks, shape.parents)])
    eng.truncate(0, 200)
    assert eng.seq_len(0) == (200, pend)
    _, _, _, _ = eng.score([0], [(toks, shape.parents)], flags=2 | S.SPEC_NO_GRAPH)
    l2 = eng.debug_logits(shape.n).copy()
    assert np.array_equal(l1, l2)  # graph replay and direct launches agree bit for bit
    from speculative_decoding_06_b200.engine import pack_trees
    tk, pr, off = pack_trees([(toks, shape.parents)])
    ids = np.array([0], np.int32)
    out = [torch.zeros(1, dtype=torch.int32, device="cuda"), None, None, torch.zeros(1, dtype=torch.int32, device="cuda")]
    eng.verify_batch_device(ids, tk, pr, off, outputs=tuple(out))
    eng.sync()
    assert int(out[0].item()) == r1[0][0] and int(out[3].item()) == r1[3][0]
    assert eng.seq_len(0) == (200 + 1 + r1[0][0], r1[3][0])


def test_non_ancestor_tokens_leave_node_logits_bitwise(mini):
    eng, om = mini
    prompt = synth.prefix_tokens(om.d.vocab, 90, stream=13)
    pend = eng.prefill(0, prompt)
    shape = synth.tree_from_widths((3, 3, 2), stream=3)
    rng = np.random.default_rng(2)
    toks = rng.integers(0, om.d.vocab, size=shape.n).astype(np.int32)
    toks[0] = pend
    eng.score([0], [(toks, shape.parents)], flags=2)
    base = eng.debug_logits(shape.n).copy()
    from oracle import tree_meta
    _, anc = tree_meta(shape.parents)
    for j in range(1, shape.n):
        t2 = toks.copy()
        t2[j] = (t2[j] + 5) % om.d.vocab
        eng.score([0], [(t2, shape.parents)], flags=2)
        pert = eng.debug_logits(shape.n)
        for i in range(shape.n):
            if j not in anc[i]:
                assert np.array_equal(pert[i], base[i]), (i, j)


def test_fp16_range_overflow_fails_the_step(mini):
    """q, K and V live in fp16: a key beyond +-65504 fails the step with SPEC_ERR_RANGE and leaves the
    sequence as it was; with the weights restored the same step succeeds."""
    eng, om = mini
    prompt = synth.prefix_tokens(om.d.vocab, 60, stream=21)
    pend = eng.prefill(2, prompt)
    before = eng.seq_len(2)
    wk = eng._weights["layers"][1]["wk"]
    saved = wk.clone()
    wk.mul_(1e7)  # |k| ~ 1e5 and beyond
    try:
        with pytest.raises(S.SpecError) as e:
            eng.verify(2, [pend, 3, 4], [-1, 0, 1])
        assert e.value.code == S.SPEC_ERR_RANGE
        assert eng.seq_len(2) == before
    finally:
        wk.copy_(saved)
    a, acc, bonus = eng.verify(2, [pend, 3, 4], [-1, 0, 1])
    assert eng.seq_len(2) == (before[0] + 1 + a, bonus)
