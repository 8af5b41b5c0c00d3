"""GPU parity: the library (through its C ABI) against the float64 oracle.

Compared element by element on the same seeded inputs: logits at every tree
node (within 1e-4 for fp32 models, 2e-2 for bf16), the argmax at every node
whose margin leaves no doubt, the step's outputs (accepted length, tokens,
bonus), the compacted K/V cache and the sequence state.  Shapes span several
GEMM and attention tiles, ragged tails, root-only trees, chains, 128-node
trees and batches of sequences with different prefix lengths.
"""

import os

import numpy as np
import pytest

import synth
from oracle import oracle_verify, top2_margin
from gpu_common import (DECISIVE, TOL, decided_case, decided_tree, decisive_nodes, decisive_prefix, gpu_kv,
                        kv_close, make_pair)

pytestmark = pytest.mark.gpu


def _check_step(eng, om, seq_id, seq, shape, tokens, dtype, check_kv=True):
    """Score (logits), then verify; compare everything with the oracle."""
    n = shape.n
    tol = TOL[dtype]
    amax, t1, t2, _ = eng.score([seq_id], [(tokens, shape.parents)], flags=2)
    logits = eng.debug_logits(n)
    P = seq.length
    r = oracle_verify(om, seq, tokens, shape.parents)
    err = float(np.max(np.abs(logits - r["logits"])))
    assert err <= tol, "max |logit error| %.3g > %.3g" % (err, tol)
    # argmax: exact wherever the oracle's margin exceeds twice the observed error
    thr = min(DECISIVE, max(2.5 * err, 1e-6))
    sure = r["margin"] > thr
    assert np.array_equal(amax[sure], r["argmax"][sure])
    np.testing.assert_allclose(t1, r["logits"].max(axis=1), atol=tol)
    a, acc_tok, bonus = eng.verify(seq_id, tokens, shape.parents)
    decided = bool(np.all(r["margin"][decisive_nodes(r, shape.parents)] > thr))
    if decided:
        assert a == r["accepted_len"]
        assert acc_tok == r["accepted_tokens"]
        assert bonus == r["bonus"]
        ln, pend = eng.seq_len(seq_id)
        assert ln == P + 1 + a and pend == bonus
        if check_kv:
            gk, gv = gpu_kv(eng, seq_id, ln)
            for l in range(om.d.n_layers):
                kt = 1e-5 if dtype == "f32" else 2e-2
                assert kv_close(gk[l], seq.k[l], kt) <= kt, "layer %d K" % l
                assert kv_close(gv[l], seq.v[l], kt) <= kt, "layer %d V" % l
    return decided, err


def test_tiny_fp32_config():
    """fp32 tiny decoder: prefix 64, 8 drafts at depth 4 (widths 2,4,1,1), planted p = 0.8."""
    eng, om = make_pair(synth.TINY, max_batch=1, max_seq=512, max_nodes=16)
    prefix, seq = decisive_prefix(om, 64, min_margin=1e-3)
    pend = eng.prefill(0, prefix)
    assert pend == seq.pending
    gk, gv = gpu_kv(eng, 0, 64)
    assert kv_close(gk[0], seq.k[0], 1e-5) <= 1e-5
    for step in range(4):
        shape = synth.tiny_tree()
        toks, _ = decided_tree(om, seq, shape, 0.8, stream=step, min_margin=1e-3)
        assert toks is not None
        d, err = _check_step(eng, om, 0, seq, shape, toks, "f32")
        assert d, "step %d was not decided" % step
        assert err < 1e-4


# (model, prefix length, tree, prefix stream, planting stream): the streams are the
# first ones from which gpu_common.decided_case finds a decided step (the search
# runs again in each test and ends at its first candidate)
BF16_CASES = [
    ("mini", 37, "root", 37, 37),
    ("mini", 37, "chain2", 37, 37),
    ("mini", 300, "tiny", 300, 300),
    ("mini", 1000, "tree60", 1000, 3000),
    ("mini", 129, "tree127", 133, 133),
    ("small", 700, "tree60", 700, 2700),
    ("small", 64, "chain8", 64, 64),
    ("small", 500, "tree80", 500, 500),  # 81 tokens: 96-token GEMM tiles
    ("small", 400, "tree72", 400, 400),  # 73 tokens: 80-token GEMM tiles
    ("mini", 200, "tree72", 200, 200),
]


def _shape(kind):
    if kind == "root":
        return synth.chain(0)
    if kind == "chain2":
        return synth.chain(2)
    if kind == "chain8":
        return synth.chain(8)
    if kind == "tiny":
        return synth.tiny_tree()
    if kind == "tree60":
        return synth.tree_from_widths(synth.TREE60_WIDTHS, stream=4)
    if kind == "tree127":
        return synth.tree_from_widths((10, 12, 16, 20, 20, 20, 16, 13), stream=5)
    if kind == "tree80":
        return synth.tree_from_widths(synth.SWEEP_WIDTHS[80], stream=6)
    if kind == "tree72":
        return synth.tree_from_widths((10, 10, 10, 10, 10, 8, 8, 6), stream=7)
    raise KeyError(kind)


_pairs = {}


def _pair(which):
    if which not in _pairs:
        dims = synth.MINI_BF16 if which == "mini" else synth.SMALL_BF16
        _pairs[which] = make_pair(dims, max_batch=4, max_seq=1400, max_nodes=128)
    return _pairs[which]


@pytest.mark.parametrize("which,P,kind,s_prefix,s_plant", BF16_CASES)
def test_bf16_verify_parity(which, P, kind, s_prefix, s_plant):
    eng, om = _pair(which)
    shape = _shape(kind)
    if kind == "tree72":
        assert "qkv bn80 " in eng.info(1, shape.n, P)
    prefix, seq, toks = decided_case(om, P, shape, 0.8, stream0=s_prefix, plant0=s_plant)
    pend = eng.prefill(0, prefix)
    assert pend == seq.pending
    gk, gv = gpu_kv(eng, 0, P)
    for l in range(om.d.n_layers):
        assert kv_close(gk[l], seq.k[l], 2e-2) <= 2e-2
    decided, _ = _check_step(eng, om, 0, seq, shape, toks, "bf16")
    assert decided, "the step was not decided: outputs and K/V went unchecked"


def test_bf16_batch_of_sequences():
    """Three sequences with different prefix lengths and trees in one batched step."""
    eng, om = _pair("mini")
    Ps = [45, 410, 130]
    shapes = [synth.tree_from_widths((3, 3, 2), stream=1), synth.tiny_tree(), synth.chain(5)]
    seqs, trees = [], []
    for i, (P, sh) in enumerate(zip(Ps, shapes)):
        prefix, seq, toks = decided_case(om, P, sh, 0.8, stream0=(101, 112, 120)[i])
        assert eng.prefill(i, prefix) == seq.pending
        seqs.append(seq)
        trees.append((toks, sh.parents))
    amax, t1, t2, off = eng.score([0, 1, 2], trees, flags=2)
    logits = eng.debug_logits(int(off[-1]))
    acc_len, acc_nodes, acc_tok, bonus = eng.verify_batch([0, 1, 2], trees)
    for i, (seq, (toks, par)) in enumerate(zip(seqs, trees)):
        r = oracle_verify(om, seq, toks, par)
        lg = logits[off[i]:off[i + 1]]
        err = float(np.max(np.abs(lg - r["logits"])))
        assert err <= TOL["bf16"]
        thr = min(DECISIVE, max(2.5 * err, 1e-6))
        assert np.all(r["margin"][decisive_nodes(r, par)] > thr), "sequence %d was not decided" % i
        assert acc_len[i] == r["accepted_len"]
        assert list(acc_nodes[i, :acc_len[i]]) == r["accepted_nodes"]
        assert list(acc_tok[i, :acc_len[i]]) == r["accepted_tokens"]
        assert bonus[i] == r["bonus"]
        ln, _ = eng.seq_len(i)
        gk, gv = gpu_kv(eng, i, ln)
        for l in range(om.d.n_layers):
            assert kv_close(gk[l], seq.k[l], 2e-2) <= 2e-2
            assert kv_close(gv[l], seq.v[l], 2e-2) <= 2e-2


WIDE_STREAMS = (7, 7)  # (prefix, planting) streams of the decided step on the 8B-layer-shape model


@pytest.mark.parametrize("tune", ["sk=0", "", "sk=1"])
def test_wide_bf16_full_size_tiles(tune, monkeypatch):
    """8B layer shapes (d 4096, 32/8 heads, ffn 14336), 2 layers, vocab 16384: full-size tiles and splits;
    whole tiles everywhere with sk=0, the LM head on stream-K by default (its 128 tiles on 296 CTAs: equal
    k-block shares, partial sums handed over), gate/up too with sk=1."""
    monkeypatch.setenv("SPEC_TUNE", tune)
    eng, om = make_pair(synth.WIDE_BF16, max_batch=1, max_seq=512, max_nodes=64)
    plan = eng.info(1, 61, 200)
    assert ("stream-K" in plan.split("; lm ")[1]) == (tune != "sk=0")
    assert ("stream-K" in plan.split("; gate_up ")[1].split(";")[0]) == (tune == "sk=1")
    shape = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=0)
    prefix, seq, toks = decided_case(om, 200, shape, 0.8, stream0=WIDE_STREAMS[0], plant0=WIDE_STREAMS[1])
    assert eng.prefill(0, prefix) == seq.pending
    decided, _ = _check_step(eng, om, 0, seq, shape, toks, "bf16")
    assert decided


def _check_batch(eng, om, ids, seqs, trees):
    """Score and verify a batch; compare logits, outputs and the compacted K/V per sequence."""
    amax, t1, t2, off = eng.score(ids, trees, flags=2)
    logits = eng.debug_logits(int(off[-1]))
    acc_len, acc_nodes, acc_tok, bonus = eng.verify_batch(ids, trees)
    decided = 0
    for i, (seq, (toks, par)) in enumerate(zip(seqs, trees)):
        r = oracle_verify(om, seq, toks, par)
        lg = logits[off[i]:off[i + 1]]
        err = float(np.max(np.abs(lg - r["logits"])))
        assert err <= TOL["bf16"], "sequence %d: max |logit error| %.3g" % (i, err)
        thr = min(DECISIVE, max(2.5 * err, 1e-6))
        sure = r["margin"] > thr
        assert np.array_equal(amax[off[i]:off[i + 1]][sure], r["argmax"][sure])
        if np.all(r["margin"][decisive_nodes(r, par)] > thr):
            decided += 1
            assert acc_len[i] == r["accepted_len"]
            assert list(acc_nodes[i, :acc_len[i]]) == r["accepted_nodes"]
            assert list(acc_tok[i, :acc_len[i]]) == r["accepted_tokens"]
            assert bonus[i] == r["bonus"]
            ln, _ = eng.seq_len(ids[i])
            gk, gv = gpu_kv(eng, ids[i], ln)
            for l in range(om.d.n_layers):
                assert kv_close(gk[l], seq.k[l], 2e-2) <= 2e-2
                assert kv_close(gv[l], seq.v[l], 2e-2) <= 2e-2
    return decided


# per sequence: (prefix stream, planting stream) of a decided step
LARGE_STREAMS = [(302, 3302), (308, 308), (320, 320), (322, 322), (328, 1328), (335, 335), (350, 350), (350, 350),
                 (360, 360), (364, 364), (370, 370), (377, 377), (384, 1384), (392, 3392), (399, 2399), (405, 405),
                 (412, 412), (419, 419), (427, 427), (433, 1433)]


def test_bf16_large_batch_unchunked():
    """20 sequences (prefixes 150-600) x 61-node trees = 1220 tokens: 128-token GEMM tiles, several token
    tiles, and attention without key chunks (one CTA walks every 128-key block with the online softmax)."""
    eng, om = make_pair(synth.SMALL_BF16, max_batch=20, max_seq=1024, max_nodes=64)
    B = 20
    Ps = np.random.default_rng(4).integers(150, 601, size=B)
    seqs, trees = [], []
    for i in range(B):
        sh = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=i)
        prefix, seq, toks = decided_case(om, int(Ps[i]), sh, 0.8, stream0=LARGE_STREAMS[i][0],
                                         plant0=LARGE_STREAMS[i][1])
        assert eng.prefill(i, prefix) == seq.pending
        trees.append((toks, sh.parents))
        seqs.append(seq)
    assert "chunks 1 x" in eng.info(B, 61, int(Ps.max()))
    assert _check_batch(eng, om, list(range(B)), seqs, trees) == B


def _engine_tuned(dims, tune, **kw):
    old = os.environ.get("SPEC_TUNE")
    os.environ["SPEC_TUNE"] = tune
    try:
        return make_pair(dims, **kw)
    finally:
        if old is None:
            del os.environ["SPEC_TUNE"]
        else:
            os.environ["SPEC_TUNE"] = old


@pytest.mark.parametrize("tune", ["chunks=2", "chunks=1", "chunks=2,rescale=0", "chunks=1,rescale=0", "chunks=4,dsmem=0",
                                  "chunks=4"])
def test_bf16_multiblock_attention(tune):
    """Prefix 700 + 61 nodes = 6 key blocks per (sequence, kv head) in 4, 2 or 1 chunks; slack 0 makes every
    growth of the running max rescale the accumulated output; chunks merge through distributed shared memory
    (a cluster of chunk CTAs, idle ones included for the shorter sequence) or, with dsmem=0, through global
    memory."""
    eng, om = _engine_tuned(synth.MINI_BF16, tune, max_batch=2, max_seq=1024, max_nodes=64)
    seqs, trees = [], []
    for i, P in enumerate((700, 530)):
        sh = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=3 + i)
        prefix, seq, toks = decided_case(om, P, sh, 0.8, stream0=(501, 512)[i], plant0=(1501, 512)[i])
        assert eng.prefill(i, prefix) == seq.pending
        trees.append((toks, sh.parents))
        seqs.append(seq)
    assert _check_batch(eng, om, [0, 1], seqs, trees) == 2


@pytest.mark.parametrize("tune", ["chunks=4,dsmem=0", "chunks=4"])
def test_bf16_chunk_merge_mixed_lengths(tune):
    """A batch whose sequences split into different chunk counts: prefix 90 + 61 nodes fits one key chunk (its
    rows are written by its CTA directly), prefix 700 + 61 takes four whose partials are merged through global
    memory (dsmem=0) or a cluster; the longer sequence comes second in the batch and first in the attention's
    work order."""
    eng, om = _engine_tuned(synth.MINI_BF16, tune, max_batch=2, max_seq=1024, max_nodes=64)
    assert ("(global merge)" if "dsmem=0" in tune else "(cluster merge)") in eng.info(2, 61, 700)
    seqs, trees = [], []
    for i, P in enumerate((90, 700)):
        sh = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=7 + i)
        prefix, seq, toks = decided_case(om, P, sh, 0.8, stream0=(601, 501)[i])
        assert eng.prefill(i, prefix) == seq.pending
        trees.append((toks, sh.parents))
        seqs.append(seq)
    assert _check_batch(eng, om, [0, 1], seqs, trees) == 2
