"""Draft-head features from the verification step (SPEC_FEATURES) against the oracle.

EAGLE-3's draft head takes the target's low-, mid- and high-level hidden
states of every position, recorded during verification ("EAGLE-3: Scaling up
Inference Acceleration of Large Language Models via Training-Time Test",
draft-stage description).  With feature layers (j_low, j_mid, j_high) the step
writes, for each batch entry, the residual stream after those many decoder
layers at the root and at each accepted node, in path order, as bf16.

Each row is compared with the float64 oracle's features of the node the GPU
step accepted (so a near-tie that changes the accepted path does not matter
here; acceptance itself is checked by the parity tests).  Tolerance: the bf16
rounding of the output (2^-8 relative) plus the step's compute error, 1e-2 of
the row's RMS for bf16 models and 1e-4 for fp32 models.  Rows past
accepted_len must be left as they were.
"""

import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import oracle_prefill
from oracle.model import oracle_tree_features
from speculative_decoding_06_b200 import spec as S
from gpu_common import decisive_prefix, make_pair, planted_tree

pytestmark = pytest.mark.gpu

SMALL4 = dataclasses.replace(synth.SMALL_BF16, n_layers=4)


def _pair(dims, taps, max_batch):
    return make_pair(dims, max_batch=max_batch, max_seq=1024, max_nodes=64, feature_layers=taps)


def _check(eng, om, taps, B, rel_compute, shapes, stream0):
    seqs, trees = [], []
    for i in range(B):
        prefix, seq = decisive_prefix(om, 90 + 37 * i, stream0=stream0 + 11 * i)
        assert eng.prefill(i, prefix) == seq.pending
        sh = shapes[i]
        trees.append((planted_tree(om, seq, sh, 0.8, stream=stream0 + i), sh.parents))
        seqs.append(seq)
    buf = eng.feature_buffer()
    buf.fill_(7.0)
    acc_len, acc_nodes, _, _, feats = eng.verify_batch(list(range(B)), trees, features=True)
    torch.cuda.synchronize()
    g = feats.float().cpu().numpy()
    for b, (seq, (toks, par)) in enumerate(zip(seqs, trees)):
        _, _, ref_all = oracle_tree_features(om, seq, toks, par, taps)
        a = int(acc_len[b])
        path = [0] + [int(x) for x in acc_nodes[b, :a]]
        for k, node in enumerate(path):
            ref = ref_all[node]
            rms = np.sqrt(np.mean(ref ** 2, axis=1, keepdims=True))
            err = np.abs(g[b, k] - ref)
            bound = 2.0 ** -8 * np.abs(ref) + rel_compute * rms
            assert np.all(err <= bound), "entry %d path row %d: worst excess %.3g" % (b, k, float(np.max(err - bound)))
        assert np.all(g[b, a + 1:] == 7.0), "rows past accepted_len were written"
    return acc_len


def test_features_bf16_four_layers():
    taps = (2, 1, 4)  # out of order: each slot keeps its own layer
    eng, om = _pair(SMALL4, taps, max_batch=3)
    try:
        shapes = [synth.tree_from_widths(synth.TREE60_WIDTHS, stream=0), synth.chain(5), synth.tiny_tree()]
        acc = _check(eng, om, taps, 3, 1e-2, shapes, stream0=500)
        assert int(np.max(acc)) >= 2  # planted trees accept several nodes
    finally:
        eng.close()


def test_features_fp32():
    taps = (1, 2, 2)
    eng, om = _pair(synth.TINY, taps, max_batch=2)
    try:
        shapes = [synth.tree_from_widths((4, 4, 3, 2, 2), stream=1), synth.chain(4)]
        _check(eng, om, taps, 2, 1e-4, shapes, stream0=700)
    finally:
        eng.close()


def test_features_need_feature_layers_and_a_buffer():
    eng, om = make_pair(synth.TINY, max_batch=1, max_seq=256, max_nodes=16)
    try:
        prompt = synth.prefix_tokens(om.d.vocab, 16, seed=2)
        pend = eng.prefill(0, prompt)
        sh = synth.chain(2)
        toks = np.array([pend, 1, 2], np.int32)
        with pytest.raises(S.SpecError) as e:
            eng.verify_batch([0], [(toks, sh.parents)], flags=S.SPEC_FEATURES)
        assert e.value.code == S.SPEC_ERR_STATE
        with pytest.raises(S.SpecError):
            eng.feature_buffer()  # spec_set_feature_out refuses: no feature layers
    finally:
        eng.close()
