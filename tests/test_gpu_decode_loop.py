"""The closed draft-and-verify loop through the library (greedy EAGLE-3 decoding).

* Prefill features (spec_prefill_features) against the float64 oracle's
  residual streams after the feature layers, within the bf16 feature tolerance.
* Losslessness ("EAGLE-3投机解码：树验证器方法", section 验证-接受语义: the
  verified output equals what the target alone would produce): the tokens the
  loop emits (draft tree -> verification with features -> draft prefix
  extension) equal brute-force greedy decoding by the oracle up to the first
  position whose top-2 margin is within the bf16 tolerance.
* The draft prefix stays one row behind the target sequence.
"""

import numpy as np
import pytest

import synth
from oracle import OracleModel, causal_logits, top2_margin
from oracle.model import causal_features

pytestmark = pytest.mark.gpu

TAPS = (1, 1, 2)


@pytest.fixture(scope="module")
def loop_pair():
    from speculative_decoding_06_b200.engine import SpecEngine
    d = synth.SMALL_BF16
    w = synth.model_weights(d, seed=0, device="cuda")
    dw = synth.draft_head_weights(d, seed=6, device="cuda")
    eng = SpecEngine(d, w, max_batch=1, max_seq=512, max_nodes=64, draft=dw, feature_layers=TAPS)
    yield eng, OracleModel(d, synth.weights_to_host(w))
    eng.close()


def test_prefill_features_match_oracle(loop_pair):
    eng, om = loop_pair
    prompt = synth.prefix_tokens(om.d.vocab, 150, seed=3)  # three chunks of max_nodes rows
    pend, feats = eng.prefill_features(0, prompt)
    ref = causal_features(om, prompt, TAPS)
    g = feats.float().cpu().numpy()
    rms = np.sqrt(np.mean(ref ** 2, axis=2, keepdims=True))
    err = np.abs(g - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-2 * rms), float(np.max(err))
    assert pend == int(np.argmax(causal_logits(om, prompt)[-1])) or top2_margin(causal_logits(om, prompt)[-1]) <= 0.05


def _greedy(om, prompt, n):
    seqt = list(prompt)
    greedy, margins = [], []
    for _ in range(n + 1):
        lg = causal_logits(om, seqt)[-1]
        greedy.append(int(np.argmax(lg)))
        margins.append(float(top2_margin(lg)))
        seqt.append(greedy[-1])
    return greedy, next((i for i, mg in enumerate(margins) if mg <= 0.05), n + 1)


def test_speculative_decode_is_lossless(loop_pair):
    eng, om = loop_pair
    n = 24
    # a prompt whose greedy continuation stays clear of near-ties for a while
    for stream in range(4, 200):
        prompt = synth.prefix_tokens(om.d.vocab, 40, seed=1, stream=stream)
        greedy, safe = _greedy(om, prompt, n)
        if safe >= 12:
            break
    assert safe >= 12
    emitted, accepted = eng.speculative_decode(0, prompt, n, steps=3, topk=4, total=12)
    m = min(len(emitted), safe)
    assert m >= 1
    assert emitted[:m] == greedy[:m]
    ln, pending = eng.seq_len(0)
    assert ln == len(prompt) + len(emitted) - 1 and pending == emitted[-1]
    assert eng.draft_len(0) == ln - 1
    print("steps %d, accepted per step %s, compared %d tokens" % (len(accepted), accepted, m))


def test_speculative_decode_batch_is_lossless():
    """Two sequences decoded together: each equals its own greedy continuation."""
    from speculative_decoding_06_b200.engine import SpecEngine
    d = synth.SMALL_BF16
    w = synth.model_weights(d, seed=0, device="cuda")
    dw = synth.draft_head_weights(d, seed=6, device="cuda")
    eng = SpecEngine(d, w, max_batch=2, max_seq=512, max_nodes=64, draft=dw, feature_layers=TAPS)
    om = OracleModel(d, synth.weights_to_host(w))
    try:
        n = 16
        prompts, greedys, safes = [], [], []
        stream = 40
        while len(prompts) < 2 and stream < 400:
            prompt = synth.prefix_tokens(om.d.vocab, 30 + 9 * len(prompts), seed=2, stream=stream)
            greedy, safe = _greedy(om, prompt, n)
            if safe >= 8:
                prompts.append(prompt)
                greedys.append(greedy)
                safes.append(safe)
            stream += 1
        assert len(prompts) == 2
        emitted, accepted = eng.speculative_decode_batch([1, 0], prompts, n, steps=2, topk=4, total=8)
        for e, g, safe in zip(emitted, greedys, safes):
            m = min(len(e), safe)
            assert e[:m] == g[:m]
        for s, e in zip([1, 0], emitted):
            ln, pending = eng.seq_len(s)
            assert pending == e[-1] and eng.draft_len(s) == ln - 1
    finally:
        eng.close()
