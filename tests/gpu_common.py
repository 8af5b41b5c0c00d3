"""Shared set-up for the GPU parity tests: one seeded model, the library
engine on the GPU and the float64 oracle on the CPU, fed the same bits."""

from __future__ import annotations

import copy

import numpy as np
import torch

import synth
from oracle import OracleModel, argmax_fn_for_planting, oracle_prefill, oracle_verify, top2_margin

# logit tolerance stated for the verification step: 2e-2 absolute for bf16
# models, 1e-4 for fp32 models
TOL = {"bf16": 2e-2, "f32": 1e-4}
# the step's outputs must be identical wherever the oracle's top-1 / top-2
# margin exceeds this on every node that decides them
DECISIVE = 0.05
# small test models (vocab <= 16384, d <= 1024) have top-1 / top-2 gaps of about
# 0.1, so a 61-node tree rarely has all its deciding margins above 0.05; their
# parity cases are chosen with every deciding margin above this instead, which
# is still 10x the logit error those models show (~1e-3) and above the tests'
# own threshold min(0.05, 2.5 x observed error) while that error stays below 8e-3
DECIDED_SMALL = 0.02


def gpu_available() -> bool:
    return torch.cuda.is_available()


def make_pair(dims, max_batch=1, max_seq=1024, max_nodes=128, seed=0, device_gen=False, **engine_kw):
    """Engine (GPU) and oracle (CPU) over the same seeded weights."""
    from speculative_decoding_06_b200.engine import SpecEngine
    if device_gen:
        wdev = synth.model_weights(dims, seed=seed, device="cuda")
        host = synth.weights_to_host(wdev)
    else:
        wcpu = synth.model_weights(dims, seed=seed, device="cpu")
        host = synth.weights_to_host(wcpu)
        wdev = {k: v.cuda() for k, v in wcpu.items() if k != "layers"}
        wdev["layers"] = [{k: v.cuda() for k, v in lw.items()} for lw in wcpu["layers"]]
    eng = SpecEngine(dims, wdev, max_batch=max_batch, max_seq=max_seq, max_nodes=max_nodes, **engine_kw)
    return eng, OracleModel(dims, host)


def decisive_prefix(om, length, stream0=0, min_margin=DECISIVE, tries=20):
    """A seeded prefix whose last-position margin is decisive, with its oracle state."""
    for s in range(stream0, stream0 + tries):
        p = synth.prefix_tokens(om.d.vocab, length, stream=s)
        seq, logits = oracle_prefill(om, p)
        if top2_margin(logits[-1]) > min_margin:
            return p, seq
    raise RuntimeError("no decisive prefix found")


def planted_tree(om, seq, shape, p, stream):
    draws = synth.plant_draws(shape.n, om.d.vocab, stream=stream)
    return synth.plant_tree(shape, seq.pending, p, draws, argmax_fn_for_planting(om, seq))


def seq_copy(seq):
    """An independent copy of an oracle sequence state (oracle_verify replaces, never edits, its arrays)."""
    c = copy.copy(seq)
    c.k, c.v, c.tokens = list(seq.k), list(seq.v), list(seq.tokens)
    return c


def decided_tree(om, seq, shape, p, stream, min_margin=DECIDED_SMALL, tries=60):
    """A planted tree whose step is decided: the oracle's top-1 / top-2 margin exceeds
    `min_margin` at the root and along the accepted path.  Planting streams stream,
    stream + 1000, ... are tried in turn (the oracle alone decides; no GPU input).
    Returns (tokens, planting stream), or (None, None) when none of them is decided."""
    for k in range(tries):
        toks = planted_tree(om, seq, shape, p, stream + 1000 * k)
        r = oracle_verify(om, seq_copy(seq), toks, shape.parents)
        if np.all(r["margin"][[0] + list(r["accepted_nodes"])] > min_margin):
            return toks, stream + 1000 * k
    return None, None


def decided_case(om, P, shape, p, stream0, plant0=None, min_margin=DECIDED_SMALL, plant_tries=4, prefix_tries=40):
    """(prefix, oracle state, tree tokens) of a decided step.

    Planting mostly follows the target's greedy continuation, so a prefix whose
    continuation holds a near-tie leaves every planting undecided: prefixes of
    streams stream0, stream0 + 1, ... are tried, each with planting streams from
    `plant0` (default: the prefix's stream) on.  The tests pass the streams this
    search found, so that it ends at its first candidate."""
    for s in range(stream0, stream0 + prefix_tries):
        pre = synth.prefix_tokens(om.d.vocab, P, stream=s)
        seq, logits = oracle_prefill(om, pre)
        if top2_margin(logits[-1]) <= DECISIVE:
            continue
        toks, t = decided_tree(om, seq, shape, p, s if plant0 is None or s != stream0 else plant0, min_margin,
                               plant_tries)
        if toks is not None:
            decided_case.found = (s, t)
            return pre, seq, toks
    raise RuntimeError("no decided case within %d prefixes" % prefix_tries)


def decisive_nodes(result, parents):
    """Root plus the accepted path: the nodes whose argmax fixes the step's outputs."""
    return [0] + list(result["accepted_nodes"])


def kv_close(gpu, ref, tol):
    """|gpu - ref| <= tol * (1 + |ref|) elementwise."""
    return float(np.max(np.abs(gpu - ref) / (1.0 + np.abs(ref))))


def gpu_kv(eng, seq, length):
    """Cached K and V of one sequence as float64 arrays [layer][pos][Hkv][hd] (bf16 models: K = K + K_lo)."""
    kv = eng.kv_view()[:, :, seq, :, :length, :].to(torch.float64).cpu().numpy()
    kk = kv[:, 0] + kv[:, 2] if kv.shape[1] == 3 else kv[:, 0]
    k = np.transpose(kk, (0, 2, 1, 3))
    v = np.transpose(kv[:, 1], (0, 2, 1, 3))
    return k, v
