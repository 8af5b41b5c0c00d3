"""Shared set-up for the GPU parity tests: one seeded model, the library
engine on the GPU and the float64 oracle on the CPU, fed the same bits."""

from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import OracleModel, argmax_fn_for_planting, oracle_prefill, top2_margin

# logit tolerance stated for the verification step: 2e-2 absolute for bf16
# models, 1e-4 for fp32 models
TOL = {"bf16": 2e-2, "f32": 1e-4}
# the step's outputs must be identical wherever the oracle's top-1 / top-2
# margin exceeds this on every node that decides them
DECISIVE = 0.05


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


def decisive_nodes(result, parents):
    """Root plus the accepted path: the nodes whose argmax fixes the step's outputs."""
    return [0] + list(result["accepted_nodes"])


def kv_close(gpu, ref, tol):
    """|gpu - ref| <= tol * (1 + |ref|) elementwise."""
    return float(np.max(np.abs(gpu - ref) / (1.0 + np.abs(ref))))


def gpu_kv(eng, seq, length):
    """Cached K and V of one sequence as float64 arrays [layer][pos][Hkv][hd]."""
    kv = eng.kv_view()[:, :, seq, :, :length, :].to(torch.float64).cpu().numpy()
    k = np.transpose(kv[:, 0], (0, 2, 1, 3))
    v = np.transpose(kv[:, 1], (0, 2, 1, 3))
    return k, v
