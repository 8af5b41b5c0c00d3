"""Seeded synthetic workloads for EAGLE-3 tree verification.

Seeds (one stream per purpose, so that changing one input never shifts another):

    0  model weights: N(0, 0.02) for every matrix and embedding, norm weights 1
    1  prefix tokens, uniform over [0, V)
    2  tree shapes (parent draws)
    3  planting draws (one uniform and one random token per draft node)
    4  per-sequence prefix lengths and acceptance probabilities (batch-64 case)
    5  draft-head input features N(0, 1)

The workloads stand in for the benchmarks the EAGLE-3 pages measure on
(MT-bench, HumanEval, GSM8K, Alpaca, CNN/DM, Spec-Bench), whose prompts and
trained weights are not available here: random-init models of the named shapes,
uniform random prefixes and trees whose acceptance is planted with a fixed
probability.  Tree-inference parameters (depth 8, 60 draft tokens, top-k 10)
follow the inference-parameter table of the aitangshan.cn walkthrough of
EAGLE-3 (section 4.2, table 6).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Callable, Dict, List, Optional, Sequence

import numpy as np

try:  # torch is only needed for weight generation
    import torch
except Exception:  # pragma: no cover
    torch = None


# ---------------------------------------------------------------------------
# model shapes
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class ModelDims:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float
    rope_theta: float
    dtype: str  # "f32" or "bf16"

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim


# 2 layers, hidden 256, 4 heads of 64 (MHA), SwiGLU 688, vocab 1024, fp32.
TINY = ModelDims(2, 256, 4, 4, 64, 688, 1024, 1e-5, 10000.0, "f32")
# Llama-3.1-8B shape (no llama3 frequency scaling), bf16.
LLAMA8B = ModelDims(32, 4096, 32, 8, 128, 14336, 128256, 1e-5, 500000.0, "bf16")
# Small bf16 models with the 8B structure (GQA 4:1, head_dim 128) that the
# oracle finishes in seconds; they span several GEMM tiles and ragged tails.
MINI_BF16 = ModelDims(2, 512, 4, 1, 128, 1024, 2048, 1e-5, 500000.0, "bf16")
SMALL_BF16 = ModelDims(2, 1024, 8, 2, 128, 2816, 8320, 1e-5, 500000.0, "bf16")
# 8B layer shapes with fewer layers and a shorter vocab: full-size GEMM tiles
# and split factors at an oracle cost of seconds.
WIDE_BF16 = ModelDims(2, 4096, 32, 8, 128, 14336, 16384, 1e-5, 500000.0, "bf16")


# ---------------------------------------------------------------------------
# weights
# ---------------------------------------------------------------------------

LAYER_KEYS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "attn_norm", "mlp_norm")


def layer_shapes(d: ModelDims) -> Dict[str, tuple]:
    return {
        "wq": (d.q_dim, d.hidden),
        "wk": (d.kv_dim, d.hidden),
        "wv": (d.kv_dim, d.hidden),
        "wo": (d.hidden, d.q_dim),
        "w_gate": (d.ffn, d.hidden),
        "w_up": (d.ffn, d.hidden),
        "w_down": (d.hidden, d.ffn),
        "attn_norm": (d.hidden,),
        "mlp_norm": (d.hidden,),
    }


def model_weights(d: ModelDims, seed: int = 0, device: str = "cpu") -> dict:
    """Random-init weights as torch tensors in the model dtype.

    Matrices are drawn in a fixed order from one generator: embed, then per
    layer wq, wk, wv, wo, w_gate, w_up, w_down, then lm_head.  Every matrix is
    stored [out][in], row-major.  Norm weights are ones.
    """
    assert torch is not None
    tdt = torch.float32 if d.dtype == "f32" else torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def mat(r, c):
        t = torch.randn(r, c, generator=g, device=device, dtype=torch.float32)
        t.mul_(0.02)
        return t.to(tdt)

    def ones(n):
        return torch.ones(n, device=device, dtype=tdt)

    w = {"embed": mat(d.vocab, d.hidden), "layers": []}
    shapes = layer_shapes(d)
    for _ in range(d.n_layers):
        lw = {}
        for k in LAYER_KEYS:
            s = shapes[k]
            lw[k] = mat(*s) if len(s) == 2 else ones(s[0])
        w["layers"].append(lw)
    w["lm_head"] = mat(d.vocab, d.hidden)
    w["final_norm"] = ones(d.hidden)
    return w


def tensor_to_host(t) -> np.ndarray:
    """fp32 tensors become float32 arrays; bf16 tensors become their uint16 bit patterns."""
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def weights_to_host(w: dict) -> dict:
    out = {k: tensor_to_host(v) for k, v in w.items() if k != "layers"}
    out["layers"] = [{k: tensor_to_host(v) for k, v in lw.items()} for lw in w["layers"]]
    return out


# ---------------------------------------------------------------------------
# prefix tokens
# ---------------------------------------------------------------------------

def prefix_tokens(vocab: int, length: int, seed: int = 1, stream: int = 0) -> np.ndarray:
    rng = np.random.default_rng([seed, stream])
    return rng.integers(0, vocab, size=length, dtype=np.int64).astype(np.int32)


# ---------------------------------------------------------------------------
# draft-tree shapes
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class TreeShape:
    """Nodes in BFS order: node 0 is the root (the pending token), parents[0] = -1."""
    parents: np.ndarray  # int32 [n]
    level: np.ndarray    # int32 [n], level 0 = root

    @property
    def n(self) -> int:
        return int(self.parents.shape[0])


MAX_CHILDREN = 10  # top-k 10 expansion


def tree_from_widths(widths: Sequence[int], seed: int = 2, stream: int = 0) -> TreeShape:
    """Seeded tree with the given per-level widths (level 1 .. depth).

    Each level-l node draws its parent among the level-(l-1) nodes with
    probability proportional to 1/(rank+1), rank being the parent's position in
    its level (a top-heavy shape like a confidence-ranked expansion); no parent
    takes more than 10 children.  Within a level the nodes are sorted by
    (parent, draw order), which keeps the array in BFS order.
    """
    rng = np.random.default_rng([seed, stream])
    parents = [-1]
    level = [0]
    prev = [0]  # node ids of the previous level
    for lvl, w in enumerate(widths, start=1):
        counts = {p: 0 for p in prev}
        draws = []
        for j in range(w):
            cand = [p for p in prev if counts[p] < MAX_CHILDREN]
            if not cand:
                raise ValueError("level %d wider than %d x previous level" % (lvl, MAX_CHILDREN))
            wts = np.array([1.0 / (prev.index(p) + 1) for p in cand])
            p = cand[int(rng.choice(len(cand), p=wts / wts.sum()))]
            counts[p] += 1
            draws.append((p, j))
        draws.sort()
        cur = []
        for p, _ in draws:
            cur.append(len(parents))
            parents.append(p)
            level.append(lvl)
        prev = cur
    return TreeShape(np.asarray(parents, np.int32), np.asarray(level, np.int32))


def chain(length: int) -> TreeShape:
    """Root plus a linear chain of `length` drafts."""
    parents = np.arange(-1, length, dtype=np.int32)
    return TreeShape(parents, np.arange(length + 1, dtype=np.int32))


def tiny_tree() -> TreeShape:
    """8 drafts at depth 4 with per-level widths 2, 4, 1, 1.

    The root has two children; each of them has two; only the lowest-index
    level-2 node has a child, which has one child.
    """
    parents = np.array([-1, 0, 0, 1, 1, 2, 2, 3, 7], np.int32)
    level = np.array([0, 1, 1, 2, 2, 2, 2, 3, 4], np.int32)
    return TreeShape(parents, level)


# per-level widths of the trees in the chain-versus-tree sweep (depth 8)
SWEEP_WIDTHS = {
    16: (3, 3, 3, 2, 2, 1, 1, 1),
    32: (6, 6, 5, 4, 4, 3, 2, 2),
    60: (10, 10, 10, 8, 8, 6, 4, 4),
    80: (10, 12, 12, 12, 10, 10, 8, 6),
}
TREE60_WIDTHS = SWEEP_WIDTHS[60]


# ---------------------------------------------------------------------------
# planting
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class PlantDraws:
    u: np.ndarray         # float64 [n]; node i copies the target's choice iff u[i] < p
    rand_tok: np.ndarray  # int32 [n]; token used otherwise


def plant_draws(n: int, vocab: int, seed: int = 3, stream: int = 0) -> PlantDraws:
    rng = np.random.default_rng([seed, stream])
    u = rng.random(n)
    rt = rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)
    return PlantDraws(u, rt)


ArgmaxFn = Callable[[np.ndarray, np.ndarray], np.ndarray]


def plant_tree(shape: TreeShape, root_token: int, p: float, draws: PlantDraws,
               argmax_fn: ArgmaxFn) -> np.ndarray:
    """Fill a tree's tokens level by level.

    With probability p a node copies the target's choice at its parent (as
    returned by `argmax_fn(tokens, parents)` for the truncated tree of all
    shallower nodes), otherwise it takes a uniform random token.  The random
    token may equal the target's choice by chance.
    """
    n = shape.n
    tokens = np.zeros(n, np.int32)
    tokens[0] = root_token
    depth = int(shape.level.max()) if n > 1 else 0
    for lvl in range(1, depth + 1):
        k = int(np.sum(shape.level < lvl))
        assert np.all(shape.level[:k] < lvl), "tree must be in BFS order"
        a = np.asarray(argmax_fn(tokens[:k].copy(), shape.parents[:k].copy()))
        for i in np.nonzero(shape.level == lvl)[0]:
            tokens[i] = a[shape.parents[i]] if draws.u[i] < p else draws.rand_tok[i]
    return tokens


# ---------------------------------------------------------------------------
# batch-64 per-sequence draws
# ---------------------------------------------------------------------------

def batch_prefix_lengths_and_p(batch: int, lo: int = 512, hi: int = 4096,
                               p_lo: float = 0.6, p_hi: float = 0.9, seed: int = 4):
    rng = np.random.default_rng([seed])
    lens = rng.integers(lo, hi + 1, size=batch, dtype=np.int64).astype(np.int32)
    ps = rng.uniform(p_lo, p_hi, size=batch)
    return lens, ps


# ---------------------------------------------------------------------------
# draft-head features
# ---------------------------------------------------------------------------

def draft_features(rows: int, hidden: int, seed: int = 5, device: str = "cpu"):
    """Low/mid/high target features, N(0, 1), as a bf16 tensor [rows][3][hidden]."""
    assert torch is not None
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(rows, 3, hidden, generator=g, device=device, dtype=torch.float32)
    return t.to(torch.bfloat16)


def draft_head_weights(d: ModelDims, seed: int = 6, device: str = "cpu") -> dict:
    """Draft-head weights: fc_fuse [d][3d], fc_in [d][2d], one decoder layer, final norm."""
    assert torch is not None
    tdt = torch.float32 if d.dtype == "f32" else torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def mat(r, c):
        t = torch.randn(r, c, generator=g, device=device, dtype=torch.float32)
        t.mul_(0.02)
        return t.to(tdt)

    w = {"fc_fuse": mat(d.hidden, 3 * d.hidden), "fc_in": mat(d.hidden, 2 * d.hidden)}
    shapes = layer_shapes(d)
    lw = {}
    for k in LAYER_KEYS:
        s = shapes[k]
        lw[k] = mat(*s) if len(s) == 2 else torch.ones(s[0], device=device, dtype=tdt)
    w["layer"] = lw
    w["final_norm"] = torch.ones(d.hidden, device=device, dtype=tdt)
    return w


# ---------------------------------------------------------------------------
# fingerprints of generated inputs
# ---------------------------------------------------------------------------

def weights_fingerprint(w: dict, row_stride: int = 509) -> str:
    """sha256 (hex, 16 digits) over every `row_stride`-th row of each matrix's raw bits.

    Stored beside precomputed expected values, so that a machine that draws
    different weights from the same seed (another torch build or CPU code
    path) is detected before any comparison is made."""
    import hashlib
    h = hashlib.sha256()

    def add(name, t):
        a = tensor_to_host(t)
        a2 = a.reshape(a.shape[0], -1) if a.ndim > 1 else a.reshape(1, -1)
        h.update(name.encode())
        h.update(np.ascontiguousarray(a2[::row_stride]).tobytes())

    for k in ("embed", "lm_head", "final_norm"):
        if k in w:
            add(k, w[k])
    for i, lw in enumerate(w.get("layers", [])):
        for k in LAYER_KEYS:
            add("%d.%s" % (i, k), lw[k])
    for k in ("fc_fuse", "fc_in"):
        if k in w:
            add(k, w[k])
    if "layer" in w:
        for k in LAYER_KEYS:
            add("layer." + k, w["layer"][k])
    return h.hexdigest()[:16]


def draft_vocab_ids(vocab: int, n: int, seed: int = 8) -> np.ndarray:
    """A reduced draft vocabulary: n distinct token ids, ascending, drawn uniformly (seed 8).

    Reduced draft vocabularies (VocabTrim, FR-Spec, SpecVocab) keep the tokens a
    corpus uses most; no corpus is available here, so a seeded uniform subset
    stands in for the frequency-ranked one."""
    rng = np.random.default_rng([seed, vocab, n])
    return np.sort(rng.choice(vocab, size=n, replace=False)).astype(np.int32)
