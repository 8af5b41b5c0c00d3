"""Float64 target-model forward, tree verification and greedy decoding (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may use this module.

Everything is float64.  Weights arrive as host arrays in their storage format
(float32, or uint16 holding bfloat16 bit patterns) and are decoded exactly.

The decoder is the standard Llama block, written out as its definition:

* RMSNorm  y = x / sqrt(mean(x^2) + eps) * w
* rotary embedding with the rotate-half pairing: element j of the first half
  and element j of the second half form one pair, rotated by pos * theta^(-2j/hd)
* grouped-query attention: query head j reads key/value head j // (Hq / Hkv),
  scores scaled by 1/sqrt(hd), softmax over the visible keys
* SwiGLU MLP  (silu(h Wg^T) * (h Wu^T)) Wd^T
* pre-norm residual blocks, a final RMSNorm and an untied LM head.

Tree verification ("EAGLE-3投机解码：树验证器方法", sections 验证-接受语义 and
树draft vs 链draft):

* node 0 is the pending token (emitted by the previous step, not yet cached)
  at position P; its logits judge its children.  Node i sits at position
  P + depth(i) and attends to the whole prefix and to its ancestors only;
* the target's argmax at each node (lowest index on ties) decides acceptance;
  the walk keeps the longest accepted root path and emits one bonus token;
* only the root and the accepted nodes' K/V enter the cache, at positions
  P, P+1, ..., P+accepted_len; the bonus becomes the next pending token.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from .tree import accept_walk, ancestor_matrix, tree_meta

try:
    import torch  # used only to decode bfloat16 bit patterns quickly (an exact format conversion)
except Exception:  # pragma: no cover
    torch = None


# ---------------------------------------------------------------------------
# format decoding
# ---------------------------------------------------------------------------

def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 copy of a float32 array or of bfloat16 bit patterns held as uint16."""
    if a.dtype == np.uint16:
        if torch is not None and a.size > (1 << 16):
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
            return t.to(torch.float64).numpy()
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# decoder pieces (definitions)
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * w


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding.  x: [T][H][hd]; pos: [T]."""
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = theta ** (-(np.arange(half, dtype=np.float64) * 2.0) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]  # [T][half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, visible: np.ndarray) -> np.ndarray:
    """q [T][Hq][hd], k/v [S][Hkv][hd], visible bool [T][S] -> [T][Hq][hd]."""
    T, Hq, hd = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    out = np.empty_like(q)
    scale = 1.0 / math.sqrt(hd)
    for h in range(Hq):
        kh = h // group
        s = (q[:, h, :] @ k[:, kh, :].T) * scale
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, kh, :]
    return out


def top2_margin(logits: np.ndarray) -> np.ndarray:
    """top-1 minus top-2 logit per row (0 on an exact tie)."""
    part = np.partition(logits, -2, axis=-1)
    return part[..., -1] - part[..., -2]


# ---------------------------------------------------------------------------
# model
# ---------------------------------------------------------------------------

class OracleModel:
    """Holds the weights (host arrays in storage format) and runs float64 forwards.

    `dims` is any object with n_layers, hidden, n_q_heads, n_kv_heads,
    head_dim, ffn, vocab, rms_eps, rope_theta.
    """

    def __init__(self, dims, weights: dict, cache_limit_bytes: int = 4 << 30):
        self.d = dims
        self.w = weights
        total = weights["embed"].size + weights["lm_head"].size
        for lw in weights["layers"]:
            total += sum(v.size for v in lw.values())
        self._cache_all = total * 8 <= cache_limit_bytes
        self._cache: Dict[tuple, np.ndarray] = {}

    def _get(self, key: tuple, arr: np.ndarray) -> np.ndarray:
        if not self._cache_all:
            return to_f64(arr)
        if key not in self._cache:
            self._cache[key] = to_f64(arr)
        return self._cache[key]

    def layer(self, l: int) -> Dict[str, np.ndarray]:
        return {k: self._get(("L", l, k), v) for k, v in self.w["layers"][l].items()}

    def embed(self, tokens: Sequence[int]) -> np.ndarray:
        rows = self.w["embed"][np.asarray(tokens, dtype=np.int64)]
        return to_f64(rows)

    def lm_logits(self, x: np.ndarray) -> np.ndarray:
        """final RMSNorm then the LM head, vocab processed in blocks to bound memory."""
        d = self.d
        h = rms_norm(x, self._get(("final_norm",), self.w["final_norm"]), d.rms_eps)
        if self._cache_all:
            return h @ self._get(("lm_head",), self.w["lm_head"]).T
        V = self.w["lm_head"].shape[0]
        out = np.empty((x.shape[0], V), np.float64)
        blk = 16384
        for s in range(0, V, blk):
            out[:, s:s + blk] = h @ to_f64(self.w["lm_head"][s:s + blk]).T
        return out

    def layer_forward(self, l: int, x: np.ndarray, pos: np.ndarray,
                      past_k: Optional[np.ndarray], past_v: Optional[np.ndarray],
                      vis_new: np.ndarray, past_visible: Optional[np.ndarray] = None):
        """One pre-norm decoder layer.  Returns (x_out, k_new, v_new).

        Rows of x attend to every past key (or to those marked in
        `past_visible`) and to the new rows marked in `vis_new`.
        """
        d = self.d
        n = x.shape[0]
        lw = self.layer(l)
        h = rms_norm(x, lw["attn_norm"], d.rms_eps)
        q = (h @ lw["wq"].T).reshape(n, d.n_q_heads, d.head_dim)
        k = (h @ lw["wk"].T).reshape(n, d.n_kv_heads, d.head_dim)
        v = (h @ lw["wv"].T).reshape(n, d.n_kv_heads, d.head_dim)
        q = rope(q, pos, d.rope_theta)
        k = rope(k, pos, d.rope_theta)
        S = 0 if past_k is None else past_k.shape[0]
        if S:
            K = np.concatenate([past_k, k], axis=0)
            Vv = np.concatenate([past_v, v], axis=0)
            pv = np.ones((n, S), bool) if past_visible is None else past_visible
            vis = np.concatenate([pv, vis_new], axis=1)
        else:
            K, Vv, vis = k, v, vis_new
        o = attention(q, K, Vv, vis)
        x = x + o.reshape(n, d.n_q_heads * d.head_dim) @ lw["wo"].T
        h2 = rms_norm(x, lw["mlp_norm"], d.rms_eps)
        x = x + (silu(h2 @ lw["w_gate"].T) * (h2 @ lw["w_up"].T)) @ lw["w_down"].T
        return x, k, v

    def forward(self, tokens: Sequence[int], pos: np.ndarray, past: Optional[List[Tuple[np.ndarray, np.ndarray]]],
                vis_new: np.ndarray):
        """Full forward of new rows on top of a cache.  Returns (logits [n][V], new K/V per layer)."""
        logits, new_kv, _ = self.forward_features(tokens, pos, past, vis_new, ())
        return logits, new_kv

    def forward_features(self, tokens: Sequence[int], pos: np.ndarray,
                         past: Optional[List[Tuple[np.ndarray, np.ndarray]]], vis_new: np.ndarray,
                         taps: Sequence[int]):
        """As `forward`, and also the residual stream after taps[f] decoder layers
        (1 <= taps[f] <= n_layers) for every row: features [n][len(taps)][d].

        EAGLE-3 (draft-stage description) feeds its draft head with the target's
        low-, mid- and high-level hidden states of each position; these are the
        residual stream between decoder blocks, before any norm."""
        L = self.d.n_layers
        for j in taps:
            if not 1 <= j <= L:
                raise ValueError("feature layer %d outside [1, %d]" % (j, L))
        x = self.embed(tokens)
        after = {}
        new_kv = []
        for l in range(L):
            pk, pv = (None, None) if not past else past[l]
            x, k, v = self.layer_forward(l, x, pos, pk, pv, vis_new)
            new_kv.append((k, v))
            after[l + 1] = x
        feats = np.stack([after[j] for j in taps], axis=1) if taps else np.zeros((x.shape[0], 0, x.shape[1]))
        return self.lm_logits(x), new_kv, feats


def causal_logits(model: OracleModel, tokens: Sequence[int]) -> np.ndarray:
    """Plain causal forward over a token sequence at positions 0..T-1 (no cache)."""
    T = len(tokens)
    vis = np.tril(np.ones((T, T), bool))
    logits, _ = model.forward(tokens, np.arange(T), None, vis)
    return logits


def causal_features(model: OracleModel, tokens: Sequence[int], taps: Sequence[int]) -> np.ndarray:
    """Residual stream after taps[f] layers of a plain causal forward (no cache): [T][len(taps)][d]."""
    T = len(tokens)
    vis = np.tril(np.ones((T, T), bool))
    _, _, feats = model.forward_features(tokens, np.arange(T), None, vis, taps)
    return feats


# ---------------------------------------------------------------------------
# sequence state, prefill, tree verification
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class OracleSeq:
    k: List[np.ndarray]       # per layer [len][Hkv][hd], post-rotary keys
    v: List[np.ndarray]       # per layer [len][Hkv][hd]
    tokens: List[int]         # tokens whose K/V are cached, position by position
    pending: int              # emitted, not yet cached; the root of the next tree

    @property
    def length(self) -> int:
        return len(self.tokens)


def oracle_prefill(model: OracleModel, prompt: Sequence[int]) -> Tuple[OracleSeq, np.ndarray]:
    """Causal forward over the prompt; caches every position; pending = argmax at the last one."""
    T = len(prompt)
    vis = np.tril(np.ones((T, T), bool))
    logits, kv = model.forward(prompt, np.arange(T), None, vis)
    seq = OracleSeq([k for k, _ in kv], [v for _, v in kv], [int(t) for t in prompt],
                    int(np.argmax(logits[-1])))
    return seq, logits


def oracle_tree_logits(model: OracleModel, seq: OracleSeq, tokens: Sequence[int], parents: Sequence[int]):
    """One target forward over a whole draft tree on top of the cache.

    Returns (logits [n][V], per-layer tree K/V).  Node i is at position
    P + depth(i) and sees the prefix plus its ancestors (itself included).
    """
    logits, kv, _ = oracle_tree_features(model, seq, tokens, parents, ())
    return logits, kv


def oracle_tree_features(model: OracleModel, seq: OracleSeq, tokens: Sequence[int], parents: Sequence[int],
                         taps: Sequence[int]):
    """As `oracle_tree_logits`, plus the residual stream after taps[f] layers at every node."""
    depth, _ = tree_meta(parents)
    P = seq.length
    vis = ancestor_matrix(parents)
    past = list(zip(seq.k, seq.v)) if P else None
    return model.forward_features(tokens, P + depth, past, vis, taps)


def oracle_verify(model: OracleModel, seq: OracleSeq, tokens: Sequence[int], parents: Sequence[int],
                  check_root: bool = True, taps: Sequence[int] = ()) -> dict:
    """Tree-verification step; updates `seq` in place (KV compaction, length, pending).

    Returns accepted_len (accepted drafts), accepted_nodes, accepted_tokens,
    bonus, plus argmax / logits / margin per node for parity checks.  With
    `taps`, also "features": the residual stream after taps[f] layers of the
    root and of each accepted node, in path order ([accepted_len + 1][len(taps)][d]),
    the draft head's input for the positions the step emits.
    """
    tokens = [int(t) for t in tokens]
    if check_root and tokens[0] != seq.pending:
        raise ValueError("tokens[0] must be the pending token %d" % seq.pending)
    logits, tree_kv, feats = oracle_tree_features(model, seq, tokens, parents, taps)
    amax = np.argmax(logits, axis=1)  # first (lowest) index on ties
    acc_nodes, bonus = accept_walk(tokens, parents, amax)
    keep = [0] + acc_nodes
    for l, (k, v) in enumerate(tree_kv):
        seq.k[l] = np.concatenate([seq.k[l], k[keep]], axis=0) if seq.k[l].size else k[keep]
        seq.v[l] = np.concatenate([seq.v[l], v[keep]], axis=0) if seq.v[l].size else v[keep]
    seq.tokens.extend(tokens[i] for i in keep)
    seq.pending = int(bonus)
    return {
        "accepted_len": len(acc_nodes),
        "accepted_nodes": acc_nodes,
        "accepted_tokens": [tokens[i] for i in acc_nodes],
        "bonus": int(bonus),
        "argmax": amax,
        "logits": logits,
        "margin": top2_margin(logits),
        "tree_kv": tree_kv,
        "features": feats[keep],
    }


def oracle_greedy_ar(model: OracleModel, prompt: Sequence[int], n_new: int) -> List[int]:
    """Greedy autoregressive decoding by brute force: a full causal recompute per token, no cache."""
    seq = [int(t) for t in prompt]
    out = []
    for _ in range(n_new):
        logits = causal_logits(model, seq)
        t = int(np.argmax(logits[-1]))
        out.append(t)
        seq.append(t)
    return out


def argmax_fn_for_planting(model: OracleModel, seq: OracleSeq):
    """argmax per node of a (truncated) tree on top of `seq`, for planting tree tokens."""
    def fn(tokens, parents):
        logits, _ = oracle_tree_logits(model, seq, tokens, parents)
        return np.argmax(logits, axis=1)
    return fn
