"""Stochastic (temperature) tree verification, float64 (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may use this module.

The pages state greedy acceptance only ("EAGLE-3投机解码：树验证器方法", section
验证-接受语义), say that EAGLE-3 leaves the target's output distribution
unchanged (kuma.akvtc.cn summary, introduction), mention sampling temperatures
of 0.7 to 1.2 (aitangshan.cn walkthrough, section 5.2) and cite Leviathan et
al., "Fast Inference from Transformers via Speculative Decoding" (course page,
section 参考) for the sampling case.  Reading taken here:

* The verification step is given draft tokens, not the draft's probabilities,
  so every draft token is a point-mass proposal q = delta(x).  Leviathan et
  al.'s rule with q = delta(x) accepts x with probability p(x) and, on a
  rejection, continues from the residual norm(max(0, p - q)) = p with x
  removed.  Several children of one node are tried in index order: child j
  with token x_j is accepted with probability p(x_j) / (1 - sum of the earlier
  children's distinct tokens' p), and when every child is rejected the node's
  token is drawn from p restricted to the other tokens.  The token that comes
  out at each node is then distributed exactly as p.

* That rule is carried out as one draw per node: y ~ p (temperature-T softmax
  of the target's logits), then the first child whose token equals y is
  accepted, and if none does, y is the bonus token.  Child j is accepted
  exactly when y equals x_j and no earlier child holds x_j, which has the
  probability above; the bonus, given that every child was rejected, is y
  conditioned on avoiding the children's tokens -- the residual.  With T -> 0, p
  puts all its mass on the argmax and the walk is the greedy one.

* The draw is the Gumbel-max trick: y = argmax_v (l_v / T + g_v) with g_v
  independent standard Gumbel variables (Gumbel, 1954; its use for sampling
  from a softmax is standard).  g_v = -ln(-ln u_v), u_v uniform in (0, 1).

* The uniforms come from the counter-based generator Philox4x32-10 (Salmon,
  Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011),
  keyed by a 64-bit seed, with counter (v, position, sequence, 0); word 0 of
  the output block x gives u = (2 * (x >> 9) + 1) / 2^24.  The noise of a tree
  node depends on its position P + depth only, so the emitted tokens are those
  of autoregressive sampling with the same noise (token t + 1 drawn with the
  noise of position t), whatever the tree.
"""

from __future__ import annotations

from typing import List, Sequence

import numpy as np

from .model import OracleModel, causal_logits, oracle_tree_features, top2_margin
from .tree import accept_walk, tree_meta

M0 = 0xD2511F53
M1 = 0xCD9E8D57
W0 = 0x9E3779B9
W1 = 0xBB67AE85
MASK = 0xFFFFFFFF


def _mulhilo(a: int, b: np.ndarray):
    prod = np.uint64(a) * b.astype(np.uint64)
    return (prod >> np.uint64(32)) & np.uint64(MASK), prod & np.uint64(MASK)


def philox4x32_10(ctr: Sequence[np.ndarray], key: Sequence[int]):
    """Philox4x32 with 10 rounds.  ctr: four arrays (or ints) of 32-bit words; key: two 32-bit words.

    Round: (hi0, lo0) = M0 * c0, (hi1, lo1) = M1 * c2 (full 64-bit products);
    c' = (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0); the key is bumped by the Weyl
    constants (W0, W1) before every round but the first."""
    c = [np.asarray(x, dtype=np.uint64) & np.uint64(MASK) for x in ctr]
    k0, k1 = np.uint64(key[0] & MASK), np.uint64(key[1] & MASK)
    for r in range(10):
        if r:
            k0 = np.uint64((int(k0) + W0) & MASK)
            k1 = np.uint64((int(k1) + W1) & MASK)
        hi0, lo0 = _mulhilo(M0, c[0])
        hi1, lo1 = _mulhilo(M1, c[2])
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return [x.astype(np.uint32) for x in c]


def uniforms(seed: int, seq: int, pos: int, n: int) -> np.ndarray:
    """u_v, v = 0 .. n-1, for one (seed, sequence, position): float64 in (0, 1), exact multiples of 2^-24."""
    v = np.arange(n, dtype=np.uint64)
    z = np.zeros(n, dtype=np.uint64)
    x = philox4x32_10([v, z + np.uint64(pos), z + np.uint64(seq), z], [seed & MASK, (seed >> 32) & MASK])[0]
    return (2.0 * (x.astype(np.float64) // 512) + 1.0) / float(1 << 24)


def gumbel_noise(seed: int, seq: int, pos: int, n: int) -> np.ndarray:
    """g_v = -ln(-ln u_v), written with w = 1 - u (exact) as -ln(-log1p(-w))."""
    w = 1.0 - uniforms(seed, seq, pos, n)
    return -np.log(-np.log1p(-w))


def perturbed_scores(logits: np.ndarray, temperature: float, seed: int, seq: int, pos: Sequence[int]) -> np.ndarray:
    """l / T + g per row (rows at positions pos[r]); argmax of a row is its sampled token."""
    lg = np.atleast_2d(np.asarray(logits, dtype=np.float64))
    out = np.empty_like(lg)
    for r in range(lg.shape[0]):
        out[r] = lg[r] / temperature + gumbel_noise(seed, seq, int(pos[r]), lg.shape[1])
    return out


def sampled_tokens(logits, temperature: float, seed: int, seq: int, pos: Sequence[int]) -> np.ndarray:
    """The sampled token of each row: argmax of the perturbed scores (lowest index on ties)."""
    return np.argmax(perturbed_scores(logits, temperature, seed, seq, pos), axis=1)


def softmax_t(logits: np.ndarray, temperature: float) -> np.ndarray:
    z = np.asarray(logits, dtype=np.float64) / temperature
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def sequential_rejection(p: np.ndarray, child_tokens: Sequence[int], u_accept: Sequence[float], u_residual: float):
    """Leviathan et al.'s rule with point-mass proposals, step by step, for one node whose children hold
    `child_tokens` in index order: returns (index of the accepted child or -1, emitted token).

    Child j is accepted when u_accept[j] < p'(x_j), p' being p with the tokens of the rejected earlier
    children removed and renormalised; otherwise x_j is removed.  When all are rejected, the token is drawn
    from the remaining p' by inversion with u_residual.  (A pin for the single-draw form used by the
    verification: both give the same output distribution.)"""
    q = np.asarray(p, dtype=np.float64).copy()
    for j, x in enumerate(child_tokens):
        mass = q.sum()
        if mass > 0 and u_accept[j] < q[x] / mass:
            return j, int(x)
        q[x] = 0.0
    cdf = np.cumsum(q / q.sum())
    return -1, int(min(np.searchsorted(cdf, u_residual, side="right"), len(cdf) - 1))


def oracle_sample_verify(model: OracleModel, seq, tokens: Sequence[int], parents: Sequence[int],
                         temperature: float, seed: int, seq_id: int, check_root: bool = True) -> dict:
    """Stochastic tree-verification step; updates `seq` in place like oracle.oracle_verify.

    Node i's token y_i is sampled at position P + depth(i) (Gumbel-max, see the module notes); the walk
    accepts, from the root, the first child whose token equals the current node's y and emits y of the last
    accepted node as the bonus.  Returns the oracle_verify fields plus "sampled" (y per node), "scores"
    (perturbed scores l / T + g) and "score_margin" (top-1 minus top-2 of those)."""
    tokens = [int(t) for t in tokens]
    if check_root and tokens[0] != seq.pending:
        raise ValueError("tokens[0] must be the pending token %d" % seq.pending)
    depth, _ = tree_meta(parents)
    P = seq.length
    logits, tree_kv, _ = oracle_tree_features(model, seq, tokens, parents, ())
    scores = perturbed_scores(logits, temperature, seed, seq_id, P + depth)
    y = np.argmax(scores, axis=1)
    acc_nodes, bonus = accept_walk(tokens, parents, y)
    keep = [0] + acc_nodes
    for l, (k, v) in enumerate(tree_kv):
        seq.k[l] = np.concatenate([seq.k[l], k[keep]], axis=0) if seq.k[l].size else k[keep]
        seq.v[l] = np.concatenate([seq.v[l], v[keep]], axis=0) if seq.v[l].size else v[keep]
    seq.tokens.extend(tokens[i] for i in keep)
    seq.pending = int(bonus)
    return {"accepted_len": len(acc_nodes), "accepted_nodes": acc_nodes,
            "accepted_tokens": [tokens[i] for i in acc_nodes], "bonus": int(bonus), "sampled": y,
            "logits": logits, "scores": scores, "score_margin": top2_margin(scores), "tree_kv": tree_kv}


def oracle_sample_ar(model: OracleModel, prompt: Sequence[int], n_new: int, temperature: float, seed: int,
                     seq_id: int) -> List[int]:
    """Autoregressive sampling by brute force (a full causal recompute per token): the token after position t
    is argmax(l_t / T + g(seed, seq_id, t)).  The first returned token follows the prompt's last position."""
    toks = [int(t) for t in prompt]
    out = []
    for _ in range(n_new):
        lg = causal_logits(model, toks)[-1]
        t = int(sampled_tokens(lg[None, :], temperature, seed, seq_id, [len(toks) - 1])[0])
        out.append(t)
        toks.append(t)
    return out


def sampled_pending(logits_last: np.ndarray, temperature: float, seed: int, seq_id: int, P: int) -> int:
    """The pending token after a prefill of P tokens: sampled at position P - 1."""
    return int(sampled_tokens(np.atleast_2d(logits_last), temperature, seed, seq_id, [P - 1])[0])
