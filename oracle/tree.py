"""Tree metadata and the greedy acceptance walk (float64 oracle, test infrastructure).

Pins: the chain example and the acceptance rule of "EAGLE-3投机解码：树验证器方法"
(sections 问题 and 验证-接受语义); the four-path tree of section 树draft vs 链draft.
"""

from __future__ import annotations

from typing import List, Tuple

import numpy as np


class TreeError(ValueError):
    pass


def _check_parents(parents) -> np.ndarray:
    p = np.asarray(parents, dtype=np.int64)
    if p.ndim != 1 or p.size == 0:
        raise TreeError("parents must be a non-empty 1-d array")
    if p[0] != -1:
        raise TreeError("parents[0] must be -1 (node 0 is the root)")
    for i in range(1, p.size):
        if not (0 <= p[i] < i):
            raise TreeError("parents[%d]=%d must satisfy 0 <= parent < %d" % (i, p[i], i))
    return p


def tree_meta(parents) -> Tuple[np.ndarray, List[List[int]]]:
    """Depth of every node and its ancestor set (itself included), by walking parent links.

    The tree structure is fixed before verification and every node sees only
    its ancestors ("EAGLE-3投机解码：树验证器方法", section 树draft vs 链draft).
    Node 0 is the root at depth 0.
    """
    p = _check_parents(parents)
    n = p.size
    depth = np.zeros(n, np.int64)
    anc: List[List[int]] = []
    for i in range(n):
        chain = []
        j = i
        while j != -1:
            chain.append(j)
            j = int(p[j])
        anc.append(sorted(chain))
        depth[i] = len(chain) - 1
    return depth, anc


def ancestor_matrix(parents) -> np.ndarray:
    """bool [n][n]: entry (i, j) is True iff node j is node i or one of its ancestors."""
    _, anc = tree_meta(parents)
    n = len(anc)
    m = np.zeros((n, n), bool)
    for i, a in enumerate(anc):
        m[i, a] = True
    return m


def root_paths(parents) -> List[List[int]]:
    """Node ids on the path root -> i, for every node i."""
    _, anc = tree_meta(parents)
    return anc  # ancestors sorted by index are in root-to-node order (parents[i] < i)


def accept_walk(tokens, parents, argmax) -> Tuple[List[int], int]:
    """Greedy acceptance over a tree.

    Starting at the root, move to the lowest-index child whose token equals the
    target's argmax at the current node; stop when no child matches.  Returns
    the accepted draft nodes (root excluded) and the bonus token, which is the
    target's argmax at the last accepted node ("EAGLE-3投机解码：树验证器方法",
    section 验证-接受语义: accept d_i iff d_i == argmax(p_i), stop at the first
    mismatch, emit the matches plus the target's token at that position).
    """
    p = _check_parents(parents)
    tok = np.asarray(tokens, dtype=np.int64)
    a = np.asarray(argmax, dtype=np.int64)
    n = p.size
    children: List[List[int]] = [[] for _ in range(n)]
    for i in range(1, n):
        children[int(p[i])].append(i)
    cur = 0
    accepted: List[int] = []
    while True:
        nxt = -1
        for c in children[cur]:  # increasing index
            if tok[c] == a[cur]:
                nxt = c
                break
        if nxt < 0:
            break
        accepted.append(nxt)
        cur = nxt
    return accepted, int(a[cur])
