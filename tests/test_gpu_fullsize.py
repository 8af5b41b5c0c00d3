"""Properties at the benchmark's full size: the Llama-3.1-8B shape (32 layers,
d 4096, 32/8 heads, ffn 14336, vocab 128256), prefix 2048, the 60-draft tree,
through the same launch configuration bench.py times.

The float64 oracle cannot run 32 layers of this shape, so these checks use
facts that hold at any size ("EAGLE-3投机解码：树验证器方法", section 树draft vs
链draft: every node sees only its ancestors, so a node's logits are those of
its root path verified as a chain; section 验证-接受语义: drafts equal to the
target's argmax along a path are all accepted):
  * the step is bitwise deterministic;
  * changing the tokens of nodes outside a node's ancestor set leaves its
    logits bitwise unchanged;
  * each node's logits equal those of the chain of its root path scored alone
    (same kernels, other rows and masks: within 1e-3);
  * a tree planted with p = 1 (every node the target's own argmax at its parent)
    is accepted along lowest-index children down to a leaf, and the bonus is
    the target's argmax at that leaf.
"""

import numpy as np
import pytest

import synth
from oracle import accept_walk, ancestor_matrix, tree_meta

pytestmark = pytest.mark.gpu

P = 2048


@pytest.fixture(scope="module")
def full():
    from speculative_decoding_06_b200.engine import SpecEngine
    dims = synth.LLAMA8B
    w = synth.model_weights(dims, seed=0, device="cuda")
    eng = SpecEngine(dims, w, max_batch=1, max_seq=P + 256, max_nodes=128)
    pend = eng.prefill(0, synth.prefix_tokens(dims.vocab, P, seed=1))
    shape = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=0)
    yield eng, dims, pend, shape
    eng.close()


def _score(eng, toks, parents):
    eng.score([0], [(toks, parents)], flags=2)
    return eng.debug_logits(len(toks)).copy()


def test_fullsize_determinism_and_ancestor_isolation(full):
    eng, d, pend, shape = full
    draws = synth.plant_draws(shape.n, d.vocab, stream=0)
    toks = synth.plant_tree(shape, pend, 0.8, draws, lambda t, p_: eng.score([0], [(t, p_)])[0])
    a = _score(eng, toks, shape.parents)
    b = _score(eng, toks, shape.parents)
    assert np.array_equal(a, b), "logits differ between two identical steps"
    anc = ancestor_matrix(shape.parents)  # anc[i, j]: j is an ancestor of i (or i itself)
    rng = np.random.default_rng(3)
    for i in (shape.n - 1, shape.n // 2, 12):
        others = [j for j in range(1, shape.n) if not anc[i, j]]
        t2 = toks.copy()
        t2[others] = rng.integers(0, d.vocab, size=len(others))
        c = _score(eng, t2, shape.parents)
        assert np.array_equal(c[i], a[i]), "node %d saw a non-ancestor" % i
        # ...while nodes whose ancestors changed do see it
        changed = [j for j in range(shape.n) if any(anc[j, k] for k in others)]
        assert not np.array_equal(c[changed], a[changed])


def test_fullsize_tree_equals_chains(full):
    eng, d, pend, shape = full
    draws = synth.plant_draws(shape.n, d.vocab, stream=1)
    toks = synth.plant_tree(shape, pend, 0.8, draws, lambda t, p_: eng.score([0], [(t, p_)])[0])
    tree = _score(eng, toks, shape.parents)
    errs = {}
    for i in (shape.n - 1, 37, 9):
        path = [i]
        while shape.parents[path[-1]] >= 0:
            path.append(int(shape.parents[path[-1]]))
        path = path[::-1]
        chain = _score(eng, toks[path], np.arange(-1, len(path) - 1, dtype=np.int32))
        errs[i] = float(np.max(np.abs(chain[-1] - tree[i])))
    assert max(errs.values()) <= 1e-3, "tree vs chain logits differ by %s" % errs


def test_fullsize_planted_path_fully_accepted(full):
    eng, d, pend, shape = full
    draws = synth.plant_draws(shape.n, d.vocab, stream=2)
    toks = synth.plant_tree(shape, pend, 1.0, draws, lambda t, p_: eng.score([0], [(t, p_)])[0])
    amax = eng.score([0], [(toks, shape.parents)])[0]
    # every node is its parent's argmax: the walk follows lowest-index children to a leaf
    nodes, bonus_ref = accept_walk(toks, shape.parents, amax)
    depth, _ = tree_meta(shape.parents)
    leaf = nodes[-1]
    assert not any(shape.parents[j] == leaf for j in range(shape.n)), "the walk stopped before a leaf"
    assert len(nodes) == int(depth[leaf])
    a, acc_tok, bonus = eng.verify(0, toks, shape.parents)
    assert a == len(nodes) and acc_tok == [int(toks[j]) for j in nodes] and bonus == bonus_ref
    ln, pending = eng.seq_len(0)
    assert ln == P + 1 + a and pending == bonus
    eng.truncate(0, P)
