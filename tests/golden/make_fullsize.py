"""Write the expected values for the full-size parity tests (float64 oracle only).

    python tests/golden/make_fullsize.py [verify_p2048 | sweep_p8192 | batch64 | draft_b16 | all]

Each workload runs the float64 CPU oracle (``oracle/``) at the Llama-3.1-8B
shape -- 32 layers, d 4096, 32/8 heads of 128, ffn 14336, vocab 128256 --
on weights drawn on the CPU from seed 0 (``synth.model_weights``), and stores
a compact record under ``tests/golden/``.  Nothing here calls the CUDA
library; the GPU tests (``tests/test_gpu_fullsize_oracle.py``) load these
files, regenerate the same weights, and compare.

Stored per verification step: the prefix and tree, the oracle's pending token,
per-node argmax / top-1 / top-2 / top-16 (index and value), the logits at a
seeded set of vocabulary columns, the step's outputs (accepted length, nodes,
tokens, bonus) and the compacted K/V of chosen layers at slots P .. P+a plus a
few prefix slots.  Inputs are chosen so that every step is *decided*: the
oracle's top-1 / top-2 margin exceeds 0.05 at every node that fixes the
outputs (the root and the accepted path), and at the prefill's last position.
When a seeded stream misses that, the next stream (stream + 1000) is tried and
the one used is stored.

Workloads (the pages' settings: "EAGLE-3投机解码：树验证器方法", sections
验证-接受语义 and 树draft vs 链draft; tree sizes from the aitangshan.cn
walkthrough, section 4.2, table 6):
  verify_p2048  batch 1, prefix 2048, 60-draft depth-8 tree, planted p = 0.8
  sweep_p8192   batch 1, prefix 8192, chains 5 / 8 and trees 16 / 32 / 60 / 80, p = 0.85
  batch64       8 of the 64 sequences (prefixes U[512, 4096], p U[0.6, 0.9]),
                the shortest and the longest among them
  draft_b16     the EAGLE-3 draft-head step, batch 16, draft prefix 2048, 60-draft trees
"""

from __future__ import annotations

import argparse
import copy
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from oracle import OracleDraftHead, OracleModel, oracle_prefill, oracle_tree_logits, oracle_verify  # noqa: E402
from oracle.draft import top_k_rows  # noqa: E402
from oracle.model import top2_margin  # noqa: E402

DECISIVE = 0.05
TOPK_STORED = 16
N_COLS = 512
STREAM_STEP = 1000


def log(msg):
    print("[%s] %s" % (time.strftime("%H:%M:%S"), msg), flush=True)


def path(name):
    return os.path.join(HERE, "fullsize_%s.npz" % name)


def sampled_columns(vocab, n, tag):
    rng = np.random.default_rng([11, tag])
    return np.sort(rng.choice(vocab, size=n, replace=False)).astype(np.int32)


def target(dims):
    t0 = time.time()
    w = synth.model_weights(dims, seed=0, device="cpu")
    fp = synth.weights_fingerprint(w)
    host = synth.weights_to_host(w)
    log("weights drawn (%.0f s), fingerprint %s" % (time.time() - t0, fp))
    return w, host, fp


class Undecided(Exception):
    pass


def _deciding_path(tokens, parents, amax):
    """Nodes the greedy walk visits over a (possibly truncated) tree: the root and the accepted nodes."""
    path = [0]
    while True:
        cur = path[-1]
        nxt = [c for c in range(1, len(parents)) if parents[c] == cur and tokens[c] == amax[cur]]
        if not nxt:
            return path
        path.append(nxt[0])


def decided_case(om, P, shape, p, stream0, plant_tries=3, prefix_tries=40, seed=1):
    """A decided step: prefix streams stream0, stream0 + 1000, ... (prefill margin > 0.05), each with
    planting streams s, s + 1000, ... until the root and every accepted node have margins above 0.05.

    Planting runs one oracle forward per tree level; each of them already fixes the argmax (and the
    margin) of every shallower node, so a planting whose walk meets a near-tie is abandoned at that
    level instead of at the end.  Returns (prefix, state after the prefill, tokens, oracle step result
    on a copy of the state, the copy, prefix stream, planting stream)."""
    for kp in range(prefix_tries):
        s = stream0 + STREAM_STEP * kp
        prefix = synth.prefix_tokens(om.d.vocab, P, seed=seed, stream=s)
        t0 = time.time()
        seq, logits = oracle_prefill(om, prefix)
        m = float(top2_margin(logits[-1]))
        log("prefill P=%d stream %d: %.0f s, last margin %.4f" % (P, s, time.time() - t0, m))
        if m <= DECISIVE:
            continue
        for kt in range(plant_tries):
            st = s + STREAM_STEP * kt
            t0 = time.time()

            def argmax_checked(tokens, parents):
                logits_t, _ = oracle_tree_logits(om, seq, tokens, parents)
                amax = np.argmax(logits_t, axis=1)
                marg = top2_margin(logits_t)
                path = _deciding_path(tokens, parents, amax)
                if np.min(marg[path]) <= DECISIVE:
                    raise Undecided("near-tie on the walk at %d nodes" % len(tokens))
                return amax

            try:
                toks = synth.plant_tree(shape, seq.pending, p, synth.plant_draws(shape.n, om.d.vocab, stream=st),
                                        argmax_checked)
                work = copy.copy(seq)
                work.k, work.v, work.tokens = list(seq.k), list(seq.v), list(seq.tokens)
                r = oracle_verify(om, work, toks, shape.parents)
            except Undecided as e:
                log("  tree n=%d plant stream %d: %.0f s, %s" % (shape.n, st, time.time() - t0, e))
                continue
            dec = [0] + list(r["accepted_nodes"])
            mmin = float(np.min(r["margin"][dec]))
            log("  tree n=%d plant stream %d: %.0f s, accepted %d, min deciding margin %.4f"
                % (shape.n, st, time.time() - t0, r["accepted_len"], mmin))
            if mmin > DECISIVE:
                return prefix, seq, toks, r, work, s, st
    raise RuntimeError("no decided step within %d prefixes" % prefix_tries)


def decided_tree_on(om, seq, shape, p, stream, tries=12):
    """As decided_case, for a fixed prefix state (the sweep's drafts share one prefix).  None when the
    root itself is a near-tie (no planting can help) or no planting stream is decided."""
    lg_root, _ = oracle_tree_logits(om, seq, [seq.pending], [-1])
    if float(top2_margin(lg_root)[0]) <= DECISIVE:
        log("  root near-tie: margin %.4f" % float(top2_margin(lg_root)[0]))
        return None
    for kt in range(tries):
        st = stream + STREAM_STEP * kt
        t0 = time.time()

        def argmax_checked(tokens, parents):
            logits_t, _ = oracle_tree_logits(om, seq, tokens, parents)
            amax = np.argmax(logits_t, axis=1)
            if np.min(top2_margin(logits_t)[_deciding_path(tokens, parents, amax)]) <= DECISIVE:
                raise Undecided("near-tie on the walk at %d nodes" % len(tokens))
            return amax

        try:
            toks = synth.plant_tree(shape, seq.pending, p, synth.plant_draws(shape.n, om.d.vocab, stream=st),
                                    argmax_checked)
            work = copy.copy(seq)
            work.k, work.v, work.tokens = list(seq.k), list(seq.v), list(seq.tokens)
            r = oracle_verify(om, work, toks, shape.parents)
        except Undecided as e:
            log("  tree n=%d plant stream %d: %.0f s, %s" % (shape.n, st, time.time() - t0, e))
            continue
        mmin = float(np.min(r["margin"][[0] + list(r["accepted_nodes"])]))
        log("  tree n=%d plant stream %d: %.0f s, accepted %d, min deciding margin %.4f"
            % (shape.n, st, time.time() - t0, r["accepted_len"], mmin))
        if mmin > DECISIVE:
            return toks, r, work, st
    return None


def step_record(pre, r, toks, parents, work, P, cols, kv_layers, pre_slots, rec):
    """Flatten one verified step into `rec` under keys prefixed by `pre`."""
    lg = r["logits"]
    n = lg.shape[0]
    ti, tv = top_k_rows(lg, TOPK_STORED)
    a = r["accepted_len"]
    rec[pre + "tokens"] = np.asarray(toks, np.int32)
    rec[pre + "parents"] = np.asarray(parents, np.int32)
    rec[pre + "argmax"] = np.asarray(r["argmax"], np.int32)
    rec[pre + "margin"] = np.asarray(r["margin"], np.float64)
    rec[pre + "topk_idx"] = ti.astype(np.int32)
    rec[pre + "topk_val"] = tv
    rec[pre + "logit_cols"] = lg[:, cols].astype(np.float32)
    rec[pre + "accepted_len"] = np.int32(a)
    rec[pre + "accepted_nodes"] = np.asarray(r["accepted_nodes"], np.int32)
    rec[pre + "accepted_tokens"] = np.asarray(r["accepted_tokens"], np.int32)
    rec[pre + "bonus"] = np.int32(r["bonus"])
    slots = np.arange(P, P + a + 1)
    rec[pre + "kv_layers"] = np.asarray(kv_layers, np.int32)
    rec[pre + "kv_k"] = np.stack([work.k[l][slots] for l in kv_layers]).astype(np.float32)
    rec[pre + "kv_v"] = np.stack([work.v[l][slots] for l in kv_layers]).astype(np.float32)
    if pre_slots is not None:
        ps = np.asarray(pre_slots, np.int64)
        rec[pre + "pre_slots"] = ps.astype(np.int32)
        rec[pre + "pre_k"] = np.stack([work.k[l][ps] for l in kv_layers]).astype(np.float32)
        rec[pre + "pre_v"] = np.stack([work.v[l][ps] for l in kv_layers]).astype(np.float32)
    assert n == len(toks)


def save(name, rec):
    np.savez_compressed(path(name), **rec)
    log("wrote %s (%.0f KB)" % (path(name), os.path.getsize(path(name)) / 1024))


def make_verify_p2048():
    dims = synth.LLAMA8B
    _, host, fp = target(dims)
    om = OracleModel(dims, host)
    shape = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=0)
    prefix, seq, toks, r, work, ps, st = decided_case(om, 2048, shape, 0.8, stream0=0)
    P = len(prefix)
    cols = sampled_columns(dims.vocab, N_COLS, 2048)
    L = dims.n_layers
    rec = {"fingerprint": np.array(fp), "P": np.int32(P), "prefix": prefix, "prefix_stream": np.int32(ps),
           "plant_stream": np.int32(st), "pending": np.int32(seq.pending), "cols": cols}
    step_record("", r, toks, shape.parents, work, P, cols, (0, L // 2, L - 1), (0, 1, P // 2, P - 1), rec)
    save("verify_p2048", rec)


def make_sweep_p8192():
    """One prefix for all six drafts: the first prefix stream on which every draft has a decided planting."""
    dims = synth.LLAMA8B
    _, host, fp = target(dims)
    om = OracleModel(dims, host)
    names = ["chain5", "chain8", "tree16", "tree32", "tree60", "tree80"]
    shapes = [synth.chain(5), synth.chain(8)] + [synth.tree_from_widths(synth.SWEEP_WIDTHS[n], stream=0)
                                                 for n in (16, 32, 60, 80)]
    L = dims.n_layers
    for kp in range(20):
        s = STREAM_STEP * kp
        prefix = synth.prefix_tokens(dims.vocab, 8192, seed=1, stream=s)
        t0 = time.time()
        seq, logits = oracle_prefill(om, prefix)
        m = float(top2_margin(logits[-1]))
        log("prefill P=8192 stream %d: %.0f s, last margin %.4f" % (s, time.time() - t0, m))
        if m <= DECISIVE:
            continue
        # the trees' deciding paths start along the greedy continuation: skip a prefix
        # whose first greedy tokens hold a near-tie (no planting of a wide tree avoids it)
        toks, par, near = [seq.pending], [-1], False
        for depth in range(3):
            lg, _ = oracle_tree_logits(om, seq, toks, par)
            if float(top2_margin(lg[-1:])[0]) <= DECISIVE:
                near = True
                break
            toks.append(int(np.argmax(lg[-1])))
            par.append(len(toks) - 2)
        if near:
            log("  greedy continuation near-tie at depth %d" % depth)
            continue
        P = len(prefix)
        cols = sampled_columns(dims.vocab, N_COLS, 8192)
        rec = {"fingerprint": np.array(fp), "P": np.int32(P), "prefix": prefix, "prefix_stream": np.int32(s),
               "pending": np.int32(seq.pending), "cols": cols}
        ok = True
        for i, (nm, sh) in enumerate(zip(names, shapes)):
            got = decided_tree_on(om, seq, sh, 0.85, stream=0)
            if got is None:
                ok = False
                break
            toks, r, work, st = got
            rec[nm + "_plant_stream"] = np.int32(st)
            step_record(nm + "_", r, toks, sh.parents, work, P, cols, (0, L - 1),
                        (0, P // 2 + 1, P - 1) if i == 0 else None, rec)
        if ok:
            rec["drafts"] = np.array(names)
            save("sweep_p8192", rec)
            return
    raise RuntimeError("no prefix with every draft decided")


def batch64_sample(lens):
    """The shortest and the longest prefix plus six seeded others: 8 of the 64 sequences."""
    lo, hi = int(np.argmin(lens)), int(np.argmax(lens))
    rest = [b for b in range(len(lens)) if b not in (lo, hi)]
    others = np.random.default_rng([4, 7]).choice(rest, size=6, replace=False)
    return sorted([lo, hi] + [int(b) for b in others])


def make_batch64():
    dims = synth.LLAMA8B
    _, host, fp = target(dims)
    om = OracleModel(dims, host)
    lens, pvals = synth.batch_prefix_lengths_and_p(64)
    sample = batch64_sample(lens)
    log("batch-64 sample %s, prefixes %s" % (sample, [int(lens[b]) for b in sample]))
    cols = sampled_columns(dims.vocab, N_COLS, 64)
    L = dims.n_layers
    rec = {"fingerprint": np.array(fp), "sample": np.asarray(sample, np.int32), "cols": cols,
           "lens": lens.astype(np.int32), "ps": pvals}
    for b in sample:
        sh = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=b)
        prefix, seq, toks, r, work, ps, st = decided_case(om, int(lens[b]), sh, float(pvals[b]), stream0=b)
        P = len(prefix)
        pre = "s%d_" % b
        rec[pre + "prefix"] = prefix
        rec[pre + "prefix_stream"] = np.int32(ps)
        rec[pre + "plant_stream"] = np.int32(st)
        rec[pre + "pending"] = np.int32(seq.pending)
        step_record(pre, r, toks, sh.parents, work, P, cols, (0, L - 1), (0, P - 1), rec)
    save("batch64", rec)


def draft_inputs(dims, B=16, P=2048):
    """Seeded inputs of the draft-head workload: per sequence a draft prefix of P feature rows with the
    token one step ahead per row, then one 60-draft tree per sequence with its node tokens and features."""
    prefix_feats = [synth.draft_features(P, dims.hidden, seed=100 + b) for b in range(B)]
    prefix_toks = [synth.prefix_tokens(dims.vocab, P, seed=1, stream=300 + b) for b in range(B)]
    shapes = [synth.tree_from_widths(synth.TREE60_WIDTHS, stream=b) for b in range(B)]
    node_toks = [synth.prefix_tokens(dims.vocab, sh.n, seed=1, stream=400 + b) for b, sh in enumerate(shapes)]
    M = sum(sh.n for sh in shapes)
    node_feats = synth.draft_features(M, dims.hidden, seed=5)
    return prefix_feats, prefix_toks, shapes, node_toks, node_feats


def make_draft_b16():
    dims = synth.LLAMA8B
    w, host, fp = target(dims)
    dw = synth.draft_head_weights(dims, seed=6, device="cpu")
    dfp = synth.weights_fingerprint(dw)
    dhost = {"fc_fuse": synth.tensor_to_host(dw["fc_fuse"]), "fc_in": synth.tensor_to_host(dw["fc_in"]),
             "final_norm": synth.tensor_to_host(dw["final_norm"]),
             "layer": {k: synth.tensor_to_host(v) for k, v in dw["layer"].items()}}
    head = OracleDraftHead(dims, host, dhost)
    B, P = 16, 2048
    pf, pt, shapes, nt, nf = draft_inputs(dims, B, P)
    nf_h = synth.tensor_to_host(nf)
    cols = sampled_columns(dims.vocab, 128, 16)
    rec = {"fingerprint": np.array(fp), "draft_fingerprint": np.array(dfp), "cols": cols, "B": np.int32(B),
           "P": np.int32(P)}
    off = np.zeros(B + 1, np.int64)
    off[1:] = np.cumsum([sh.n for sh in shapes])
    ti_all, tv_all, lc_all = [], [], []
    kv_seqs, kv_slots = (0, 15), (0, 1, P // 2, P - 1)
    for b in range(B):
        t0 = time.time()
        seq = head.prefill(synth.tensor_to_host(pf[b]), pt[b])
        lo, hi = int(off[b]), int(off[b + 1])
        logits = head.step_logits(seq, nf_h[lo:hi], nt[b], shapes[b].parents)
        ti, tv = top_k_rows(logits, 11)
        ti_all.append(ti.astype(np.int32))
        tv_all.append(tv)
        lc_all.append(logits[:, cols].astype(np.float32))
        if b in kv_seqs:
            rec["kv%d_k" % b] = seq.k[list(kv_slots)].astype(np.float32)
            rec["kv%d_v" % b] = seq.v[list(kv_slots)].astype(np.float32)
        log("draft sequence %d: %.0f s" % (b, time.time() - t0))
    rec["kv_seqs"] = np.asarray(kv_seqs, np.int32)
    rec["kv_slots"] = np.asarray(kv_slots, np.int32)
    rec["offsets"] = off.astype(np.int32)
    rec["node_tokens"] = np.concatenate(nt).astype(np.int32)
    rec["parents"] = np.concatenate([sh.parents for sh in shapes]).astype(np.int32)
    rec["top_idx"] = np.concatenate(ti_all)
    rec["top_val"] = np.concatenate(tv_all)
    rec["logit_cols"] = np.concatenate(lc_all)
    save("draft_b16", rec)


MAKERS = {"verify_p2048": make_verify_p2048, "sweep_p8192": make_sweep_p8192, "batch64": make_batch64,
          "draft_b16": make_draft_b16}


if __name__ == "__main__":
    if "MALLOC_MMAP_MAX_" not in os.environ:
        # The oracle decodes every weight matrix to float64 on each forward (1.75 GB per decoder
        # layer at the 8B shape).  glibc would map and unmap those arrays each time, and the page
        # faults cost more than the arithmetic: serve them from the heap and keep freed pages.
        env = dict(os.environ, MALLOC_MMAP_MAX_="0", MALLOC_TRIM_THRESHOLD_=str(1 << 40))
        os.execve(sys.executable, [sys.executable] + sys.argv, env)
    ap = argparse.ArgumentParser()
    ap.add_argument("which", nargs="*", default=["all"])
    a = ap.parse_args()
    todo = list(MAKERS) if "all" in a.which else a.which
    for nm in todo:
        t0 = time.time()
        log("== %s" % nm)
        MAKERS[nm]()
        log("== %s done in %.0f s" % (nm, time.time() - t0))
