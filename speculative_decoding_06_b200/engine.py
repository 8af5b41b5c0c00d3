"""Convenience wrapper over the C ABI: device memory from torch, numpy in and out.

Only marshalling happens here: buffers are allocated with torch (device memory
and the stream are PyTorch's), arguments are packed into the C structs, and
every computation is a call into libspec.so.
"""

from __future__ import annotations

import ctypes
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

from . import spec as S

_LAYER_KEYS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "attn_norm", "mlp_norm")


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _fptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def pack_trees(trees: Sequence[Tuple[Sequence[int], Sequence[int]]]):
    """[(tokens, parents), ...] -> concatenated tokens, parents and node offsets."""
    toks = [_i32(t) for t, _ in trees]
    pars = [_i32(p) for _, p in trees]
    off = np.zeros(len(trees) + 1, np.int32)
    off[1:] = np.cumsum([len(t) for t in toks])
    return np.concatenate(toks), np.concatenate(pars), off


class SpecEngine:
    """One handle of the library over caller-owned (torch) device buffers."""

    def __init__(self, dims, weights: Dict, max_batch: int, max_seq: int, max_nodes: int = 128,
                 stream: Optional[torch.cuda.Stream] = None, draft: Optional[Dict] = None,
                 feature_layers: Optional[Sequence[int]] = None):
        """feature_layers: (low, mid, high) layer counts whose residual streams a
        verification step can return for the draft head (see verify_batch).
        draft: the draft head's weights; with "vocab_ids" (int32 device tensor, ascending
        token ids) and "lm_head" (bf16 [len(vocab_ids)][d]: the target's rows of those ids)
        it scores a reduced vocabulary."""
        self.dims = dims
        self.cfg = S.spec_config(
            n_layers=dims.n_layers, hidden=dims.hidden, n_q_heads=dims.n_q_heads, n_kv_heads=dims.n_kv_heads,
            head_dim=dims.head_dim, ffn=dims.ffn, vocab=dims.vocab,
            dtype=S.SPEC_DTYPE_BF16 if dims.dtype == "bf16" else S.SPEC_DTYPE_F32,
            rms_eps=dims.rms_eps, rope_theta=dims.rope_theta, max_batch=max_batch, max_seq=max_seq,
            max_nodes=max_nodes, draft_head=1 if draft is not None else 0,
            draft_vocab=int(draft["vocab_ids"].numel()) if draft is not None and "vocab_ids" in draft else 0)
        self.draft_vocab = self.cfg.draft_vocab or dims.vocab
        if feature_layers is not None:
            self.cfg.feature_layers[:] = [int(j) for j in feature_layers]
        self._feat = None
        self.max_nodes = max_nodes
        self.max_batch = max_batch
        kvb = S.spec_kv_bytes(ctypes.byref(self.cfg))
        wsb = S.spec_workspace_bytes(ctypes.byref(self.cfg))
        if kvb == 0 or wsb == 0:
            raise S.SpecError(S.SPEC_ERR_ARG, "configuration rejected")
        self.kv = torch.empty(kvb, dtype=torch.uint8, device="cuda")
        self.ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        self._weights = weights  # keep the tensors alive
        self._layers = (S.spec_layer_weights * dims.n_layers)()
        for l, lw in enumerate(weights["layers"]):
            for k in _LAYER_KEYS:
                setattr(self._layers[l], k, lw[k].data_ptr())
        self._w = S.spec_weights(embed=weights["embed"].data_ptr(), final_norm=weights["final_norm"].data_ptr(),
                                 lm_head=weights["lm_head"].data_ptr(), layers=self._layers)
        self._draft = draft
        if draft is not None:
            self._dlayer = S.spec_layer_weights()
            for k in _LAYER_KEYS:
                setattr(self._dlayer, k, draft["layer"][k].data_ptr())
            self._w.draft_fc_fuse = draft["fc_fuse"].data_ptr()
            self._w.draft_fc_in = draft["fc_in"].data_ptr()
            self._w.draft_layer = ctypes.pointer(self._dlayer)
            self._w.draft_final_norm = draft["final_norm"].data_ptr()
            if "vocab_ids" in draft:
                self._w.draft_lm_head = draft["lm_head"].data_ptr()
                self._w.draft_vocab_ids = draft["vocab_ids"].data_ptr()
        # a dedicated stream: the legacy default stream cannot be captured into graphs
        self.stream = stream or torch.cuda.Stream()
        torch.cuda.synchronize()  # weights and buffers were written on torch's stream
        h = ctypes.c_void_p()
        rc = S.spec_init(ctypes.byref(self.cfg), ctypes.byref(self._w), self.kv.data_ptr(), kvb,
                         self.ws.data_ptr(), wsb, ctypes.c_void_p(self.stream.cuda_stream), ctypes.byref(h))
        if rc != S.SPEC_OK:
            raise S.SpecError(rc, "spec_init failed")
        self.h = h
        self._dbg = None

    # ------------------------------------------------------------------ helpers
    def _check(self, rc):
        if rc != S.SPEC_OK:
            raise S.SpecError(rc, S.spec_last_error(self.h).decode())

    def close(self):
        if getattr(self, "h", None):
            S.spec_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ calls
    def prefill(self, seq: int, tokens) -> int:
        t = _i32(tokens)
        pend = np.zeros(1, np.int32)
        self._check(S.spec_prefill(self.h, seq, _ptr(t), len(t), _ptr(pend)))
        return int(pend[0])

    def prefill_features(self, seq: int, tokens):
        """Prefill that also returns the draft-head features of every prompt position,
        a bf16 device tensor [n][3][hidden] (needs feature_layers)."""
        t = _i32(tokens)
        feats = torch.empty(len(t), 3, self.dims.hidden, dtype=torch.bfloat16, device="cuda")
        pend = np.zeros(1, np.int32)
        self.stream.wait_stream(torch.cuda.current_stream())
        self._check(S.spec_prefill_features(self.h, seq, _ptr(t), len(t), _ptr(pend), feats.data_ptr()))
        return int(pend[0]), feats

    def verify(self, seq: int, tokens, parents):
        t, p = _i32(tokens), _i32(parents)
        acc_len = np.zeros(1, np.int32)
        acc_tok = np.zeros(max(1, len(t)), np.int32)
        bonus = np.zeros(1, np.int32)
        self._check(S.spec_verify_tree(self.h, seq, _ptr(t), _ptr(p), len(t), _ptr(acc_len), _ptr(acc_tok),
                                       _ptr(bonus)))
        a = int(acc_len[0])
        return a, [int(x) for x in acc_tok[:a]], int(bonus[0])

    def verify_batch(self, seq_ids, trees, flags: int = 0, features: bool = False):
        """Host outputs: (accepted_len[B], accepted_nodes[B][max_nodes], accepted_tokens, bonus[B]);
        with `features`, also the draft-head features of each emitted path as a bf16 device
        tensor [B][max_nodes][3][hidden] (rows 0 .. accepted_len[b] valid)."""
        tok, par, off = pack_trees(trees)
        ids = _i32(seq_ids)
        B = len(ids)
        acc_len = np.zeros(B, np.int32)
        acc_nodes = np.zeros((B, self.max_nodes), np.int32)
        acc_tok = np.zeros((B, self.max_nodes), np.int32)
        bonus = np.zeros(B, np.int32)
        if features:
            self.feature_buffer()
            flags |= S.SPEC_FEATURES
        self._check(S.spec_verify_tree_batch(self.h, B, _ptr(ids), _ptr(tok), _ptr(par), _ptr(off),
                                             acc_len.ctypes.data, acc_nodes.ctypes.data, acc_tok.ctypes.data,
                                             bonus.ctypes.data, flags & ~S.SPEC_DEVICE_OUTPUTS))
        if features:
            return acc_len, acc_nodes, acc_tok, bonus, self._feat[:B]
        return acc_len, acc_nodes, acc_tok, bonus

    def feature_buffer(self) -> torch.Tensor:
        """The SPEC_FEATURES destination, bf16 [max_batch][max_nodes][3][hidden] (allocated once)."""
        if self._feat is None:
            self._feat = torch.zeros(self.max_batch, self.max_nodes, 3, self.dims.hidden, dtype=torch.bfloat16,
                                     device="cuda")
            self._check(S.spec_set_feature_out(self.h, self._feat.data_ptr(), self._feat.numel() * 2))
        return self._feat

    def verify_batch_device(self, ids: np.ndarray, tok: np.ndarray, par: np.ndarray, off: np.ndarray,
                            outputs: Optional[Tuple[torch.Tensor, ...]] = None, flags: int = 0):
        """Queue a step without synchronising; outputs (if given) are int32 device tensors."""
        ptrs = [None] * 4 if outputs is None else [o.data_ptr() if o is not None else None for o in outputs]
        if outputs is not None:
            self.stream.wait_stream(torch.cuda.current_stream())
        self._check(S.spec_verify_tree_batch(self.h, len(ids), _ptr(ids), _ptr(tok), _ptr(par), _ptr(off),
                                             ptrs[0], ptrs[1], ptrs[2], ptrs[3], flags | S.SPEC_DEVICE_OUTPUTS))

    def score(self, seq_ids, trees, flags: int = 0):
        tok, par, off = pack_trees(trees)
        ids = _i32(seq_ids)
        M = int(off[-1])
        if flags & S.SPEC_DEBUG_LOGITS and (self._dbg is None or self._dbg.numel() < M * self.dims.vocab):
            self.enable_debug_logits(self.max_batch * self.max_nodes)
        amax = np.zeros(M, np.int32)
        t1 = np.zeros(M, np.float32)
        t2 = np.zeros(M, np.float32)
        self._check(S.spec_score_trees(self.h, len(ids), _ptr(ids), _ptr(tok), _ptr(par), _ptr(off), _ptr(amax),
                                       _fptr(t1), _fptr(t2), flags))
        return amax, t1, t2, off

    def set_sampling(self, temperature: float, seed: int = 0):
        """Temperature sampling (T > 0) or greedy choices (T = 0) for later calls (spec_set_sampling)."""
        self._check(S.spec_set_sampling(self.h, float(temperature), int(seed)))

    def enable_debug_logits(self, rows: int):
        self._dbg = torch.empty(rows * self.dims.vocab, dtype=torch.float32, device="cuda")
        self._check(S.spec_set_debug_logits(self.h, self._dbg.data_ptr(), self._dbg.numel() * 4))
        return self._dbg

    def debug_logits(self, rows: int, width: Optional[int] = None) -> np.ndarray:
        """The SPEC_DEBUG_LOGITS rows [rows][width] (width: the vocabulary, or the draft vocabulary
        after a draft step)."""
        torch.cuda.synchronize()
        w = width or self.dims.vocab
        return self._dbg[: rows * w].view(rows, w).cpu().numpy()

    def truncate(self, seq: int, new_len: int):
        self._check(S.spec_truncate(self.h, seq, new_len))

    def seq_len(self, seq: int):
        ln = np.zeros(1, np.int32)
        pd = np.zeros(1, np.int32)
        self._check(S.spec_seq_len(self.h, seq, _ptr(ln), _ptr(pd)))
        return int(ln[0]), int(pd[0])

    def profile(self, enable: bool):
        self._check(S.spec_profile(self.h, 1 if enable else 0))

    def profile_read(self):
        ms = (ctypes.c_double * len(S.PROF_CLASSES))()
        n = (ctypes.c_int64 * len(S.PROF_CLASSES))()
        self._check(S.spec_profile_read(self.h, ms, n))
        return {k: (ms[i], n[i]) for i, k in enumerate(S.PROF_CLASSES)}

    def info(self, B: int, n_nodes: int, prefix: int) -> str:
        buf = ctypes.create_string_buffer(4096)
        self._check(S.spec_info(self.h, B, n_nodes, prefix, buf, 4096))
        return buf.value.decode()

    def step_launches(self) -> int:
        return int(S.spec_step_launches(self.h))

    def io_bytes(self):
        a, b = ctypes.c_size_t(), ctypes.c_size_t()
        self._check(S.spec_io_bytes(self.h, ctypes.byref(a), ctypes.byref(b)))
        return int(a.value), int(b.value)

    def sync(self):
        self._check(S.spec_sync(self.h))

    # ------------------------------------------------------------------ draft head
    def draft_prefill(self, seq: int, feats: torch.Tensor, tokens):
        """feats: bf16 device tensor [n][3][d]; tokens: the token one step ahead per row."""
        t = _i32(tokens)
        f = feats.contiguous()
        self.stream.wait_stream(torch.cuda.current_stream())
        self._check(S.spec_draft_prefill(self.h, seq, f.data_ptr(), _ptr(t), len(t)))

    def draft_append(self, seq: int, feats: torch.Tensor, tokens):
        """Extend the draft prefix by rows of features [n][3][d] and their next tokens."""
        t = _i32(tokens)
        f = feats.contiguous()
        self.stream.wait_stream(torch.cuda.current_stream())
        self._check(S.spec_draft_append(self.h, seq, f.data_ptr(), _ptr(t), len(t)))

    def speculative_decode(self, seq: int, prompt, n_new: int, steps: int = 8, topk: int = 10, total: int = 60):
        """Greedy EAGLE-3 decoding of one sequence (see speculative_decode_batch)."""
        emitted, accepted = self.speculative_decode_batch([seq], [prompt], n_new, steps, topk, total)
        return emitted[0], accepted[0]

    def speculative_decode_batch(self, seq_ids, prompts, n_new: int, steps: int = 8, topk: int = 10,
                                 total: int = 60):
        """Greedy EAGLE-3 decoding of several sequences at once, through the library.

        Prefill each prompt with features; a sequence's draft prefix holds one row per
        position but the last: row p is the fused features of position p with the
        embedding of token p + 1.  Each decoding step drafts one tree per sequence
        (rooted at its pending token, from the features of its last verified position),
        verifies the batch (returning the features of each root and its accepted nodes)
        and appends to every draft prefix the rows the step verified.  Sequences that
        have emitted n_new + 1 tokens drop out of later steps.  Returns (emitted tokens
        per sequence, accepted draft tokens per step per sequence); the first emitted
        token of a sequence is its prefill's pending token."""
        ids = [int(s) for s in seq_ids]
        pend, last, emitted, accepted = {}, {}, {}, {}
        for s, prompt in zip(ids, prompts):
            p = _i32(prompt)
            T = len(p)
            if T < 2:
                raise ValueError("every prompt needs at least two tokens")
            pend[s], feats = self.prefill_features(s, p)
            self.draft_prefill(s, feats[:T - 1], p[1:])
            last[s] = feats[T - 1:T].clone()
            emitted[s], accepted[s] = [pend[s]], []
        live = [s for s in ids if len(emitted[s]) < n_new + 1]
        while live:
            root_feats = torch.cat([last[s] for s in live], dim=0)
            tok, par, _ = self.draft_tree(live, root_feats, [pend[s] for s in live], steps=steps, topk=topk,
                                          total=total)
            acc_len, _, acc_tok, bonus, F = self.verify_batch(live, [(tok[b], par[b]) for b in range(len(live))],
                                                              features=True)
            for b, s in enumerate(live):
                a = int(acc_len[b])
                acc = [int(x) for x in acc_tok[b, :a]]
                self.draft_append(s, torch.cat([last[s], F[b, :a]], dim=0), [pend[s]] + acc)
                last[s] = F[b, a:a + 1].clone()
                pend[s] = int(bonus[b])
                emitted[s] += acc + [pend[s]]
                accepted[s].append(a)
            live = [s for s in live if len(emitted[s]) < n_new + 1]
        return [emitted[s] for s in ids], [accepted[s] for s in ids]

    def draft_step(self, seq_ids, feats: torch.Tensor, trees, flags: int = 0):
        """Host outputs top_idx [nodes][10] int32, top_val [nodes][10] fp32, node offsets."""
        tok, par, off = pack_trees(trees)
        ids = _i32(seq_ids)
        M = int(off[-1])
        if flags & S.SPEC_DEBUG_LOGITS and (self._dbg is None or self._dbg.numel() < M * self.dims.vocab):
            self.enable_debug_logits(self.max_batch * self.max_nodes)
        ti = np.zeros((M, S.SPEC_DRAFT_TOPK), np.int32)
        tv = np.zeros((M, S.SPEC_DRAFT_TOPK), np.float32)
        f = feats.contiguous()
        self.stream.wait_stream(torch.cuda.current_stream())
        self._check(S.spec_draft_step(self.h, len(ids), _ptr(ids), f.data_ptr(), _ptr(tok), _ptr(par), _ptr(off),
                                      ti.ctypes.data, tv.ctypes.data, flags & ~S.SPEC_DEVICE_OUTPUTS))
        return ti, tv, off

    def draft_step_device(self, ids, feats: torch.Tensor, tok, par, off, outputs=None, flags: int = 0):
        """Queue a draft step without synchronising (outputs: optional int32 / fp32 device tensors)."""
        ptrs = [None, None] if outputs is None else [o.data_ptr() if o is not None else None for o in outputs]
        self._check(S.spec_draft_step(self.h, len(ids), _ptr(ids), feats.data_ptr(), _ptr(tok), _ptr(par),
                                      _ptr(off), ptrs[0], ptrs[1], flags | S.SPEC_DEVICE_OUTPUTS))

    def draft_tree(self, seq_ids, root_feats: torch.Tensor, root_tokens, steps: int = 8, topk: int = 10,
                   total: int = 60):
        """Dynamic draft tree per sequence: (tokens [B][total+1], parents [B][total+1], values)."""
        ids = _i32(seq_ids)
        B = len(ids)
        rt = _i32(root_tokens)
        tok = np.zeros((B, total + 1), np.int32)
        par = np.zeros((B, total + 1), np.int32)
        val = np.zeros((B, total + 1), np.float32)
        f = root_feats.contiguous()
        self.stream.wait_stream(torch.cuda.current_stream())
        self._check(S.spec_draft_tree(self.h, B, _ptr(ids), f.data_ptr(), _ptr(rt), steps, topk, total,
                                      _ptr(tok), _ptr(par), _fptr(val)))
        return tok, par, val

    def draft_len(self, seq: int) -> int:
        ln = np.zeros(1, np.int32)
        self._check(S.spec_draft_len(self.h, seq, _ptr(ln)))
        return int(ln[0])

    def kv_view(self) -> torch.Tensor:
        """The cache as a tensor [layer][plane][max_batch][Hkv][max_seq][hd]: planes K, V (fp32 models) or
        K, V, K_lo in fp16 (bf16 models; the key is K + K_lo)."""
        d = self.dims
        tdt = torch.float16 if d.dtype == "bf16" else torch.float32
        planes = 3 if d.dtype == "bf16" else 2
        layers = d.n_layers + (1 if self._draft is not None else 0)  # the draft head's layer comes last
        return self.kv.view(tdt).view(layers, planes, self.max_batch, d.n_kv_heads, -1, d.head_dim)
