"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/spec.h declares, sizes its buffers, and rejects bad
trees and configurations before touching the device."""

import ctypes
import os
import re

import numpy as np
import pytest

from speculative_decoding_06_b200 import spec as S
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "spec.h")).read()
    return re.findall(r"SPEC_API\s+[\w\s\*]+?\b(spec_\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    lib = S.lib()
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(names) == sorted(S.declared_symbols())


def cfg_of(d, max_batch=1, max_seq=512, max_nodes=64):
    return S.spec_config(n_layers=d.n_layers, hidden=d.hidden, n_q_heads=d.n_q_heads, n_kv_heads=d.n_kv_heads,
                         head_dim=d.head_dim, ffn=d.ffn, vocab=d.vocab,
                         dtype=S.SPEC_DTYPE_BF16 if d.dtype == "bf16" else S.SPEC_DTYPE_F32,
                         rms_eps=d.rms_eps, rope_theta=d.rope_theta, max_batch=max_batch, max_seq=max_seq,
                         max_nodes=max_nodes, draft_head=0)


def test_kv_bytes_matches_layout():
    d = synth.LLAMA8B
    c = cfg_of(d, max_batch=1, max_seq=4096, max_nodes=64)
    # [layer][K|V|K_lo][seq][kv head][slot][hd] fp16
    assert S.spec_kv_bytes(ctypes.byref(c)) == 32 * 3 * 1 * 8 * 4096 * 128 * 2
    cf = cfg_of(synth.TINY, max_batch=2, max_seq=512, max_nodes=16)
    # fp32 models: [layer][K|V][seq][kv head][slot][hd] fp32
    assert S.spec_kv_bytes(ctypes.byref(cf)) == 2 * 2 * 2 * 4 * 512 * 64 * 4
    ws = S.spec_workspace_bytes(ctypes.byref(c))
    assert 0 < ws < 512 << 20


@pytest.mark.parametrize("layers,ok", [((0, 0, 0), True), ((1, 1, 2), True), ((2, 1, 2), True),
                                       ((0, 1, 2), False), ((1, 3, 2), False), ((-1, 1, 1), False)])
def test_feature_layers_checked_and_sized(layers, ok):
    """feature_layers: all zero (no tap) or each in [1, n_layers]; a tap adds [3][Mpad][d] bf16 of workspace."""
    d = synth.MINI_BF16  # 2 layers
    base = S.spec_workspace_bytes(ctypes.byref(cfg_of(d, max_batch=2, max_nodes=64)))
    c = cfg_of(d, max_batch=2, max_nodes=64)
    c.feature_layers[:] = list(layers)
    ws = S.spec_workspace_bytes(ctypes.byref(c))
    if not ok:
        assert ws == 0 and S.spec_kv_bytes(ctypes.byref(c)) == 0
    elif layers == (0, 0, 0):
        assert ws == base
    else:
        assert ws >= base + 3 * 128 * d.hidden * 2  # Mpad = 128 for 2 x 64 nodes


@pytest.mark.parametrize("field,value", [
    ("n_kv_heads", 3), ("head_dim", 64), ("hidden", 4000), ("max_nodes", 129), ("max_nodes", 0), ("dtype", 7),
    ("ffn", 100), ("rope_theta", 0.5), ("draft_vocab", 1), ("draft_vocab", 100),
])
def test_bad_bf16_config_rejected(field, value):
    c = cfg_of(synth.MINI_BF16)
    setattr(c, field, value)
    assert S.spec_kv_bytes(ctypes.byref(c)) == 0
    assert S.spec_workspace_bytes(ctypes.byref(c)) == 0
    h = ctypes.c_void_p()
    w = S.spec_weights()
    assert S.spec_init(ctypes.byref(c), ctypes.byref(w), None, 0, None, 0, None, ctypes.byref(h)) == S.SPEC_ERR_ARG


def test_init_rejects_missing_buffers_without_gpu():
    c = cfg_of(synth.TINY)
    h = ctypes.c_void_p()
    w = S.spec_weights()
    assert S.spec_init(ctypes.byref(c), ctypes.byref(w), None, 0, None, 0, None, ctypes.byref(h)) == S.SPEC_ERR_ARG


def _validate(tokens, parents, vocab=100, max_nodes=64):
    t = np.asarray(tokens, np.int32)
    p = np.asarray(parents, np.int32)
    return S.spec_validate_tree(t.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                p.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(t), vocab, max_nodes)


def test_validate_tree():
    assert _validate([1, 2, 3], [-1, 0, 1]) == S.SPEC_OK
    assert _validate([1], [-1]) == S.SPEC_OK
    assert _validate([1, 2], [0, 0]) == S.SPEC_ERR_TREE          # root must have parent -1
    assert _validate([1, 2, 3], [-1, 2, 0]) == S.SPEC_ERR_TREE   # forward reference
    assert _validate([1, 2, 3], [-1, 0, 2]) == S.SPEC_ERR_TREE   # self loop
    assert _validate([1, 2], [-1, -1]) == S.SPEC_ERR_TREE        # two roots
    assert _validate([1, 200], [-1, 0]) == S.SPEC_ERR_TOKEN
    assert _validate([1, -4], [-1, 0]) == S.SPEC_ERR_TOKEN
    assert _validate(list(range(65)), [-1] + list(range(64))) == S.SPEC_ERR_CAPACITY
    assert _validate([], []) == S.SPEC_ERR_CAPACITY


def test_new_entry_points_reject_bad_arguments_without_gpu():
    """NULL handles and buffers are refused before any CUDA call."""
    i32 = ctypes.c_int32(0)
    assert S.spec_draft_tree(None, 1, None, None, None, 8, 10, 60, None, None, None) == S.SPEC_ERR_ARG
    assert S.spec_prefill_features(None, 0, None, 1, None, None) == S.SPEC_ERR_ARG
    assert S.spec_draft_append(None, 0, None, None, 1) == S.SPEC_ERR_ARG
    assert S.spec_set_feature_out(None, None, 0) == S.SPEC_ERR_ARG
    assert S.spec_wait_selftest(None, 1000, ctypes.byref(i32)) == S.SPEC_ERR_ARG
    assert S.spec_wait_selftest(ctypes.c_void_p(16), 0, ctypes.byref(i32)) == S.SPEC_ERR_ARG
    assert S.spec_wait_selftest(ctypes.c_void_p(18), 1000, ctypes.byref(i32)) == S.SPEC_ERR_ARG  # misaligned


def test_draft_head_workspace_holds_no_logits():
    """The draft head's top-10 is selected inside the LM-head GEMM: at batch 16 x 64 nodes the
    workspace holds per-tile candidates (24 slots x 1002 tiles per row), not [1024][128256]
    fp32 logits (525 MB)."""
    c = cfg_of(synth.LLAMA8B, max_batch=16, max_seq=2112, max_nodes=64)
    base = S.spec_workspace_bytes(ctypes.byref(c))
    c.draft_head = 1
    with_draft = S.spec_workspace_bytes(ctypes.byref(c))
    assert 0 < base < with_draft
    assert with_draft - base < 1024 * 128256 * 4


def test_sampling_setter_without_handle():
    assert S.spec_set_sampling(None, 0.7, 1) == S.SPEC_ERR_ARG
