"""The C-ABI library loads on a machine without a GPU, exports every entry point
include/dsa.h declares, and rejects bad arguments on the host before touching
CUDA.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import sparse_attention_19_b200 as dsa
from sparse_attention_19_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def L():
    dsa_build.build()
    return dsa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_attn", "dsa_forward", "dsa_workspace_size",
              "dsa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert isinstance(getattr(L, name), ctypes._CFuncPtr)


def test_status_strings(L):
    assert dsa.status_string(0) == "DSA_OK"
    for code in range(1, 6):
        assert dsa.status_string(code).startswith("DSA_ERR_")
    assert dsa.status_string(99) == "DSA_ERR_UNKNOWN"
    assert dsa.version() >= 100


def _idx_args(**kw):
    base = dict(B=1, Lq=8, Lk=8, q_offset=0, H_I=64, d_I=128, q_I=16, q_scale=None, w=16, k_I=16, k_scale=None)
    base.update(kw)
    return dsa.IndexerArgs(**base)


def test_indexer_rejects_bad_arguments_before_any_launch(L):
    out = ctypes.c_void_p(16)
    assert L.dsa_indexer_scores(None, out, None) == 1
    assert L.dsa_indexer_scores(ctypes.byref(_idx_args(q_I=None)), out, None) == 1
    assert L.dsa_indexer_scores(ctypes.byref(_idx_args(Lq=0)), out, None) == 1
    assert L.dsa_indexer_scores(ctypes.byref(_idx_args(q_offset=1)), out, None) == 1   # q_offset+Lq > Lk
    assert L.dsa_indexer_scores(ctypes.byref(_idx_args(q_I=8)), out, None) == 1        # misaligned
    assert L.dsa_indexer_scores(ctypes.byref(_idx_args(H_I=32)), out, None) == 2       # unsupported
    assert L.dsa_indexer_scores(ctypes.byref(_idx_args(d_I=96)), out, None) == 2
    assert L.dsa_indexer_scores(ctypes.byref(_idx_args()), None, None) == 1


def test_topk_rejects_bad_arguments(L):
    p = ctypes.c_void_p(16)
    assert L.dsa_topk(None, 1, 4, 4, 0, 2, p, None, 0, None) == 1
    assert L.dsa_topk(p, 1, 4, 4, 1, 2, p, None, 0, None) == 1                          # q_offset+Lq > Lk
    assert L.dsa_topk(p, 1, 4, 4, 0, 0, p, None, 0, None) == 2                          # k < 1
    assert L.dsa_topk(p, 1, 4, 4, 0, 4096, p, None, 0, None) == 2                       # k > 2048


def test_attention_rejects_bad_arguments(L):
    good = dsa.AttnArgs(128, 576, 512, 0.07, 16, 16)
    p = ctypes.c_void_p(16)
    assert L.dsa_sparse_attn(ctypes.byref(dsa.AttnArgs(128, 576, 512, 0.07, None, 16)), 1, 1, 8, p, 8, p, None,
                             None, 0, None) == 1
    assert L.dsa_sparse_attn(ctypes.byref(dsa.AttnArgs(64, 576, 512, 0.07, 16, 16)), 1, 1, 8, p, 8, p, None,
                             None, 0, None) == 2
    assert L.dsa_sparse_attn(ctypes.byref(dsa.AttnArgs(128, 576, 512, -1.0, 16, 16)), 1, 1, 8, p, 8, p, None,
                             None, 0, None) == 1
    assert L.dsa_sparse_attn(ctypes.byref(good), 1, 1, 8, p, 0, p, None, None, 0, None) == 2
    assert L.dsa_sparse_attn(ctypes.byref(good), 1, 1, 8, None, 8, p, None, None, 0, None) == 1


def test_forward_checks_the_workspace(L):
    ia = _idx_args(Lq=8, Lk=8)
    aa = dsa.AttnArgs(128, 576, 512, 0.07, 16, 16)
    p = ctypes.c_void_p(16)
    need = dsa.workspace_size(dsa.OP_FORWARD, 1, 8, 8, 8, 128, 512)
    assert need >= 8 * 8 * 4
    assert L.dsa_forward(ctypes.byref(ia), ctypes.byref(aa), 8, p, p, None, p, need - 1, None) == 3
    assert L.dsa_forward(ctypes.byref(ia), ctypes.byref(aa), 8, p, p, None, None, need, None) == 3


def test_workspace_sizes():
    assert dsa.workspace_size(dsa.OP_TOPK, 1, 8192, 8192, 2048, 128, 512) == 0
    # prefill: one query row per unit, no split-k partials
    assert dsa.workspace_size(dsa.OP_SPARSE_ATTN, 1, 8192, 8192, 2048, 128, 512) == 0
    # decode with few rows -> split-k partials (fp32 O + lse per split); 4 rows on
    # 74 CTA pairs are split 16 ways (one key tile per unit)
    ws = dsa.workspace_size(dsa.OP_SPARSE_ATTN, 4, 1, 131072, 2048, 128, 512)
    assert ws >= 4 * 16 * 128 * 512 * 4
    # 64 rows already occupy most pairs: whole rows per unit, no partials
    assert dsa.workspace_size(dsa.OP_SPARSE_ATTN, 64, 1, 131072, 2048, 128, 512) == 0
    # The staged forward keeps the fp32 score matrix in its workspace ...
    fwd = dsa.workspace_size(dsa.OP_FORWARD, 1, 4096, 131072, 2048, 128, 512)
    assert 4096 * 131072 * 4 <= fwd < 4096 * 131072 * 4 + (1 << 20)
    # ... the low-memory one selects on chip: candidate lists (at most 2k + 512
    # per row in flight), never the [Lq, Lk] score matrix.
    low = dsa.workspace_size(dsa.OP_FORWARD_LOWMEM, 1, 4096, 131072, 2048, 128, 512)
    assert 0 < low < 4096 * 131072 * 4 // 4
    low32 = dsa.workspace_size(dsa.OP_FORWARD_LOWMEM, 1, 32768, 32768, 2048, 128, 512)
    assert 0 < low32 < 32768 * 32768 * 4 // 16
    for op in (dsa.OP_FORWARD, dsa.OP_FORWARD_LOWMEM):
        assert dsa.workspace_size(op, 0, 1, 1, 1, 1, 1) == 0
    # the exact query agrees with the convention-based one when q_offset = Lk - Lq
    ia = _idx_args(B=64, Lq=1, Lk=131072, q_offset=131071)
    for op in (dsa.OP_FORWARD, dsa.OP_FORWARD_LOWMEM):
        assert dsa.workspace_size_args(op, ia, 2048, 128, 512) == \
            dsa.workspace_size(op, 64, 1, 131072, 2048, 128, 512)
    assert dsa.workspace_size_args(dsa.OP_INDEXER_TOPK, ia, 2048) == \
        dsa.workspace_size(dsa.OP_INDEXER_TOPK, 64, 1, 131072, 2048, 128, 512) > 0
    # invalid indexer arguments: no size
    assert dsa.workspace_size_args(dsa.OP_FORWARD, _idx_args(q_I=None), 2048, 128, 512) == 0


def test_indexer_topk_rejects_bad_arguments(L):
    p = ctypes.c_void_p(16)
    f = L.dsa_indexer_topk
    ia = _idx_args(Lq=8, Lk=8)
    need = dsa.workspace_size_args(dsa.OP_INDEXER_TOPK, ia, 8)
    assert need > 0
    assert f(None, 8, p, None, p, need, None) == 1
    assert f(ctypes.byref(_idx_args(q_I=None)), 8, p, None, p, need, None) == 1
    assert f(ctypes.byref(ia), 8, None, None, p, need, None) == 1                       # no indices
    assert f(ctypes.byref(ia), 8, p, ctypes.c_void_p(8), p, need, None) == 1            # misaligned scores
    assert f(ctypes.byref(ia), 0, p, None, p, need, None) == 2                          # k < 1
    assert f(ctypes.byref(ia), 4096, p, None, p, need, None) == 2                       # k > 2048
    assert f(ctypes.byref(_idx_args(H_I=32)), 8, p, None, p, need, None) == 2
    assert f(ctypes.byref(ia), 8, p, None, p, need - 1, None) == 3                      # workspace too small
    assert f(ctypes.byref(ia), 8, p, None, None, need, None) == 3


def test_indexer_kl_loss_selected_rejects_bad_arguments(L):
    good = dsa.AttnArgs(128, 576, 512, 0.07, 16, 16)
    p = ctypes.c_void_p(16)
    f = L.dsa_indexer_kl_loss_selected
    assert f(ctypes.byref(good), 1, 1, 8, p, 8, None, p, None, p, None) == 1           # no lse
    assert f(ctypes.byref(good), 1, 1, 8, p, 8, p, None, None, p, None) == 1           # no selected scores
    assert f(ctypes.byref(good), 1, 1, 8, p, 8, p, ctypes.c_void_p(8), None, p, None) == 1
    assert f(ctypes.byref(good), 1, 1, 8, p, 4096, p, p, None, p, None) == 2


def test_indexer_kl_loss_rejects_bad_arguments(L):
    good = dsa.AttnArgs(128, 576, 512, 0.07, 16, 16)
    p = ctypes.c_void_p(16)
    f = L.dsa_indexer_kl_loss
    assert f(ctypes.byref(good), 1, 1, 8, p, 8, None, p, None, p, None) == 1           # no lse
    assert f(ctypes.byref(good), 1, 1, 8, p, 8, p, None, None, p, None) == 1           # no scores
    assert f(ctypes.byref(good), 1, 1, 8, p, 8, p, p, None, None, None) == 1           # no kl
    assert f(ctypes.byref(good), 1, 1, 8, p, 8, p, p, ctypes.c_void_p(8), p, None) == 1   # misaligned target
    assert f(ctypes.byref(good), 1, 1, 8, p, 0, p, p, None, p, None) == 2              # k < 1
    assert f(ctypes.byref(good), 1, 1, 8, p, 4096, p, p, None, p, None) == 2           # k > 2048
    assert f(ctypes.byref(dsa.AttnArgs(64, 576, 512, 0.07, 16, 16)), 1, 1, 8, p, 8, p, p, None, p, None) == 2


def test_product_code_never_reaches_the_oracle():
    # The oracle is test infrastructure: the package (binding, build script, kernels,
    # C ABI) neither imports, loads nor includes anything from it.
    pkg = os.path.join(ROOT, "sparse_attention_19_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if not f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                continue
            text = open(os.path.join(dirpath, f)).read()
            assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
            assert "liboracle" not in text and "dsa_oracle" not in text, f
