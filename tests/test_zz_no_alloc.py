"""dsa_sparse_attn_noalloc (split-k partials in the library's fixed scratch array)
against dsa_sparse_attn (caller-provided workspace), through the C ABI.

Some callers cannot allocate device memory when they run attention: a serving
loop that handed all device memory to its own pool at start-up, or code that
must not risk the device-wide synchronisation that freeing memory brings.
dsa_sparse_attn_noalloc serves them with a fixed array inside the library.

Both entry points run the same kernels with the same split of each row over
the key tiles; only the address of the partials differs, so their results must
be identical bit for bit.  One case is also held against the fp64 oracle.

Collected last on purpose: it must give the same results whether it runs alone
or after every other test has used the device."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_19_b200 as dsa
import parity as P

DEV = "cuda"
H, D, DV = 128, 576, 512
SCALE = 192 ** -0.5
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _case(B, Lq, Lk, k, seed, pad_every=0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, H, D, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lk, D, generator=g).to(torch.bfloat16)
    idx = torch.stack([torch.randperm(Lk, generator=g)[:k].sort().values for _ in range(B * Lq)]).int()
    if pad_every:
        idx[::pad_every, k // 2:] = -1           # short rows: padding after the valid entries
    return q.to(DEV), kv.to(DEV), idx.reshape(B, Lq, k).to(DEV)


def _compare(q, kv, idx):
    ref_out, ref_lse = dsa.sparse_attn(q, kv, idx, DV, SCALE)
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    dsa.sparse_attn_noalloc(q, kv, idx, DV, SCALE, out, lse)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out), "output differs from dsa_sparse_attn"
    assert torch.equal(lse, ref_lse), "lse differs from dsa_sparse_attn"
    return out, lse


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # Few rows: every row is split over the 16 key tiles, so the scratch array is used.
    B, Lq, Lk, k = 4, 1, 8192, 2048
    need = dsa.workspace_size(dsa.OP_SPARSE_ATTN, B, Lq, Lk, k, H, DV)
    assert 0 < need <= dsa.NOALLOC_SCRATCH_BYTES
    q, kv, idx = _case(B, Lq, Lk, k, seed=1)
    first, first_lse = _compare(q, kv, idx)
    # the first call against the fp64 oracle as well
    rows = np.arange(B * Lq)
    oo, ol = oracle.sparse_attn(rows // Lq, P.bf16_bits(q).reshape(B * Lq, H, D), P.bf16_bits(kv),
                                idx.reshape(B * Lq, k).cpu().numpy(), SCALE, DV)
    P.check_attention(first.reshape(B * Lq, H, DV), first_lse.reshape(B * Lq, H), oo, ol)
    second, _ = _compare(*_case(B, Lq, Lk, k, seed=2, pad_every=3))
    # the second call really recomputed (different inputs, same scratch)
    assert not torch.equal(first, second)
    assert dsa.device_status() == 0


@pytest.mark.gpu
def test_noalloc_without_split_needs_no_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B, Lq, Lk, k = 1, 320, 1024, 256
    assert dsa.workspace_size(dsa.OP_SPARSE_ATTN, B, Lq, Lk, k, H, DV) == 0
    _compare(*_case(B, Lq, Lk, k, seed=3))
    assert dsa.device_status() == 0


def test_noalloc_rejects_calls_beyond_the_scratch_size():
    # The smallest number of single-query rows whose split-k partials exceed the
    # array, for the SM count this process sees (the workspace query reads it
    # from the device, or assumes 148 without one).  The call must refuse before
    # launching anything or reading any pointer: the pointers here are fake.
    rows = next(r for r in range(1, 4096)
                if dsa.workspace_size(dsa.OP_SPARSE_ATTN, r, 1, 131072, 2048, H, DV) > dsa.NOALLOC_SCRATCH_BYTES)
    L = dsa.lib()
    a = dsa.AttnArgs(H=H, d_qk=D, d_v=DV, scale=SCALE, q=16, kv=16)
    fake = ctypes.c_void_p(256)
    rc = L.dsa_sparse_attn_noalloc(ctypes.byref(a), rows, 1, 131072, fake, 2048, fake, None, None)
    assert rc == 3 and dsa.status_string(rc).startswith("DSA_ERR_WORKSPACE")


def test_binding_scratch_size_matches_the_header():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    m = re.search(r"#define\s+DSA_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", text)
    assert m, "DSA_NOALLOC_SCRATCH_BYTES not found in include/dsa.h"
    assert dsa.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
