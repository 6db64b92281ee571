"""dsa_sparse_attn_noalloc (split-k partials in the library's fixed scratch array)
against dsa_sparse_attn (caller-provided workspace), through the C ABI.

Collected last on purpose: it must give the same results whether it runs alone
or after every other test has used the device."""
import ctypes

import pytest
import torch

import sparse_attention_19_b200 as dsa
import parity as P

DEV = "cuda"
H, D, DV = 128, 576, 512
SCALE = 192 ** -0.5


def _case(B, Lq, Lk, k, seed, pad_every=0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, H, D, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lk, D, generator=g).to(torch.bfloat16)
    idx = torch.stack([torch.randperm(Lk, generator=g)[:k].sort().values for _ in range(B * Lq)]).int()
    if pad_every:
        idx[::pad_every, k // 2:] = -1           # short rows: padding after the valid entries
    return q.to(DEV), kv.to(DEV), idx.reshape(B, Lq, k).to(DEV)


def _compare(q, kv, idx):
    B, Lq, _, _ = q.shape
    ref_out, ref_lse = dsa.sparse_attn(q, kv, idx, DV, SCALE)
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    dsa.sparse_attn_noalloc(q, kv, idx, DV, SCALE, out, lse)
    torch.cuda.synchronize()
    P.check_attention(out, lse, ref_out.float().cpu().numpy(), ref_lse.cpu().numpy())
    return out, ref_out


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # Few rows: every row is split over the 16 key tiles, so the scratch array is used.
    B, Lq, Lk, k = 4, 1, 8192, 2048
    need = dsa.workspace_size(dsa.OP_SPARSE_ATTN, B, Lq, Lk, k, H, DV)
    assert 0 < need <= dsa.NOALLOC_SCRATCH_BYTES
    first = _compare(*_case(B, Lq, Lk, k, seed=1))
    second = _compare(*_case(B, Lq, Lk, k, seed=2, pad_every=3))
    # the second call really recomputed (different inputs, same scratch)
    assert not torch.equal(first[0], second[0])
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
    # 160 single-query rows are split two ways (on 148 SMs): ~80 MiB of partials >
    # 64 MiB.  The call must refuse on the host before touching CUDA (the pointers
    # are never used).
    L = dsa.lib()
    a = dsa.AttnArgs(H=H, d_qk=D, d_v=DV, scale=SCALE, q=16, kv=16)
    fake = ctypes.c_void_p(256)
    assert dsa.workspace_size(dsa.OP_SPARSE_ATTN, 160, 1, 131072, 2048, H, DV) > dsa.NOALLOC_SCRATCH_BYTES
    rc = L.dsa_sparse_attn_noalloc(ctypes.byref(a), 160, 1, 131072, fake, 2048, fake, None, None)
    assert rc == 3 and dsa.status_string(rc).startswith("DSA_ERR_WORKSPACE")
