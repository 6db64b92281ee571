"""Short-sequence mode of dsa_forward (q_offset + Lq <= k): every row selects all
of its positions 0..t, so the pass is dense causal MLA attention (the masked
dense form the V3.2 report page keeps for short sequences, section "Стоимость").
The attention kernel then reads keys 0..t as contiguous tiles and writes the
index lists itself; no indexer or top-k runs.

Held against the fp64 oracle, and against the gather path (dsa_sparse_attn over
explicit index lists 0..t), which runs the same arithmetic on the same rows and
must agree bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_19_b200 as dsa
from dsa_inputs import WORKLOADS, make_inputs
import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.lib()
    yield
    assert dsa.device_status() == 0


def _dense_case(wl, seed, rows):
    inp = make_inputs(wl, DEV, seed)
    idx, out, lse = dsa.forward(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], inp["q"],
                                inp["kv"], wl.k, wl.Dv, wl.scale, wl.q_offset)
    torch.cuda.synchronize()
    t = wl.q_offset + np.arange(wl.B * wl.Lq) % wl.Lq
    want = np.where(np.arange(wl.k)[None, :] <= t[:, None], np.arange(wl.k)[None, :], -1).astype(np.int32)
    assert np.array_equal(idx.reshape(-1, wl.k).cpu().numpy(), want)
    # the gather path over the same index lists: identical arithmetic, identical bits
    g_out, g_lse = dsa.sparse_attn(inp["q"], inp["kv"], idx, wl.Dv, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, g_out) and torch.equal(lse, g_lse)
    keys = oracle.keys_from_inputs(inp)
    r = oracle.rows_from_inputs(inp, rows, wl.Lq, wl.q_offset)
    oo, ol = oracle.sparse_attn(r["row_b"], r["q"], keys["kv"], want[rows], wl.scale, wl.Dv)
    sel = torch.as_tensor(rows, device=DEV)
    P.check_attention(out.reshape(-1, wl.H, wl.Dv)[sel], lse.reshape(-1, wl.H)[sel], oo, ol)


def test_dense_prefill_2k():
    wl = WORKLOADS["prefill_8k"].with_(Lq=2048, Lk=2048)
    _dense_case(wl, 0, np.r_[0, 1, 127, 128, 129, 1000, 2046, 2047])


def test_dense_chunk_with_offset_and_batches():
    # q_offset > 0, two sequences (keys of the next sequence follow in memory and
    # must be masked), ragged tail
    wl = WORKLOADS["prefill_8k"].with_(B=2, Lq=333, Lk=1500, q_offset=1167)
    _dense_case(wl, 1, np.r_[0, 1, 200, 332, 333, 500, 665])


def test_dense_few_rows_split_over_units():
    # four rows: each row's key tiles are split over several CTA pairs and merged
    wl = WORKLOADS["prefill_8k"].with_(Lq=4, Lk=2000, q_offset=1996)
    assert dsa.workspace_size(dsa.OP_SPARSE_ATTN, 1, 4, 2000, 2048, 128, 512) > 0
    _dense_case(wl, 2, np.arange(4))


def test_dense_tiny_shape_all_rows():
    wl = WORKLOADS["tiny"].with_(Lq=100, Lk=120, q_offset=20)
    _dense_case(wl, 3, np.arange(100))
