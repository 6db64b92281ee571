"""The indexer with the top-k fused into it (dsa_indexer_topk, the selection step
of dsa_forward) through the C ABI.

Its scores are the same fp32 values the scores-mode indexer writes, so its index
sets must equal dsa_topk over dsa_indexer_scores bit for bit, and its selected
scores must equal those scores at the selected positions.  The integer config
(exact scores, many ties) is held against the fp64 oracle directly.  Cases cover
rows split over several units (decode), rows shorter than k, chunk offsets,
all-equal scores (every later tie loses to the earlier positions) and +-0."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_19_b200 as dsa
from dsa_inputs import WORKLOADS, make_inputs, make_key_side, make_query_side
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


def _staged(inp, q_offset, k):
    scores = dsa.indexer_scores(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], q_offset)
    idx = dsa.topk(scores, k, q_offset)
    return scores, idx


def _fused(inp, q_offset, k):
    return dsa.indexer_topk(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], k, q_offset)


def _same_as_staged(inp, q_offset, k):
    scores, idx_s = _staged(inp, q_offset, k)
    idx_f, sel = _fused(inp, q_offset, k)
    torch.cuda.synchronize()
    assert torch.equal(idx_f, idx_s), "fused selection differs from dsa_topk over dsa_indexer_scores"
    valid = idx_f >= 0
    gathered = torch.gather(scores, 2, idx_f.clamp_min(0).long())
    assert torch.equal(sel[valid], gathered[valid]), "selected scores differ from the scores-mode values"
    assert torch.all(torch.isneginf(sel[~valid]))
    return idx_f, sel, scores


def test_fused_integer_config_matches_the_oracle_exactly():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, DEV, 0)
    idx, sel, _ = _same_as_staged(inp, 0, wl.k)
    r = oracle.rows_from_inputs(inp, np.arange(wl.Lq), wl.Lq, 0)
    keys = oracle.keys_from_inputs(inp)
    sc = oracle.indexer_scores(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"], keys["k_scale"])
    exp = oracle.topk(sc, r["row_t"], wl.k)
    assert np.array_equal(idx.reshape(-1, wl.k).cpu().numpy(), exp)
    got = sel.reshape(-1, wl.k).double().cpu().numpy()
    want = np.where(exp >= 0, np.take_along_axis(sc, np.maximum(exp, 0), axis=1), -np.inf)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("Lq,Lk,q_offset", [(8192, 8192, 0), (700, 700, 0), (1000, 5096, 4096)])
def test_fused_prefill_equals_staged(Lq, Lk, q_offset):
    wl = WORKLOADS["prefill_32k"].with_(Lq=Lq, Lk=Lk, q_offset=q_offset)
    keys = make_key_side(wl, DEV, 1)
    inp = dict(keys, **make_query_side(wl, DEV, 1))
    _same_as_staged(inp, q_offset, wl.k)


def test_fused_decode_rows_split_over_units_equal_staged():
    # few long rows: each row's key tiles are spread over several units, and the
    # last unit of a row selects over all of their candidate lists
    wl = WORKLOADS["decode_128k"].with_(B=6, Lk=40000, q_offset=39999)
    inp = make_inputs(wl, DEV, 2)
    _same_as_staged(inp, wl.q_offset, wl.k)


@pytest.mark.parametrize("Lq", [2, 3, 4])
def test_fused_few_query_blocks_equal_staged(Lq):
    # 2-4 new tokens per sequence: query blocks of two (the deep-ring sizes, whose
    # candidate lists and staging need the shorter key ring), three and four
    wl = WORKLOADS["decode_128k"].with_(B=3, Lq=Lq, Lk=9000, q_offset=9000 - Lq)
    inp = make_inputs(wl, DEV, 10 + Lq)
    _same_as_staged(inp, wl.q_offset, wl.k)


def test_fused_decode_full_size_sampled_against_the_oracle():
    wl = WORKLOADS["decode_128k"]
    inp = make_key_side(wl, DEV, 0)
    inp.update(make_query_side(wl, DEV, 0))
    idx, sel = _fused(inp, wl.q_offset, wl.k)
    torch.cuda.synchronize()
    rows = np.array([0, 21, 63])
    r = oracle.rows_from_inputs(inp, rows, 1, wl.q_offset)
    keys = oracle.keys_from_inputs(inp)
    sc = oracle.indexer_scores(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"], keys["k_scale"])
    gi = idx.reshape(-1, wl.k)[torch.as_tensor(rows, device=DEV)].cpu().numpy()
    P.check_index_sets(gi, sc, r["row_t"], wl.k)
    gs = sel.reshape(-1, wl.k)[torch.as_tensor(rows, device=DEV)].double().cpu().numpy()
    want = np.take_along_axis(sc, gi, axis=1)
    P.check_scores(gs, want, np.full(len(rows), wl.k - 1))


def test_fused_all_equal_scores_keep_the_first_positions():
    # q_I = 0: every score is exactly 0 (and -0 where a negative weight multiplies
    # it), so every row takes its first min(k, t+1) positions.
    wl = WORKLOADS["prefill_8k"].with_(Lq=600, Lk=5000, q_offset=4400)
    inp = make_inputs(wl, DEV, 3)
    inp["q_I"] = torch.zeros_like(inp["q_I"])
    idx, sel, _ = _same_as_staged(inp, wl.q_offset, wl.k)
    want = torch.arange(wl.k, device=DEV, dtype=torch.int32).expand(wl.Lq, -1)
    assert torch.equal(idx[0], want)
    assert torch.all(sel == 0)


def test_fused_rows_shorter_than_k_take_every_position():
    wl = WORKLOADS["prefill_8k"].with_(Lq=300, Lk=300)
    inp = make_inputs(wl, DEV, 4)
    idx, _, _ = _same_as_staged(inp, 0, wl.k)
    n = np.arange(wl.Lq) + 1
    want = np.where(np.arange(wl.k)[None, :] < n[:, None], np.arange(wl.k)[None, :], -1)
    assert np.array_equal(idx[0].cpu().numpy(), want)


def test_forward_selected_scores_feed_the_loss_like_the_full_matrix():
    wl = WORKLOADS["prefill_8k"].with_(Lq=2048, Lk=6144, q_offset=4096)
    inp = make_inputs(wl, DEV, 5)
    sel = torch.empty(wl.B, wl.Lq, wl.k, dtype=torch.float32, device=DEV)
    idx, out, lse = dsa.forward(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], inp["q"],
                                inp["kv"], wl.k, wl.Dv, wl.scale, wl.q_offset, sel_scores=sel)
    scores, idx_s = _staged(inp, wl.q_offset, wl.k)
    assert torch.equal(idx, idx_s)
    t_full, kl_full = dsa.indexer_kl_loss(inp["q"], inp["kv"], idx, lse, scores, wl.Dv, wl.scale)
    t_sel, kl_sel = dsa.indexer_kl_loss_selected(inp["q"], inp["kv"], idx, lse, sel, wl.Dv, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(kl_sel, kl_full)
    assert torch.equal(t_sel, t_full)
