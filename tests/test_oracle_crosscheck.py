"""C oracle vs the independent numpy restatement on generator inputs (CPU)."""
import numpy as np
import pytest

import oracle
from dsa_inputs import WORKLOADS, make_inputs, make_key_side, make_query_side

import np_restatement as npr


def _compare(wl, inp, rows, tol_scores=1e-12):
    r = oracle.rows_from_inputs(inp, rows, wl.Lq, wl.q_offset)
    keys = oracle.keys_from_inputs(inp)
    res = oracle.dsa_forward(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"],
                             keys["k_scale"], r["q"], keys["kv"], wl.k, wl.scale, wl.Dv,
                             want_scores=True)
    I = npr.indexer(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"], keys["k_scale"])
    fin = np.isfinite(I)
    assert np.array_equal(fin, np.isfinite(res["scores"]))
    np.testing.assert_allclose(res["scores"][fin], I[fin], rtol=tol_scores,
                               atol=tol_scores * np.abs(I[fin]).max())
    idx = npr.topk(res["scores"], r["row_t"], wl.k)      # same scores -> same decision
    assert np.array_equal(idx, res["indices"])
    out, lse = npr.attention(r["row_b"], r["q"], keys["kv"], res["indices"], wl.scale, wl.Dv)
    np.testing.assert_allclose(res["out"], out, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse, rtol=1e-12, atol=1e-12)
    return res


def test_crosscheck_tiny_config_rows():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, "cpu", seed=0)
    rows = np.array([0, 1, 2, 126, 127, 128, 129, 500, 1022, 1023])
    res = _compare(wl, inp, rows, tol_scores=0.0)
    # integer config: exact scores
    fin = np.isfinite(res["scores"])
    assert np.all(res["scores"][fin] == np.round(res["scores"][fin]))


def test_crosscheck_random_fp8_shapes_small():
    # prefill-like distributions (per-token scales, N(0,1/8) weights, salient keys)
    # at a size numpy handles quickly
    wl = WORKLOADS["prefill_32k"].with_(Lq=300, Lk=300, k=64, H=8, D=128, Dv=64, H_I=16, d_I=64)
    inp = make_inputs(wl, "cpu", seed=1)
    rows = np.array([0, 10, 63, 64, 65, 200, 299])
    _compare(wl, inp, rows)


def test_crosscheck_decode_like_batches():
    wl = WORKLOADS["decode_128k"].with_(B=3, Lk=500, q_offset=499, k=64, H=4, D=128, Dv=64,
                                        H_I=8, d_I=64)
    inp = make_key_side(wl, "cpu", 2)
    inp.update(make_query_side(wl, "cpu", 2))
    _compare(wl, inp, np.arange(3))
