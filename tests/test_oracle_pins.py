"""Pins for the fp64 CPU oracle, against facts that do not come from the oracle.

Each test ties one part of the oracle to something independent of it: a value
worked out by hand, a library routine that a special case reduces to, brute
force over tiny inputs, or an identity that a plausible mistake (a dropped
ReLU, a flipped sign, a transposed index, a wrong tie-break) would break.

Equations pinned (DeepSeek-V3.2 technical-report summary, section
"DSA: внимание только к важному"):
  indexer   I[t,s] = sum_j w[t,j] ReLU(q_I[t,j] . k_I[s])      ("Молниеносный индексатор")
  selection u_t = Attn(h_t, {c_s : I[t,s] in Top-k(I[t,:])})    ("Отбор и основное внимание")
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def e4m3_codes(values):
    return torch.tensor(values, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def bf16_bits(values):
    return torch.tensor(values, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- number formats

def test_e4m3_every_code_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2  # S.1111.111 for both signs; e4m3 has no infinity
    assert np.array_equal(ref[~nan], got[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(got[~nan]))


def test_e4m3_format_landmarks():
    assert oracle.e4m3_value(0x38) == 1.0          # exponent field 7 = bias
    assert oracle.e4m3_value(0x7E) == 448.0        # largest finite
    assert oracle.e4m3_value(0x08) == 2.0 ** -6    # smallest normal
    assert oracle.e4m3_value(0x01) == 2.0 ** -9    # smallest subnormal
    assert oracle.e4m3_value(0xB8) == -1.0
    assert math.copysign(1.0, oracle.e4m3_value(0x80)) == -1.0


def test_bf16_landmarks():
    assert oracle.bf16_value(0x3F80) == 1.0
    assert oracle.bf16_value(0xC000) == -2.0
    assert oracle.bf16_value(0x3E00) == 0.125
    assert oracle.bf16_value(0x7F7F) == float(torch.tensor(3.3895e38).to(torch.bfloat16))


# ---------------------------------------------------------------- indexer

def test_indexer_hand_worked_case():
    g = json.load(open(os.path.join(GOLD, "indexer_hand.json")))
    k_I = e4m3_codes(g["k_values"])[None]                 # [1, 2 keys, 2]
    q_I = e4m3_codes(g["q_values"])                       # [2 rows, 2 heads, 2]
    got = oracle.indexer_scores(
        row_b=[0, 0], row_t=g["row_t"], q_I=q_I,
        q_scale=np.array(g["q_scale"], np.float32), w=bf16_bits(g["w"]),
        k_I=k_I, k_scale=np.array([g["k_scale"]], np.float32))
    exp = np.array([[float(x) for x in row] for row in g["expected"]])
    assert np.array_equal(got, exp)


def _rand_int_inputs(rng, n_rows, Lk, H_I, d_I, lo=-4, hi=4):
    q = rng.integers(lo, hi + 1, size=(n_rows, H_I, d_I))
    k = rng.integers(lo, hi + 1, size=(1, Lk, d_I))
    return q, k


def test_indexer_one_head_unit_weight_is_relu_of_matmul():
    # H_I = 1, w = 1: I = sq*sk*ReLU(q8 . k8), a masked ReLU of a plain matrix product.
    rng = np.random.default_rng(1)
    n, Lk, d = 7, 11, 16
    q, k = _rand_int_inputs(rng, n, Lk, 1, d)
    sq = rng.uniform(0.25, 4.0, n).astype(np.float32)
    sk = rng.uniform(0.25, 4.0, (1, Lk)).astype(np.float32)
    t = np.array([0, 1, 3, 5, 8, 10, 10])
    got = oracle.indexer_scores(np.zeros(n, np.int64), t, e4m3_codes(q), sq, bf16_bits(np.ones((n, 1))),
                                e4m3_codes(k), sk)
    dots = np.matmul(q[:, 0, :].astype(np.float64) * sq[:, None].astype(np.float64),
                     (k[0].astype(np.float64) * sk[0][:, None].astype(np.float64)).T)
    exp = np.maximum(dots, 0.0)
    exp[np.arange(Lk)[None, :] > t[:, None]] = -np.inf
    np.testing.assert_allclose(got, exp, rtol=1e-15, atol=0)


def test_indexer_relu_identities_against_matmul():
    # Negating every query (flip the e4m3 sign bit) gives
    #   I(q) - I(-q) = sum_j w_j (q_j . k)   (linear: a matrix product)
    #   I(q) + I(-q) = sum_j w_j |q_j . k|
    # A dropped ReLU, a ReLU on the wrong side of w, or a wrong sign fails one of them.
    rng = np.random.default_rng(2)
    n, Lk, H_I, d = 5, 9, 3, 8
    q, k = _rand_int_inputs(rng, n, Lk, H_I, d)
    w = rng.integers(-2, 3, size=(n, H_I)).astype(np.float64)
    t = np.full(n, Lk - 1)
    qc = e4m3_codes(q)
    plus = oracle.indexer_scores(np.zeros(n, np.int64), t, qc, None, bf16_bits(w), e4m3_codes(k), None)
    minus = oracle.indexer_scores(np.zeros(n, np.int64), t, qc ^ 0x80, None, bf16_bits(w), e4m3_codes(k), None)
    x = np.einsum("rjd,sd->rjs", q.astype(np.float64), k[0].astype(np.float64))
    lin = np.einsum("rj,rjs->rs", w, x)
    mag = np.einsum("rj,rjs->rs", w, np.abs(x))
    assert np.array_equal(plus - minus, lin)
    assert np.array_equal(plus + minus, mag)
    # and the two halves are separately exact: ReLU(x) = (x + |x|) / 2
    assert np.array_equal(plus, (lin + mag) / 2)


def test_indexer_causal_mask_follows_position_not_row():
    rng = np.random.default_rng(3)
    q, k = _rand_int_inputs(rng, 3, 6, 2, 4, lo=1, hi=3)   # all dots positive
    t = np.array([4, 0, 2])
    got = oracle.indexer_scores(np.zeros(3, np.int64), t, e4m3_codes(q), None,
                                bf16_bits(np.ones((3, 2))), e4m3_codes(k), None)
    assert np.all(np.isneginf(got) == (np.arange(6)[None, :] > t[:, None]))
    assert np.all(got[np.isfinite(got)] > 0)


def test_indexer_batches_use_their_own_keys():
    rng = np.random.default_rng(4)
    q, _ = _rand_int_inputs(rng, 2, 5, 1, 4, lo=1, hi=2)
    k = rng.integers(1, 3, size=(2, 5, 4))
    got = oracle.indexer_scores(np.array([1, 0]), np.array([4, 4]), e4m3_codes(q), None,
                                bf16_bits(np.ones((2, 1))), e4m3_codes(k), None)
    exp0 = np.maximum(q[0, 0] @ k[1].T, 0)
    exp1 = np.maximum(q[1, 0] @ k[0].T, 0)
    assert np.array_equal(got[0], exp0) and np.array_equal(got[1], exp1)


def test_indexer_integer_config_is_exact_in_fp32():
    # Small integers in e4m3 and integer w: every partial sum is an integer far
    # below 2^24, so an fp32 evaluation in any order equals the fp64 oracle.
    from dsa_inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny"].with_(Lq=96, Lk=96)
    inp = make_inputs(wl, "cpu", seed=0)
    rows = np.arange(96)
    r = oracle.rows_from_inputs(inp, rows, wl.Lq, wl.q_offset)
    keys = oracle.keys_from_inputs(inp)
    got = oracle.indexer_scores(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"],
                                keys["k_I"], keys["k_scale"])
    qf = inp["q_I"].view(torch.float8_e4m3fn).float()[0]          # [Lq, H_I, d_I]
    kf = inp["k_I"].view(torch.float8_e4m3fn).float()[0]          # [Lk, d_I]
    wf = inp["w"].float()[0]
    x32 = torch.einsum("ijd,sd->ijs", qf, kf)
    i32 = torch.einsum("ij,ijs->is", wf, torch.relu(x32)).double().numpy()
    mask = np.arange(96)[None, :] > np.arange(96)[:, None]
    i32[mask] = -np.inf
    assert np.array_equal(got, i32)
    assert np.all(got[np.isfinite(got)] == np.round(got[np.isfinite(got)]))


# ---------------------------------------------------------------- top-k

def _brute_force_topk(v, t, k):
    """The unique subset S of [0, t] of size min(k, t+1) such that every member
    is >= every non-member, and on equal values members have smaller positions."""
    n = t + 1
    m = min(k, n)
    found = []
    for S in itertools.combinations(range(n), m):
        Sset = set(S)
        ok = True
        for a in S:
            for b in range(n):
                if b in Sset:
                    continue
                if v[a] < v[b] or (v[a] == v[b] and a > b):
                    ok = False
                    break
            if not ok:
                break
        if ok:
            found.append(S)
    assert len(found) == 1
    return list(found[0])


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(5)
    for trial in range(200):
        Lk = int(rng.integers(1, 9))
        t = int(rng.integers(0, Lk))
        k = int(rng.integers(1, 6))
        v = rng.integers(-3, 4, size=Lk).astype(np.float64)   # many ties
        got = oracle.topk(v[None, :], np.array([t]), k)[0]
        exp = _brute_force_topk(v, t, k)
        m = len(exp)
        assert list(got[:m]) == exp
        assert np.all(got[m:] == -1)


def test_topk_matches_stable_descending_sort():
    rng = np.random.default_rng(6)
    n, Lk, k = 40, 300, 17
    sc = np.round(rng.normal(size=(n, Lk)), 1)              # rounding forces ties
    t = rng.integers(0, Lk, size=n)
    got = oracle.topk(sc, t, k)
    for r in range(n):
        m = min(k, t[r] + 1)
        order = np.argsort(-sc[r, : t[r] + 1], kind="stable")[:m]
        assert list(got[r, :m]) == sorted(order.tolist())
        assert np.all(got[r, m:] == -1)


def test_topk_invariants_and_short_rows():
    rng = np.random.default_rng(7)
    Lk, k = 64, 16
    sc = rng.normal(size=(Lk, Lk))
    t = np.arange(Lk)
    got = oracle.topk(sc, t, k)
    for r in range(Lk):
        m = min(k, r + 1)
        sel = got[r, :m]
        assert len(set(sel.tolist())) == m
        assert np.all(sel >= 0) and np.all(sel <= r)
        assert np.all(np.diff(sel) > 0)
        assert np.all(got[r, m:] == -1)
        if r + 1 <= k:
            assert list(sel) == list(range(r + 1))


def test_topk_all_equal_scores_pick_the_first_k():
    got = oracle.topk(np.full((1, 50), 3.5), np.array([49]), 10)
    assert list(got[0]) == list(range(10))


def test_topk_negative_zero_equals_positive_zero():
    v = np.array([-0.0, 0.0, -0.0, 0.0, -1.0, -2.0])
    got = oracle.topk(v[None, :], np.array([5]), 3)
    assert list(got[0]) == [0, 1, 2]


def test_topk_ignores_positions_after_t():
    v = np.array([1.0, 2.0, 3.0, 100.0, 200.0])
    got = oracle.topk(v[None, :], np.array([2]), 2)
    assert list(got[0]) == [1, 2]


# ---------------------------------------------------------------- attention

def _bf16_rand(shape, rng, scale=1.0):
    x = torch.from_numpy(rng.normal(size=shape) * scale).to(torch.bfloat16)
    return x, x.view(torch.int16).numpy().view(np.uint16)


def test_attention_all_keys_selected_equals_dense_causal_sdpa():
    # k >= t+1: the selected set is every s <= t, so the result is ordinary
    # causal MQA attention; torch's scaled_dot_product_attention in fp64 computes it.
    rng = np.random.default_rng(8)
    L, H, D, Dv, k = 23, 4, 64, 32, 32
    scale = 1.0 / math.sqrt(192.0)
    q_t, q_b = _bf16_rand((L, H, D), rng)
    kv_t, kv_b = _bf16_rand((1, L, D), rng)
    idx = np.full((L, k), -1, np.int32)
    for t in range(L):
        idx[t, : t + 1] = rng.permutation(t + 1)
    out, lse = oracle.sparse_attn(np.zeros(L, np.int64), q_b, kv_b, idx, scale, Dv)
    qd = q_t.double().permute(1, 0, 2)[None]                 # [1, H, L, D]
    kd = kv_t.double()[0][None, None].expand(1, H, L, D)
    vd = kv_t.double()[0, :, :Dv][None, None].expand(1, H, L, Dv)
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=scale)
    ref = ref[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    logits = torch.einsum("lhd,sd->lhs", q_t.double(), kv_t.double()[0]) * scale
    logits = logits.masked_fill(torch.arange(L)[None, None, :] > torch.arange(L)[:, None, None], -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_single_selected_key_returns_its_value_row():
    rng = np.random.default_rng(9)
    H, D, Dv, k = 3, 64, 32, 8
    q_t, q_b = _bf16_rand((1, H, D), rng)
    kv_t, kv_b = _bf16_rand((1, 10, D), rng)
    idx = np.full((1, k), -1, np.int32)
    idx[0, 5] = 7
    out, lse = oracle.sparse_attn(np.zeros(1, np.int64), q_b, kv_b, idx, 0.3, Dv)
    for h in range(H):
        assert np.array_equal(out[0, h], kv_t[0, 7, :Dv].double().numpy())
        z = 0.3 * float((q_t[0, h].double() * kv_t[0, 7].double()).sum())
        assert lse[0, h] == pytest.approx(z, rel=1e-14, abs=1e-14)


def test_attention_zero_query_is_the_mean_of_selected_values():
    rng = np.random.default_rng(10)
    H, D, Dv, k = 2, 64, 32, 6
    q_b = np.zeros((1, H, D), np.uint16)
    kv_t, kv_b = _bf16_rand((1, 20, D), rng)
    sel = [3, 11, 0, 19]
    idx = np.array([sel + [-1, -1]], np.int32)
    out, lse = oracle.sparse_attn(np.zeros(1, np.int64), q_b, kv_b, idx, 0.5, Dv)
    mean = kv_t[0, sel, :Dv].double().mean(0).numpy()
    np.testing.assert_allclose(out[0, 0], mean, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse[0], math.log(4.0), rtol=1e-14)


def test_attention_is_independent_of_index_order_and_padding_slots():
    rng = np.random.default_rng(11)
    H, D, Dv, k = 4, 64, 32, 12
    q_t, q_b = _bf16_rand((1, H, D), rng)
    kv_t, kv_b = _bf16_rand((1, 30, D), rng)
    sel = rng.choice(30, size=9, replace=False)
    a = np.full((1, k), -1, np.int32); a[0, :9] = sel
    b = np.full((1, k), -1, np.int32); b[0, [0, 2, 3, 5, 6, 7, 9, 10, 11]] = sel[::-1]
    oa, la = oracle.sparse_attn(np.zeros(1, np.int64), q_b, kv_b, a, 0.2, Dv)
    ob, lb = oracle.sparse_attn(np.zeros(1, np.int64), q_b, kv_b, b, 0.2, Dv)
    np.testing.assert_allclose(oa, ob, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(la, lb, rtol=1e-13)


def test_attention_scores_use_the_whole_row_values_only_the_leading_dv():
    # K is the full D-wide latent row (latent + rope); V is its first Dv columns.
    rng = np.random.default_rng(12)
    H, D, Dv = 2, 64, 32
    q_t, q_b = _bf16_rand((1, H, D), rng)
    kv_t, kv_b = _bf16_rand((1, 4, D), rng)
    idx = np.array([[0, 1, 2, 3]], np.int32)
    base, _ = oracle.sparse_attn(np.zeros(1, np.int64), q_b, kv_b, idx, 0.5, Dv)
    kv2 = kv_t.clone(); kv2[0, 1, Dv:] += 3.0                   # only the rope part changes
    o2, _ = oracle.sparse_attn(np.zeros(1, np.int64), q_b, kv2.view(torch.int16).numpy().view(np.uint16),
                               idx, 0.5, Dv)
    assert not np.allclose(base, o2)                            # it moved the softmax weights...
    qd, kd = q_t.double()[0], kv2.double()[0]
    p = torch.softmax(0.5 * qd @ kd.T, -1)
    np.testing.assert_allclose(o2[0], (p @ kd[:, :Dv]).numpy(), rtol=1e-12, atol=1e-14)  # ...but V is kv[:, :Dv]


# ---------------------------------------------------------------- whole forward

def test_forward_with_k_at_least_L_is_dense_causal_attention():
    from dsa_inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny"].with_(Lq=48, Lk=48, H=4, k=64)
    inp = make_inputs(wl, "cpu", seed=3)
    rows = np.arange(48)
    r = oracle.rows_from_inputs(inp, rows, wl.Lq, wl.q_offset)
    keys = oracle.keys_from_inputs(inp)
    res = oracle.dsa_forward(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"],
                             keys["k_scale"], r["q"], keys["kv"], wl.k, wl.scale, wl.Dv)
    qd = inp["q"].double()[0].permute(1, 0, 2)[None]
    kd = inp["kv"].double()[0][None, None].expand(1, wl.H, 48, wl.D)
    vd = inp["kv"].double()[0, :, : wl.Dv][None, None].expand(1, wl.H, 48, wl.Dv)
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=wl.scale)
    np.testing.assert_allclose(res["out"], ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)
    for t in range(48):
        assert list(res["indices"][t, : t + 1]) == list(range(t + 1))


def test_forward_is_indexer_then_topk_then_attention():
    from dsa_inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny"].with_(Lq=200, Lk=200, k=32)
    inp = make_inputs(wl, "cpu", seed=4)
    rows = np.array([0, 5, 31, 32, 33, 150, 199])
    r = oracle.rows_from_inputs(inp, rows, wl.Lq, wl.q_offset)
    keys = oracle.keys_from_inputs(inp)
    res = oracle.dsa_forward(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"],
                             keys["k_scale"], r["q"], keys["kv"], wl.k, wl.scale, wl.Dv,
                             want_scores=True)
    sc = oracle.indexer_scores(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"],
                               keys["k_I"], keys["k_scale"])
    idx = oracle.topk(sc, r["row_t"], wl.k)
    out, lse = oracle.sparse_attn(r["row_b"], r["q"], keys["kv"], idx, wl.scale, wl.Dv)
    assert np.array_equal(res["scores"], sc)
    assert np.array_equal(res["indices"], idx)
    assert np.array_equal(res["out"], out) and np.array_equal(res["lse"], lse)


def test_work_ratio_matches_the_page_exercise():
    # The page's exercise: L = 128000, k = 2048 -> L*k / L^2 = 0.016.  The
    # selected-pair count used for FLOP accounting reduces to L*k - k(k-1)/2.
    from dsa_inputs import WORKLOADS
    wl = WORKLOADS["prefill_128k"].with_(Lq=128000, Lk=128000)
    assert wl.selected_pairs == 128000 * 2048 - 2048 * 2047 // 2
    assert wl.selected_pairs / 128000 ** 2 == pytest.approx(0.016, rel=0.01)
    assert wl.causal_pairs == 128000 * 128001 // 2


# ---------------------------------------------------------------- indexer training loss
# Section "Как учили индексатор": target p = main-attention probabilities summed over
# the heads, L1-normalised; loss = D_KL(p || softmax(I)) over the selected positions.

def _num(x):
    return math.log(2.0) if x == "ln2" else float(x)


def test_kl_hand_worked_case():
    g = json.load(open(os.path.join(GOLD, "indexer_kl_hand.json")))
    q = bf16_bits(g["q"])
    kv = bf16_bits(g["kv"])
    scores = np.array([[_num(v) for v in row] for row in g["scores"]])
    target, kl = oracle.indexer_kl(np.array(g["row_b"]), q, kv, np.array(g["indices"], np.int32), scores,
                                   _num(g["scale"]))
    want_t = np.array([[a / b for a, b in row] for row in g["target_fractions"]])
    np.testing.assert_allclose(target, want_t, rtol=1e-14, atol=1e-16)
    want_kl = [sum((pn / pd) * math.log((pn / pd) / (qn / qd)) for pn, pd, qn, qd in row)
               for row in g["kl_terms_p_q"]]
    np.testing.assert_allclose(kl, want_kl, rtol=1e-13)
    # the reversed divergence D_KL(softmax(I) || p) differs, so the direction is pinned
    rev = sum((qn / qd) * math.log((qn / qd) / (pn / pd)) for pn, pd, qn, qd in g["kl_terms_p_q"][0])
    assert abs(kl[0] - rev) > 1e-3


def _kl_case(rng, n=3, H=4, D=64, Lk=40, k=16, B=2):
    q_t, q_b = _bf16_rand((n, H, D), rng)
    kv_t, kv_b = _bf16_rand((B, Lk, D), rng)
    row_b = rng.integers(0, B, size=n)
    idx = np.full((n, k), -1, np.int32)
    for r in range(n):
        m = int(rng.integers(1, k + 1))
        slots = rng.choice(k, size=m, replace=False)
        idx[r, slots] = rng.choice(Lk, size=m, replace=False)
    scores = rng.normal(size=(n, Lk)) * 3.0
    return q_t, q_b, kv_t, kv_b, row_b, idx, scores


def test_kl_matches_library_softmax_and_entropy():
    # target through torch.softmax per head; KL through scipy.stats.entropy(p, q),
    # which computes sum p log(p/q) for two distributions.
    from scipy.special import softmax
    from scipy.stats import entropy
    rng = np.random.default_rng(40)
    q_t, q_b, kv_t, kv_b, row_b, idx, scores = _kl_case(rng)
    scale = 1.0 / math.sqrt(192.0)
    target, kl = oracle.indexer_kl(row_b, q_b, kv_b, idx, scores, scale)
    for r in range(len(row_b)):
        valid = idx[r] >= 0
        pos = idx[r][valid]
        keys = kv_t[row_b[r]].double()[torch.as_tensor(pos)]                 # [m, D]
        logits = torch.einsum("hd,md->hm", q_t[r].double(), keys) * scale
        p = torch.softmax(logits, dim=-1).sum(0)
        p = (p / p.sum()).numpy()
        np.testing.assert_allclose(target[r][valid], p, rtol=1e-12, atol=1e-15)
        assert np.all(target[r][~valid] == 0.0)
        qdist = softmax(scores[r][pos])
        assert kl[r] == pytest.approx(entropy(p, qdist), rel=1e-11, abs=1e-14)


def test_kl_is_zero_exactly_when_the_indexer_reproduces_the_target():
    rng = np.random.default_rng(41)
    q_t, q_b, kv_t, kv_b, row_b, idx, scores = _kl_case(rng)
    target, kl = oracle.indexer_kl(row_b, q_b, kv_b, idx, scores, 0.2)
    nv = (idx >= 0).sum(1)
    assert np.all(kl[nv > 1] > 0.0) and np.all(kl[nv == 1] == 0.0)      # Gibbs: > 0 unless equal
    matched = scores.copy()
    for r in range(len(row_b)):
        valid = idx[r] >= 0
        matched[r, idx[r][valid]] = np.log(target[r][valid]) + 3.7        # softmax(log p + c) = p
    _, kl0 = oracle.indexer_kl(row_b, q_b, kv_b, idx, matched, 0.2)
    np.testing.assert_allclose(kl0, 0.0, atol=1e-13)


def test_kl_ignores_score_shifts_and_everything_unselected():
    rng = np.random.default_rng(42)
    q_t, q_b, kv_t, kv_b, row_b, idx, scores = _kl_case(rng)
    t0, kl0 = oracle.indexer_kl(row_b, q_b, kv_b, idx, scores, 0.3)
    _, kl1 = oracle.indexer_kl(row_b, q_b, kv_b, idx, scores - 11.5, 0.3)
    np.testing.assert_allclose(kl1, kl0, rtol=1e-12)
    sc2, kv2 = scores.copy(), kv_b.copy()
    for r in range(len(row_b)):
        unsel = np.setdiff1d(np.arange(scores.shape[1]), idx[r][idx[r] >= 0])
        sc2[r, unsel] = rng.normal(size=len(unsel)) * 50.0
    used = {(int(row_b[r]), int(s)) for r in range(len(row_b)) for s in idx[r] if s >= 0}
    for b in range(kv_b.shape[0]):
        for s in range(kv_b.shape[1]):
            if (b, s) not in used:
                kv2[b, s] = bf16_bits(rng.normal(size=kv_b.shape[2]) * 4.0)
    t2, kl2 = oracle.indexer_kl(row_b, q_b, kv2, idx, sc2, 0.3)
    np.testing.assert_array_equal(t2, t0)
    np.testing.assert_array_equal(kl2, kl0)


def test_kl_follows_slot_order_and_padding():
    rng = np.random.default_rng(43)
    q_t, q_b, kv_t, kv_b, row_b, idx, scores = _kl_case(rng, n=1)
    t0, kl0 = oracle.indexer_kl(row_b, q_b, kv_b, idx, scores, 0.25)
    perm = rng.permutation(idx.shape[1])
    t1, kl1 = oracle.indexer_kl(row_b, q_b, kv_b, idx[:, perm], scores, 0.25)
    np.testing.assert_allclose(t1, t0[:, perm], rtol=1e-13, atol=1e-16)
    assert kl1[0] == pytest.approx(kl0[0], rel=1e-12)


def test_kl_degenerate_selections():
    rng = np.random.default_rng(44)
    q_t, q_b, kv_t, kv_b, row_b, idx, scores = _kl_case(rng, n=2)
    one = np.full_like(idx, -1)
    one[0, 5] = 7                                                        # a single selected position
    target, kl = oracle.indexer_kl(row_b, q_b, kv_b, one, scores, 0.25)
    assert target[0, 5] == 1.0 and np.count_nonzero(target[0]) == 1 and kl[0] == 0.0
    assert np.all(target[1] == 0.0) and kl[1] == 0.0                      # nothing selected
