"""CUDA path vs the fp64 oracle, through the C ABI, on seeded synthetic inputs.

Stage tests feed each entry point inputs whose oracle answer is known (oracle
scores into dsa_topk, oracle index sets into dsa_sparse_attn), so every stage is
judged on its own; forward tests run the whole pass at the workload sizes and
compare sampled rows."""
import math

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


def to_dev(d):
    return {k: v.to(DEV) for k, v in d.items()}


# ------------------------------------------------------------------ indexer

def _indexer_case(wl, seed, rows=None):
    inp = to_dev(make_inputs(wl, "cpu", seed))
    scores = dsa.indexer_scores(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], wl.q_offset)
    torch.cuda.synchronize()
    n = wl.B * wl.Lq
    rows = np.arange(n) if rows is None else np.asarray(rows)
    r = oracle.rows_from_inputs(inp, rows, wl.Lq, wl.q_offset)
    keys = oracle.keys_from_inputs(inp)
    ora = oracle.indexer_scores(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"], keys["k_scale"])
    gpu = scores.reshape(n, wl.Lk)[torch.as_tensor(rows, device=DEV)].double().cpu().numpy()
    return gpu, ora, r


def test_indexer_integer_config_is_exact():
    wl = WORKLOADS["tiny"]
    gpu, ora, r = _indexer_case(wl, 0)
    assert np.array_equal(np.isneginf(gpu), np.isneginf(ora))     # -inf exactly above the diagonal
    fin = np.isfinite(ora)
    assert np.array_equal(gpu[fin], ora[fin])


def test_indexer_fp8_scaled_ragged_sizes():
    # prefill distributions (per-token scales, salient keys), sizes off every tile multiple
    wl = WORKLOADS["prefill_32k"].with_(Lq=700, Lk=700)
    rows = np.r_[0:9, 120:136, 300:310, 690:700]
    gpu, ora, r = _indexer_case(wl, 1, rows)
    assert np.all(np.isneginf(gpu[np.isneginf(ora)]))
    P.check_scores(gpu, ora, r["row_t"])


def test_indexer_query_offset_chunk():
    wl = WORKLOADS["prefill_8k"].with_(Lq=200, Lk=1000, q_offset=800)
    rows = np.r_[0:5, 97:103, 195:200]
    gpu, ora, r = _indexer_case(wl, 2, rows)
    P.check_scores(gpu, ora, r["row_t"])


def test_indexer_decode_batches_split_keys():
    wl = WORKLOADS["decode_128k"].with_(B=3, Lk=20001, q_offset=20000)
    gpu, ora, r = _indexer_case(wl, 3)
    P.check_scores(gpu, ora, r["row_t"])


@pytest.mark.parametrize("Lq", [2, 3, 4])
def test_indexer_few_query_blocks_generic_builds(Lq):
    # 2-4 new tokens per sequence (speculative or multi-token decode): query blocks
    # the specialised prefill (4 x 2) and decode (1 x 1) builds do not take -- the
    # deep-ring build with two queries per block, and the generic prefill build with
    # one sub-block of three or four queries.
    wl = WORKLOADS["decode_128k"].with_(B=2, Lq=Lq, Lk=5003, q_offset=5003 - Lq)
    gpu, ora, r = _indexer_case(wl, 40 + Lq)
    P.check_scores(gpu, ora, r["row_t"])


# ------------------------------------------------------------------ top-k

def _topk_case(scores_f32, q_offset, k, exact=True):
    """scores_f32: torch fp32 [B, Lq, Lk] on the device."""
    B, Lq, Lk = scores_f32.shape
    idx = dsa.topk(scores_f32, k, q_offset)
    torch.cuda.synchronize()
    sc = scores_f32.double().cpu().numpy().reshape(B * Lq, Lk)
    row_t = q_offset + np.arange(B * Lq) % Lq
    exp = oracle.topk(sc, row_t, k)
    got = idx.cpu().numpy().reshape(B * Lq, k)
    assert np.array_equal(got, exp)
    return got


def test_topk_on_oracle_scores_integer_config():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, "cpu", 0)
    r = oracle.rows_from_inputs(inp, np.arange(wl.Lq), wl.Lq, 0)
    keys = oracle.keys_from_inputs(inp)
    sc = oracle.indexer_scores(r["row_b"], r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"], keys["k_scale"])
    s32 = torch.from_numpy(sc.astype(np.float32)).reshape(1, wl.Lq, wl.Lk).to(DEV)
    _topk_case(s32, 0, wl.k)


def test_topk_rounded_scores_with_ties_and_offset():
    g = torch.Generator().manual_seed(11)
    s = torch.round(torch.randn(2, 37, 5000, generator=g) * 10) / 10        # heavy ties
    _topk_case(s.to(DEV), 4963, 2048)


def test_topk_long_rows_streamed_from_global():
    g = torch.Generator().manual_seed(12)
    s = torch.randn(2, 1, 140000, generator=g)
    s[0, 0, 1000:1100] = 0.0
    s[0, 0, 1100:1200] = -0.0
    _topk_case(s.to(DEV), 139999, 2048)


def test_topk_edge_cases():
    # all-equal rows select the first k positions; +-0 are equal; short rows take everything
    s = torch.full((1, 4, 3000), 2.5)
    s[0, 1] = 0.0
    s[0, 1, ::2] = -0.0
    s[0, 2] = torch.arange(3000, dtype=torch.float32) % 7
    got = _topk_case(s.to(DEV), 2996, 1000)
    assert list(got[0]) == list(range(1000))
    assert list(got[1]) == list(range(1000))
    short = torch.randn(1, 5, 64)
    got = _topk_case(short.to(DEV), 0, 16)
    assert list(got[0][:1]) == [0] and np.all(got[0][1:] == -1)


def test_topk_boundary_bin_larger_than_candidate_buffer():
    # 30000 identical values straddle the threshold: the candidate list overflows
    # and the digit passes fall back to scanning the row.
    s = torch.randn(1, 2, 33000)
    s[:, :, 1000:31000] = 1.0
    s[:, 1, 31000:] = 5.0
    _topk_case(s.to(DEV), 32998, 2048)


def test_topk_few_long_rows_spread_over_a_cluster():
    # Three rows of 131072 scores (fewer rows than SMs): each row is spread over a
    # cluster of CTAs.  Row 0 random; row 1 has 100000 equal scores at the threshold
    # spanning every CTA's segment (candidate overflow, ties to smaller positions);
    # row 2 rounded scores with +-0.
    g = torch.Generator().manual_seed(13)
    Lk = 131072
    s = torch.randn(1, 3, Lk, generator=g)
    s[0, 1, 20000:120000] = 3.0
    s[0, 2] = torch.round(s[0, 2] * 4) / 4
    s[0, 2, 60000:70000:2] = -0.0
    _topk_case(s.to(DEV), Lk - 3, 2048)


# ------------------------------------------------------------------ sparse attention

def _attn_case(B, Lq, Lk, k, H, D, Dv, idx_np, seed, q_offset_for_oracle=0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, H, D, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lk, D, generator=g).to(torch.bfloat16)
    idx = torch.from_numpy(idx_np.astype(np.int32)).reshape(B, Lq, k)
    out, lse = dsa.sparse_attn(q.to(DEV), kv.to(DEV), idx.to(DEV), Dv, 1.0 / math.sqrt(192.0))
    torch.cuda.synchronize()
    rows = np.arange(B * Lq)
    ora_idx = idx_np.reshape(B * Lq, k).copy()
    ora_idx[(ora_idx < 0) | (ora_idx >= Lk)] = -1
    oo, ol = oracle.sparse_attn(rows // Lq, P.bf16_bits(q).reshape(B * Lq, H, D), P.bf16_bits(kv), ora_idx,
                                1.0 / math.sqrt(192.0), Dv)
    err = P.check_attention(out.reshape(B * Lq, H, Dv), lse.reshape(B * Lq, H), oo, ol)
    return out, lse, err


def _compact_indices(rng, B, Lq, Lk, k, q_offset):
    idx = np.full((B * Lq, k), -1, np.int64)
    for r in range(B * Lq):
        t = q_offset + r % Lq
        m = min(k, t + 1)
        idx[r, :m] = np.sort(rng.choice(t + 1, size=m, replace=False))
    return idx


def test_attention_tiny_shape_all_rows():
    wl = WORKLOADS["tiny"]
    rng = np.random.default_rng(5)
    idx = _compact_indices(rng, 1, 300, 1024, wl.k, 724)
    _attn_case(1, 300, 1024, wl.k, wl.H, wl.D, wl.Dv, idx, 5)


def test_attention_mla_shape_padding_and_gaps():
    rng = np.random.default_rng(6)
    B, Lq, Lk, k = 1, 24, 3000, 2048
    idx = _compact_indices(rng, B, Lq, Lk, k, 2980)
    idx[3, 100:400] = -1                # holes in the middle of a row
    idx[4, ::3] = Lk + 5                # out-of-range entries are skipped
    idx[5, :] = -1
    idx[5, 777] = 42                    # a single selected key
    idx[6, :1500] = -1                  # only the tail of the row is valid
    out, lse, _ = _attn_case(B, Lq, Lk, k, 128, 576, 512, idx, 6)


def test_attention_row_without_valid_entries():
    idx = np.full((1, 2, 256), -1, np.int64)
    idx[0, 1, :5] = [1, 2, 3, 4, 5]
    out, lse, _ = _attn_case(1, 2, 64, 256, 128, 576, 512, idx, 7)
    assert torch.all(out[0, 0] == 0) and torch.all(torch.isneginf(lse[0, 0]))


def test_attention_decode_split_k():
    rng = np.random.default_rng(8)
    B, Lk, k = 6, 5000, 2048
    idx = np.stack([np.sort(rng.choice(Lk, size=k, replace=False)) for _ in range(B)])
    _attn_case(B, 1, Lk, k, 128, 576, 512, idx, 8)


# ------------------------------------------------------------------ whole forward

def _forward(inp, wl, q_offset=None, Lq=None):
    q_offset = wl.q_offset if q_offset is None else q_offset
    idx, out, lse = dsa.forward(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], inp["q"],
                                inp["kv"], wl.k, wl.Dv, wl.scale, q_offset)
    torch.cuda.synchronize()
    return idx, out, lse


def _check_forward_rows(inp, wl, idx, out, lse, rows, Lq, q_offset, exact_idx=False, keys=None):
    res, keys = P.oracle_forward_rows(inp, rows, Lq, q_offset, wl.k, wl.scale, wl.Dv, keys=keys)
    sel = torch.as_tensor(rows, device=DEV)
    gi = idx.reshape(-1, wl.k)[sel].cpu().numpy()
    swaps = P.check_index_sets(gi, res["scores"], res["row_t"], wl.k, exact=exact_idx)
    # attention judged on the GPU's own index set
    oo, ol = oracle.sparse_attn(res["row_b"], res["q"], keys["kv"], gi, wl.scale, wl.Dv)
    go = out.reshape(-1, wl.H, wl.Dv)[sel]
    gl = lse.reshape(-1, wl.H)[sel]
    err = P.check_attention(go, gl, oo, ol)
    return swaps, err


def test_forward_tiny_all_rows_exact_indices():
    wl = WORKLOADS["tiny"]
    inp = to_dev(make_inputs(wl, "cpu", 0))
    idx, out, lse = _forward(inp, wl)
    _check_forward_rows(inp, wl, idx, out, lse, np.arange(wl.Lq), wl.Lq, 0, exact_idx=True)


def test_forward_short_sequence_is_dense_causal_attention():
    # q_offset + Lq <= k: every row selects all of 0..t, the pass is dense causal
    # attention and the indexer is not consulted -- garbage indexer inputs give the
    # same result.
    wl = WORKLOADS["prefill_8k"].with_(Lq=1024, Lk=1024)
    inp = make_inputs(wl, DEV, 3)
    idx, out, lse = _forward(inp, wl)
    n = np.arange(wl.Lq) + 1
    want = np.where(np.arange(wl.k)[None, :] < n[:, None], np.arange(wl.k)[None, :], -1)
    assert np.array_equal(idx.reshape(-1, wl.k).cpu().numpy(), want)
    rows = np.r_[0, 1, 63, 500, 1022, 1023]
    keys = oracle.keys_from_inputs(inp)
    r = oracle.rows_from_inputs(inp, rows, wl.Lq, 0)
    oo, ol = oracle.sparse_attn(r["row_b"], r["q"], keys["kv"], want[rows].astype(np.int32), wl.scale, wl.Dv)
    P.check_attention(out.reshape(-1, wl.H, wl.Dv)[torch.as_tensor(rows, device=DEV)],
                      lse.reshape(-1, wl.H)[torch.as_tensor(rows, device=DEV)], oo, ol)
    garbage = dict(inp)
    garbage["q_I"] = torch.randint(0, 255, inp["q_I"].shape, dtype=inp["q_I"].dtype, device=DEV)
    idx2, out2, lse2 = _forward(garbage, wl)
    assert torch.equal(idx2, idx) and torch.equal(out2, out)


def test_forward_prefill_8k_sampled_rows():
    wl = WORKLOADS["prefill_8k"]
    inp = make_inputs(wl, DEV, 0)
    idx, out, lse = _forward(inp, wl)
    rows = np.r_[0, 1, 2, 127, 128, 1000, 2046, 2047, 2048, 2049, 4095, 5000, 8190, 8191]
    _check_forward_rows(inp, wl, idx, out, lse, rows, wl.Lq, 0)


def test_forward_decode_128k_sampled_sequences():
    wl = WORKLOADS["decode_128k"]
    inp = make_key_side(wl, DEV, 0)
    inp.update(make_query_side(wl, DEV, 0))
    idx, out, lse = _forward(inp, wl)
    _check_forward_rows(inp, wl, idx, out, lse, np.array([0, 17, 40, 63]), 1, wl.q_offset)


def _rows_32k(L, k):
    """512 rows of an L-query prefill: every 64th row of t < k, the last 64 rows,
    and the rest spread evenly over the middle."""
    head = np.arange(0, k, 64)
    tail = np.arange(L - 64, L)
    mid = np.linspace(k, L - 65, 512 - len(head) - len(tail)).round().astype(np.int64)
    rows = np.unique(np.r_[head, mid, tail])
    assert len(rows) == 512
    return rows


def test_forward_prefill_32k_sampled_rows():
    wl = WORKLOADS["prefill_32k"]
    inp = make_inputs(wl, DEV, 0)
    idx, out, lse = _forward(inp, wl)
    _check_forward_rows(inp, wl, idx, out, lse, _rows_32k(wl.Lq, wl.k), wl.Lq, 0)


def test_forward_prefill_128k_chunked_as_benchmarked():
    # The 32 chunk calls the benchmark times (bench.Runner), 256 rows checked:
    # eight per chunk, spread over the chunk, in every chunk.
    from bench import Runner
    wl = WORKLOADS["prefill_128k"]
    runner = Runner(wl, seed=0, device=DEV)
    runner.step(torch.cuda.current_stream())
    torch.cuda.synchronize()
    keys = oracle.keys_from_inputs(runner.keys)
    c = runner.chunk_len
    local = np.linspace(0, c - 1, 8).round().astype(np.int64)
    for n, (q_offset, qs) in enumerate(runner.chunks):
        inp = dict(runner.keys, **qs)
        cw = wl.with_(Lq=c, q_offset=q_offset)
        sl = slice(n * c, (n + 1) * c)
        _check_forward_rows(inp, cw, runner.indices[:, sl], runner.out[:, sl], runner.lse[:, sl], local, c,
                            q_offset, keys=keys)
    del runner
    torch.cuda.empty_cache()


def test_forward_decode_single_cached_token():
    # Lk = 1: the one key is selected and every head returns its value row.
    wl = WORKLOADS["decode_128k"].with_(B=5, Lk=1, q_offset=0)
    inp = make_inputs(wl, DEV, 4)
    idx, out, lse = _forward(inp, wl)
    got = idx.reshape(-1, wl.k).cpu().numpy()
    assert np.all(got[:, 0] == 0) and np.all(got[:, 1:] == -1)
    _check_forward_rows(inp, wl, idx, out, lse, np.arange(wl.B), 1, 0, exact_idx=True)


def test_forward_multi_token_decode():
    # three new tokens per sequence over a 6000-token cache: the generic indexer
    # build, the one-CTA top-k with rows kept in shared memory, attention unsplit
    wl = WORKLOADS["decode_128k"].with_(B=4, Lq=3, Lk=6000, q_offset=5997)
    inp = make_inputs(wl, DEV, 6)
    idx, out, lse = _forward(inp, wl)
    _check_forward_rows(inp, wl, idx, out, lse, np.arange(wl.B * wl.Lq), wl.Lq, wl.q_offset)


def test_wait_timeout_is_reported_not_trapped():
    assert dsa.selftest_wait_timeout(1 << 14) == 5
    assert dsa.device_status() == 0
    x = torch.ones(4, device=DEV)
    assert float(x.sum()) == 4.0          # the context is still usable


# ------------------------------------------------------------------ context-parallel prefill

def test_context_parallel_single_rank_matches_the_whole_sequence():
    # One rank owning both zig-zag chunks: per-chunk forwards over the gathered
    # key prefix reproduce the one-call forward of the whole sequence.
    from sparse_attention_19_b200 import context_parallel as cp
    wl = WORKLOADS["prefill_8k"].with_(Lq=4096, Lk=4096)
    inp = to_dev(make_inputs(wl, "cpu", 3))
    idx, out, lse = _forward(inp, wl)
    chunk = 2048
    mine = cp.zigzag_chunks(2, 1, 0)
    local = cp.local_key_side(inp, mine, chunk)
    queries = {c: {f: inp[f][:, c * chunk:(c + 1) * chunk].contiguous() for f in ("q_I", "q_scale", "w", "q")}
               for c in mine}
    res = cp.cp_forward(queries, local, 2, chunk, wl.k, wl.Dv, wl.scale, world=1, rank=0)
    torch.cuda.synchronize()
    keys = oracle.keys_from_inputs(inp)
    for c in mine:
        ci, co, cl = res[c]
        sl = slice(c * chunk, (c + 1) * chunk)
        assert torch.equal(ci, idx[:, sl])
        assert float((co.float() - out[:, sl].float()).abs().max()) <= 1e-2
        assert float((cl - lse[:, sl]).abs().max()) <= 1e-4
        # each chunk's own result against the oracle, rows spread over the chunk
        cw = wl.with_(Lq=chunk, q_offset=c * chunk)
        qin = dict(inp, **queries[c])
        _check_forward_rows(qin, cw, ci, co, cl, np.r_[0, 1, 700, 1500, chunk - 2, chunk - 1], chunk, c * chunk,
                            keys=keys)
