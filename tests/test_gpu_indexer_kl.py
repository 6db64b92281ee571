"""CUDA indexer-loss forward vs the fp64 oracle, through the C ABI.

The loss (DeepSeek-V3.2 technical-report summary, section "Как учили
индексатор"): target p = the main attention's probabilities summed over the
heads and L1-normalised; per-row loss D_KL(p || softmax(I)) over the selected
positions.  The GPU path gets the attention's lse from dsa_sparse_attn and the
scores as given; the oracle recomputes the attention itself in fp64 and takes
the same scores (widened to fp64) and the same selection."""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_19_b200 as dsa
from dsa_inputs import WORKLOADS, make_inputs
import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCALE = 1.0 / math.sqrt(192.0)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.lib()
    yield
    assert dsa.device_status() == 0


def _compact_indices(rng, n_rows, Lq, k, q_offset):
    idx = np.full((n_rows, k), -1, np.int64)
    for r in range(n_rows):
        t = q_offset + r % Lq
        m = min(k, t + 1)
        idx[r, :m] = rng.permutation(rng.choice(t + 1, size=m, replace=False))
    return idx


def _kl_case(B, Lq, Lk, k, H, D, Dv, idx_np, seed, scores=None, rows=None):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, H, D, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lk, D, generator=g).to(torch.bfloat16)
    if scores is None:
        scores = torch.randn(B, Lq, Lk, generator=g) * 3.0
    idx = torch.from_numpy(idx_np.astype(np.int32)).reshape(B, Lq, k)
    qd, kvd, idxd = q.to(DEV), kv.to(DEV), idx.to(DEV)
    _, lse = dsa.sparse_attn(qd, kvd, idxd, Dv, SCALE)
    target, kl = dsa.indexer_kl_loss(qd, kvd, idxd, lse, scores.to(DEV), Dv, SCALE)
    torch.cuda.synchronize()
    n = B * Lq
    rows = np.arange(n) if rows is None else np.asarray(rows)
    ora_idx = idx_np.reshape(n, k)[rows].copy()
    ora_idx[(ora_idx < 0) | (ora_idx >= Lk)] = -1
    ot, ok = oracle.indexer_kl(rows // Lq, P.bf16_bits(q).reshape(n, H, D)[rows], P.bf16_bits(kv), ora_idx,
                               scores.reshape(n, Lk)[torch.as_tensor(rows)].double().numpy(), SCALE)
    sel = torch.as_tensor(rows, device=DEV)
    errs = P.check_kl(target.reshape(n, k)[sel], kl.reshape(n)[sel], ot, ok)
    return target, kl, ot, ok, errs


def test_kl_tiny_shape_all_rows():
    wl = WORKLOADS["tiny"]
    rng = np.random.default_rng(50)
    idx = _compact_indices(rng, 300, 300, wl.k, 724)
    _kl_case(1, 300, 1024, wl.k, wl.H, wl.D, wl.Dv, idx, 50)


def test_kl_mla_shape_padding_gaps_and_ragged_k():
    rng = np.random.default_rng(51)
    B, Lq, Lk, k = 2, 12, 3000, 2000          # k not a multiple of the 64-key tile
    idx = _compact_indices(rng, B * Lq, Lq, k, 2980)
    idx[3, 100:400] = -1                      # holes in the middle of a row
    idx[4, ::3] = Lk + 5                      # out-of-range entries are padding
    idx[5, :] = -1
    idx[5, 777] = 42                          # a single selected key: p = 1, KL = 0
    idx[6, :1500] = -1                        # only the tail of the row is valid
    idx[7, :] = -1                            # nothing selected: target 0, KL 0
    target, kl, ot, ok, _ = _kl_case(B, Lq, Lk, k, 128, 576, 512, idx, 51)
    assert float(target.reshape(-1, k)[5, 777]) == pytest.approx(1.0, rel=1e-6)
    assert float(kl.reshape(-1)[5]) == pytest.approx(0.0, abs=1e-6)
    assert torch.all(target.reshape(-1, k)[7] == 0) and float(kl.reshape(-1)[7]) == 0.0


def test_kl_vanishes_when_the_scores_reproduce_the_target():
    rng = np.random.default_rng(52)
    B, Lq, Lk, k = 1, 8, 4096, 2048
    idx = _compact_indices(rng, Lq, Lq, k, 4088)
    g = torch.Generator().manual_seed(53)
    q = torch.randn(B, Lq, 128, 576, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lk, 576, generator=g).to(torch.bfloat16)
    ot, _ = oracle.indexer_kl(np.zeros(Lq, np.int64), P.bf16_bits(q).reshape(Lq, 128, 576), P.bf16_bits(kv),
                              idx, np.zeros((Lq, Lk)), SCALE)
    scores = torch.full((B, Lq, Lk), -1e4)
    for r in range(Lq):
        scores[0, r, torch.from_numpy(idx[r])] = torch.from_numpy(np.log(ot[r]) + 2.5).float()
    idxd = torch.from_numpy(idx.astype(np.int32)).reshape(B, Lq, k).to(DEV)
    _, lse = dsa.sparse_attn(q.to(DEV), kv.to(DEV), idxd, 512, SCALE)
    _, kl = dsa.indexer_kl_loss(q.to(DEV), kv.to(DEV), idxd, lse, scores.to(DEV), 512, SCALE, want_target=False)
    torch.cuda.synchronize()
    assert float(kl.abs().max()) <= 2e-5


@pytest.mark.parametrize("name", ["prefill_8k", "prefill_32k"])
def test_kl_prefill_forward_sampled_rows(name):
    # The loss on the forward pass's own outputs at the 8K and 32K prefill sizes
    # (32K is the launch the benchmark times): the indexer scores, the selection
    # and the lse come from the library's own stages.
    wl = WORKLOADS[name]
    inp = {k_: v.to(DEV) for k_, v in make_inputs(wl, "cpu", 0).items()}
    scores = dsa.indexer_scores(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], wl.q_offset)
    idx = dsa.topk(scores, wl.k, wl.q_offset)
    _, lse = dsa.sparse_attn(inp["q"], inp["kv"], idx, wl.Dv, wl.scale)
    target, kl = dsa.indexer_kl_loss(inp["q"], inp["kv"], idx, lse, scores, wl.Dv, wl.scale)
    torch.cuda.synchronize()
    n = wl.B * wl.Lq
    rows = np.unique(np.concatenate([[0, 1, 2, 63, 2047, 2048, 2049], np.arange(n - 8, n),
                                     np.random.default_rng(54).choice(n, 16, replace=False)]))
    sel = torch.as_tensor(rows, device=DEV)
    q_rows = P.bf16_bits(inp["q"].reshape(n, wl.H, wl.D)[sel])
    gi = idx.reshape(n, wl.k)[sel].cpu().numpy()
    gs = scores.reshape(n, wl.Lk)[sel].double().cpu().numpy()
    ot, ok = oracle.indexer_kl(rows // wl.Lq, q_rows, P.bf16_bits(inp["kv"]), gi, gs, wl.scale)
    P.check_kl(target.reshape(n, wl.k)[sel], kl.reshape(n)[sel], ot, ok)
    assert torch.isfinite(kl).all() and float(kl.min()) >= -1e-5
