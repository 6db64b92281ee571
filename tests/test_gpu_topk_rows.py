"""Top-k over many rows (prefill-sized row counts), the shape that runs one warp
per row: a sampled key range, one histogram pass, the exact threshold inside the
boundary bin (its keys straight to a 512-entry buffer when they fit, else
histogram levels over the row), and an ordered output pass.

Every row is held against the fp64 oracle's top-k ("Отбор и основное внимание":
the k positions with the largest I[t, s]; ties to the smaller position, -0.0
equal to +0.0), bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_19_b200 as dsa
from dsa_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROWS = 2600          # above the many-rows threshold (16 rows per SM on a 148-SM part)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.lib()
    yield
    assert dsa.device_status() == 0


def _check(scores, q_offset, k):
    B, Lq, Lk = scores.shape
    idx = dsa.topk(scores, k, q_offset)
    torch.cuda.synchronize()
    sc = scores.double().cpu().numpy().reshape(B * Lq, Lk)
    row_t = q_offset + np.arange(B * Lq) % Lq
    exp = oracle.topk(sc, row_t, k)
    got = idx.cpu().numpy().reshape(B * Lq, k)
    bad = np.nonzero(~np.all(got == exp, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:5]}"
    return got


def test_many_rows_random_scores_aligned_rows():
    g = torch.Generator().manual_seed(21)
    s = torch.randn(1, ROWS, 6000, generator=g)       # 16-byte aligned rows
    _check(s.to(DEV), 6000 - ROWS, 2048)


def test_many_rows_ragged_length_and_heavy_ties():
    # Lk not a multiple of four (4-byte loads); scores on a 0.1 grid: many ties
    g = torch.Generator().manual_seed(22)
    s = torch.round(torch.randn(1, ROWS, 5003, generator=g) * 10) / 10
    _check(s.to(DEV), 5003 - ROWS, 2048)


def test_many_rows_boundary_bin_overflows_the_buffer():
    # a block of 3000 equal scores straddles the threshold in every row: the
    # boundary bin holds more than 512 keys, so the threshold comes from
    # histogram levels over the row
    g = torch.Generator().manual_seed(23)
    s = torch.randn(1, ROWS, 8000, generator=g)
    s[:, :, 2000:5000] = 1.25
    _check(s.to(DEV), 8000 - ROWS, 2048)


def test_many_rows_all_equal_and_signed_zero():
    s = torch.full((2, ROWS // 2, 4100), 0.75)
    s[0, ::2] = 0.0
    s[0, ::2, ::3] = -0.0
    got = _check(s.to(DEV), 4100 - ROWS // 2, 1024)
    assert np.array_equal(got[0], np.arange(1024))


def test_forward_selected_scores_from_the_many_rows_kernel():
    # dsa_forward's staged selection returns I[t, s] at every selected position
    wl = WORKLOADS["prefill_8k"].with_(Lq=ROWS, Lk=6000, q_offset=6000 - ROWS)
    inp = make_inputs(wl, DEV, 7)
    sel = torch.empty(wl.B, wl.Lq, wl.k, dtype=torch.float32, device=DEV)
    idx, _, _ = dsa.forward(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], inp["q"],
                            inp["kv"], wl.k, wl.Dv, wl.scale, wl.q_offset, sel_scores=sel)
    scores = dsa.indexer_scores(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], wl.q_offset)
    torch.cuda.synchronize()
    assert torch.equal(idx, dsa.topk(scores, wl.k, wl.q_offset))
    valid = idx >= 0
    want = torch.gather(scores, 2, idx.clamp_min(0).long())
    assert torch.equal(sel[valid], want[valid])
    assert torch.all(torch.isneginf(sel[~valid]))


# Long rows (more than 32768 scores, or fewer rows than the one-warp kernel
# wants): one CTA per row reads the row once, keeping every key at or above a
# threshold taken from a strided sample, and falls back to two passes when the
# kept keys number fewer than k or more than the 8192-entry buffer.

def test_long_rows_single_pass_random_scores():
    g = torch.Generator().manual_seed(31)
    s = torch.randn(1, 300, 40000, generator=g)
    _check(s.to(DEV), 40000 - 300, 2048)


def test_long_rows_ragged_length_with_planted_block():
    # Lk not a multiple of four; a block of high scores at the start of every row
    # (the strided sample sees few of them) and a band of ties
    g = torch.Generator().manual_seed(32)
    s = torch.randn(1, 200, 50001, generator=g)
    s[:, :, :1500] += 6.0
    s[:, :, 30000:30100] = 2.0
    _check(s.to(DEV), 50001 - 200, 2048)


def test_long_rows_fall_back_when_too_many_keys_pass():
    # half of every row equal to one value above the sample's threshold: far more
    # than 8192 keys pass, so the row takes the two-pass route
    g = torch.Generator().manual_seed(33)
    s = torch.randn(2, 100, 36000, generator=g)
    s[:, :, ::2] = 1.5
    s[1, :, 1::3] = -0.0
    _check(s.to(DEV), 36000 - 100, 2048)


# Few long rows (decode): each row spread over a cluster of CTAs, one pass over the
# row first (keys at or above a sampled threshold, per CTA segment), the two-pass
# route when the keys that pass are fewer than k over the row or overflow any
# segment's buffer.

def test_cluster_rows_one_pass_and_segment_overflow():
    g = torch.Generator().manual_seed(41)
    Lk = 131072
    s = torch.randn(1, 6, Lk, generator=g)
    s[0, 1, 1000:5500] = 5.0                         # one segment holds more than its buffer
    s[0, 2, ::87] = 4.0                              # 1507 planted ties, spread over all segments
    s[0, 2] = torch.where(s[0, 2] == 4.0, s[0, 2], torch.round(s[0, 2] * 8) / 8)
    s[0, 3] = 0.5                                    # every key passes: the two-pass route
    s[0, 4, ::13] = 5.0                              # ~10 K kept keys: one pass, refined over the cluster
    s[0, 5] *= 0.5                                   # ~5 K kept keys, refined by each CTA on a copy of all
    s[0, 5, ::67] = 5.0                              # of them; the threshold's ties (4.5) straddle the
    s[0, 5, 32700:32800] = 4.5                       # first two segments
    # ~7.6 K kept keys, none of them in the last segment and ~3 K in the third: a
    # CTA with nothing to share and one holding most of the copy
    g2 = torch.Generator().manual_seed(43)
    r6 = torch.randn(Lk, generator=g2)
    high = torch.randperm(32768, generator=g2)[:800] + 65536
    r6[high] = torch.randn(800, generator=g2) + 5.0
    r6[98304:] -= 10.0
    s = torch.cat([s, r6.view(1, 1, Lk)], dim=1)
    _check(s.to(DEV), Lk - 7, 2048)


def test_rows_not_16_byte_aligned_take_the_4_byte_passes():
    # Rows whose length is not a multiple of four start at addresses that are not
    # 16-byte aligned, so the single passes read 4-byte scores: a few long rows
    # spread over clusters (one with a block of planted ties), and ~100 rows of
    # 40 K scores, one CTA per row.
    g = torch.Generator().manual_seed(47)
    Lk = 131069
    s = torch.randn(1, 3, Lk, generator=g)
    s[0, 1, 50000:50600] = 4.0
    _check(s.to(DEV), Lk - 3, 2048)
    Lk = 40001
    s = torch.randn(1, 100, Lk, generator=g)
    s[0, 7, ::5] = 3.5
    _check(s.to(DEV), Lk - 100, 2048)
