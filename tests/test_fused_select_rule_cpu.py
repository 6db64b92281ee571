"""The selection rule the fused indexer + top-k kernel follows, re-enacted in
numpy and held against the oracle's top-k (no GPU).

The kernel never sees a whole row of scores.  Per row it keeps a list of
candidates in position order.  A score joins the list only if its key beats the
row's current threshold, which may be stale.  When the list is full, it is cut
to the exact top-k (key descending, position ascending), and the threshold
becomes the k-th key.  A later score equal to it loses the tie, since every later
position is larger.  Rows split over several units are cut per unit and finished
over the units' lists in position order.  The rule must give exactly the oracle's
index set, ties, +-0 and rows shorter than k included."""
import numpy as np
import pytest

import oracle


def _key(v):
    u = np.asarray(v, np.float32).view(np.uint32).copy()
    u[(u << 1) == 0] = 0                                     # -0.0 -> +0.0
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def _cut(keys, pos, m):
    """Top-m of a list in position order: keys > thr and the first m - gt keys == thr."""
    thr = np.sort(keys)[::-1][m - 1]
    gt = int(np.sum(keys > thr))
    keep = keys > thr
    keep[np.where(keys == thr)[0][: m - gt]] = True
    return keys[keep], pos[keep], thr


def _unit(scores, t, k, cap, kt0, kt1, lag):
    """One unit's tiles [kt0, kt1) of one row; the epilogue filters with the
    threshold published `lag` tiles earlier (a stale value is allowed)."""
    xk, xp = np.zeros(0, np.uint32), np.zeros(0, np.int64)
    published = [0]                                          # threshold history, 0 passes every score
    for kt in range(kt0, kt1):
        s = np.arange(kt * 128, kt * 128 + 128)
        s = s[(s <= t) & (s < len(scores))]
        keys = _key(scores[s])
        th_epi = published[max(0, len(published) - 1 - lag)]
        staged_k, staged_p = keys[keys > th_epi], s[keys > th_epi]
        if len(xk) + len(staged_k) > cap:
            xk, xp, thr = _cut(xk, xp, k)
            published.append(thr)
        keep = staged_k > published[-1]
        xk, xp = np.concatenate([xk, staged_k[keep]]), np.concatenate([xp, staged_p[keep]])
    return xk, xp


@pytest.mark.parametrize("kind", ["normal", "rounded", "zeros", "integers"])
def test_streaming_rule_equals_the_oracle_top_k(kind):
    rng = np.random.default_rng({"normal": 0, "rounded": 1, "zeros": 2, "integers": 3}[kind])
    for _ in range(60):
        n = int(rng.integers(1, 9000))
        t = n - 1
        k = int(rng.choice([1, 7, 128, 300, 2048]))
        if kind == "normal":
            sc = rng.standard_normal(n).astype(np.float32)
        elif kind == "rounded":
            sc = np.round(rng.standard_normal(n) * 3).astype(np.float32)
        elif kind == "zeros":
            sc = np.zeros(n, np.float32)
            sc[::3] = -0.0
        else:
            sc = rng.integers(-2, 3, n).astype(np.float32)
        k32 = (k + 31) // 32 * 32
        cap = k32 + max(k32, 256)                              # the kernel's list capacity
        ntiles = t // 128 + 1
        chunks = int(rng.integers(1, 6))
        per = (ntiles + chunks - 1) // chunks
        lists = []
        for c in range(chunks):
            xk, xp = _unit(sc, t, k, cap, min(ntiles, c * per), min(ntiles, (c + 1) * per), int(rng.integers(0, 4)))
            if chunks > 1 and len(xk) > k:
                xk, xp, _ = _cut(xk, xp, k)
            lists.append((xk, xp))
        xk = np.concatenate([a for a, _ in lists])
        xp = np.concatenate([b for _, b in lists])
        assert np.all(np.diff(xp) > 0)                         # lists stay in position order
        if len(xk) > k:
            xk, xp, _ = _cut(xk, xp, k)
        got = np.full(k, -1, np.int64)
        got[: len(xp)] = xp
        want = oracle.topk(sc[None, :].astype(np.float64), np.array([t]), k)[0]
        assert np.array_equal(got, want), (n, k, chunks)
