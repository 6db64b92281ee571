"""An independent numpy restatement of the DSA forward pass (test helper).

Written separately from the C oracle to catch indexing slips in either: it uses
whole-array numpy operations where the oracle uses scalar loops.  It is a
cross-check, not a pin: agreement with the oracle shows the two statements match,
while the pins in test_oracle_pins.py tie the oracle to independent facts.

Equations (DeepSeek-V3.2 technical-report summary, "DSA: внимание только к
важному"): I[t,s] = sum_j w[t,j] ReLU(q_I[t,j].k_I[s]); top-k over s <= t;
softmax attention over the selected latent rows, V = the leading Dv columns.
"""
import numpy as np
import torch


def e4m3_to_f64(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def bf16_to_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def indexer(row_b, row_t, q_I, q_scale, w, k_I, k_scale):
    qd = e4m3_to_f64(q_I) * np.asarray(q_scale, np.float64)[:, None, None]    # [n, H_I, d]
    kd = e4m3_to_f64(k_I) * np.asarray(k_scale, np.float64)[:, :, None]        # [B, Lk, d]
    wd = bf16_to_f64(w)                                                         # [n, H_I]
    keys = kd[np.asarray(row_b)]                                                # [n, Lk, d]
    x = np.einsum("njd,nsd->njs", qd, keys)
    I = np.einsum("nj,njs->ns", wd, np.maximum(x, 0.0))
    Lk = kd.shape[1]
    I[np.arange(Lk)[None, :] > np.asarray(row_t)[:, None]] = -np.inf
    return I


def topk(I, row_t, k):
    n, Lk = I.shape
    out = np.full((n, k), -1, np.int32)
    for r in range(n):
        t = int(row_t[r])
        cand = np.arange(min(t + 1, Lk))
        # lexsort: last key is primary -> (score descending, position ascending)
        order = np.lexsort((cand, -I[r, cand]))
        m = min(k, len(cand))
        out[r, :m] = np.sort(cand[order[:m]])
    return out


def attention(row_b, q, kv, idx, scale, Dv):
    qd = bf16_to_f64(q)                  # [n, H, D]
    kvd = bf16_to_f64(kv)                # [B, Lk, D]
    n, H, _ = qd.shape
    out = np.zeros((n, H, Dv))
    lse = np.full((n, H), -np.inf)
    for r in range(n):
        sel = idx[r][idx[r] >= 0]
        if len(sel) == 0:
            continue
        rows = kvd[row_b[r]][sel]        # [m, D]
        z = scale * qd[r] @ rows.T       # [H, m]
        zmax = z.max(1, keepdims=True)
        p = np.exp(z - zmax)
        l = p.sum(1, keepdims=True)
        out[r] = (p / l) @ rows[:, :Dv]
        lse[r] = (zmax + np.log(l))[:, 0]
    return out, lse
