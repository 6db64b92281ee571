"""TEST INFRASTRUCTURE ONLY: ctypes wrapper around the fp64 CPU oracle.

The oracle (``dsa_oracle.c`` beside this file) is a plain statement of the
DeepSeek Sparse Attention forward pass from the DeepSeek-V3.2 technical-report
summary, section "DSA: внимание только к важному" (lightning-indexer equation
for I_{t,s}; selection-and-attention equation for u_t).  Only the tests, the
package smoke check and the benchmark's CPU-baseline leg may import this module.
It imports nothing from the CUDA package, and the CUDA package imports nothing
from here.

All arrays cross this boundary as numpy arrays: FP8 values as their uint8 e4m3
codes, bf16 values as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (OpenMP, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_e4m3_value.restype = f64
            lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.oracle_bf16_value.restype = f64
            lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
            lib.oracle_num_threads.restype = i32
            lib.oracle_indexer_scores.restype = i32
            lib.oracle_indexer_scores.argtypes = [i64, P, P, i32, i32, P, P, P, i32, P, P, P]
            lib.oracle_topk.restype = i32
            lib.oracle_topk.argtypes = [P, i64, i32, P, i32, P]
            lib.oracle_sparse_attn.restype = i32
            lib.oracle_sparse_attn.argtypes = [i64, P, i32, i32, i32, f64, P, i32, P, P, i32, P, P]
            lib.oracle_indexer_kl.restype = i32
            lib.oracle_indexer_kl.argtypes = [i64, P, i32, i32, f64, P, i32, P, P, i32, P, P, P]
            lib.oracle_dsa_forward.restype = i32
            lib.oracle_dsa_forward.argtypes = [i64, P, P, i32, i32, P, P, P, i32, P, P,
                                               i32, i32, i32, f64, P, P, i32, P, P, P, P]
            _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _opt(a, dtype):
    if a is None:
        return None, None
    return _c(a, dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def e4m3_value(code: int) -> float:
    return float(_load().oracle_e4m3_value(int(code)))


def bf16_value(bits: int) -> float:
    return float(_load().oracle_bf16_value(int(bits)))


def indexer_scores(row_b, row_t, q_I, q_scale, w, k_I, k_scale):
    """I[r, s] for query rows r (own inputs q_I[r], q_scale[r], w[r]) against all keys.

    q_I: uint8 [n, H_I, d_I]; q_scale: f32 [n] or None; w: uint16 (bf16 bits) [n, H_I];
    k_I: uint8 [B, Lk, d_I]; k_scale: f32 [B, Lk] or None.  Returns f64 [n, Lk]
    with -inf where s > t.
    """
    q_I = np.asarray(q_I)
    n, H_I, d_I = q_I.shape
    Lk = np.asarray(k_I).shape[1]
    rb, prb = _c(row_b, np.int64)
    rt, prt = _c(row_t, np.int64)
    qa, pq = _c(q_I, np.uint8)
    qs, pqs = _opt(q_scale, np.float32)
    wa, pw = _c(w, np.uint16)
    ka, pk = _c(k_I, np.uint8)
    ks, pks = _opt(k_scale, np.float32)
    out = np.empty((n, Lk), dtype=np.float64)
    rc = _load().oracle_indexer_scores(n, prb, prt, H_I, d_I, pq, pqs, pw, Lk, pk, pks,
                                       out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError(f"oracle_indexer_scores failed ({rc})")
    return out


def topk(scores, row_t, k):
    """Top-k positions per row (ties to smaller s), ascending, -1 padded: int32 [n, k]."""
    sc, ps = _c(scores, np.float64)
    n, Lk = sc.shape
    rt, prt = _c(row_t, np.int64)
    out = np.empty((n, k), dtype=np.int32)
    rc = _load().oracle_topk(ps, n, Lk, prt, k, out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError(f"oracle_topk failed ({rc})")
    return out


def sparse_attn(row_b, q, kv, indices, scale, Dv):
    """Softmax attention of rows q[r] (uint16 bf16 bits [n, H, D]) over kv[b][indices[r]].

    kv: uint16 [B, Lk, D]; indices: int32 [n, k].  Returns (out f64 [n, H, Dv], lse f64 [n, H]).
    """
    qa, pq = _c(q, np.uint16)
    n, H, D = qa.shape
    kva, pkv = _c(kv, np.uint16)
    Lk = kva.shape[1]
    ia, pi = _c(indices, np.int32)
    k = ia.shape[1]
    rb, prb = _c(row_b, np.int64)
    out = np.empty((n, H, Dv), dtype=np.float64)
    lse = np.empty((n, H), dtype=np.float64)
    rc = _load().oracle_sparse_attn(n, prb, H, D, Dv, float(scale), pq, Lk, pkv, pi, k,
                                    out.ctypes.data_as(ctypes.c_void_p),
                                    lse.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError(f"oracle_sparse_attn failed ({rc})")
    return out, lse


def indexer_kl(row_b, q, kv, indices, scores, scale):
    """The indexer's training loss over the selected positions, per query row.

    DeepSeek-V3.2 technical-report summary, section "Как учили индексатор": the
    target p is the main attention's probabilities summed over the heads and
    L1-normalised; the loss is D_KL(p || softmax(I)) over the selected positions
    (the sparse stage).  q: uint16 bf16 bits [n, H, D]; kv: uint16 [B, Lk, D];
    indices: int32 [n, k] (negative = padding); scores: float [n, Lk], row r's
    indexer scores.  Returns (target f64 [n, k] aligned with the index slots,
    kl f64 [n]).
    """
    qa, pq = _c(q, np.uint16)
    n, H, D = qa.shape
    kva, pkv = _c(kv, np.uint16)
    Lk = kva.shape[1]
    ia, pi = _c(indices, np.int32)
    k = ia.shape[1]
    sa, ps = _c(scores, np.float64)
    if sa.shape != (n, Lk):
        raise ValueError("scores must be [n, Lk]")
    rb, prb = _c(row_b, np.int64)
    target = np.empty((n, k), dtype=np.float64)
    kl = np.empty(n, dtype=np.float64)
    rc = _load().oracle_indexer_kl(n, prb, H, D, float(scale), pq, Lk, pkv, pi, k, ps,
                                   target.ctypes.data_as(ctypes.c_void_p),
                                   kl.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError(f"oracle_indexer_kl failed ({rc})")
    return target, kl


def dsa_forward(row_b, row_t, q_I, q_scale, w, k_I, k_scale, q, kv, k, scale, Dv,
                want_scores=False):
    """Indexer -> top-k -> sparse attention for the given query rows.

    Returns dict(indices int32 [n,k], out f64 [n,H,Dv], lse f64 [n,H], scores f64 [n,Lk] or None).
    """
    qa, pqi = _c(q_I, np.uint8)
    n, H_I, d_I = qa.shape
    ka, pk = _c(k_I, np.uint8)
    Lk = ka.shape[1]
    qs, pqs = _opt(q_scale, np.float32)
    ks, pks = _opt(k_scale, np.float32)
    wa, pw = _c(w, np.uint16)
    qq, pq = _c(q, np.uint16)
    _, H, D = qq.shape
    kva, pkv = _c(kv, np.uint16)
    rb, prb = _c(row_b, np.int64)
    rt, prt = _c(row_t, np.int64)
    idx = np.empty((n, k), dtype=np.int32)
    out = np.empty((n, H, Dv), dtype=np.float64)
    lse = np.empty((n, H), dtype=np.float64)
    scores = np.empty((n, Lk), dtype=np.float64) if want_scores else None
    rc = _load().oracle_dsa_forward(
        n, prb, prt, H_I, d_I, pqi, pqs, pw, Lk, pk, pks, H, D, Dv, float(scale), pq, pkv, k,
        idx.ctypes.data_as(ctypes.c_void_p), out.ctypes.data_as(ctypes.c_void_p),
        lse.ctypes.data_as(ctypes.c_void_p),
        scores.ctypes.data_as(ctypes.c_void_p) if scores is not None else None)
    if rc != 0:
        raise ValueError(f"oracle_dsa_forward failed ({rc})")
    return {"indices": idx, "out": out, "lse": lse, "scores": scores}


# ---- helpers turning generator tensors into oracle arrays ------------------------

def rows_from_inputs(inp: dict, rows, Lq: int, q_offset: int):
    """Gather the query-side inputs of flattened rows (b*Lq + i) as numpy arrays.

    ``inp`` holds torch tensors (any device) shaped [B, Lq, ...] as produced by
    ``dsa_inputs``; ``rows`` is a 1-D integer array.  Row b*Lq + i sits at
    position q_offset + i.  Returns a dict ready for ``dsa_forward``.
    """
    import torch
    rows = np.asarray(rows, dtype=np.int64)
    sel = torch.as_tensor(rows)

    def take(name):
        t = inp[name]
        flat = t.reshape(-1, *t.shape[2:]) if t.dim() > 2 else t.reshape(-1)
        return flat[sel.to(flat.device)].cpu()

    return {
        "row_b": rows // Lq,
        "row_t": q_offset + rows % Lq,
        "q_I": take("q_I").numpy(),
        "q_scale": take("q_scale").numpy(),
        "w": take("w").view(torch.int16).numpy().view(np.uint16),
        "q": take("q").view(torch.int16).numpy().view(np.uint16),
    }


def keys_from_inputs(inp: dict):
    """The key side (k_I, k_scale, kv) as numpy arrays on the host."""
    import torch
    return {
        "k_I": inp["k_I"].cpu().numpy(),
        "k_scale": inp["k_scale"].cpu().numpy(),
        "kv": inp["kv"].cpu().view(torch.int16).numpy().view(np.uint16),
    }
