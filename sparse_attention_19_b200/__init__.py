"""DeepSeek Sparse Attention (DSA) forward pass on B200 (sm_100a).

Thin Python binding over the C ABI of ``libdsa.so`` (declared in
``include/dsa.h``).  Functions carry the C names without the ``dsa_`` prefix and
only marshal arguments: tensors must already be on the GPU, with the dtypes and
shapes the header documents; every step of the computation runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.

Equations (DeepSeek-V3.2 technical-report summary, section "DSA: внимание
только к важному"):
    I[t,s] = sum_j w[t,j] ReLU(q_I[t,j] . k_I[s])                 (lightning indexer)
    u_t    = Attn(h_t, {c_s : I[t,s] in Top-k(I[t,:])}), k = 2048  (selection + MQA attention)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "DSAError", "lib", "lib_path", "indexer_scores", "topk", "indexer_topk", "sparse_attn", "sparse_attn_noalloc",
    "forward", "indexer_kl_loss", "indexer_kl_loss_selected",
    "workspace_size", "workspace_size_args", "status_string", "device_status", "selftest_wait_timeout", "version",
    "OP_TOPK", "OP_SPARSE_ATTN", "OP_FORWARD", "OP_INDEXER_TOPK", "OP_FORWARD_LOWMEM",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libdsa.so")

OP_TOPK, OP_SPARSE_ATTN, OP_FORWARD, OP_INDEXER_TOPK, OP_FORWARD_LOWMEM = 0, 1, 2, 3, 4
_STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_WORKSPACE",
           4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT"}


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class IndexerArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Lq", ctypes.c_int), ("Lk", ctypes.c_int), ("q_offset", ctypes.c_int),
                ("H_I", ctypes.c_int), ("d_I", ctypes.c_int),
                ("q_I", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("k_I", ctypes.c_void_p), ("k_scale", ctypes.c_void_p)]


class AttnArgs(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("d_qk", ctypes.c_int), ("d_v", ctypes.c_int), ("scale", ctypes.c_float),
                ("q", ctypes.c_void_p), ("kv", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError(f"libdsa.so not built at {lib_path}; run python -m sparse_attention_19_b200.build")
        L = ctypes.CDLL(lib_path)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.dsa_indexer_scores.argtypes = [ctypes.POINTER(IndexerArgs), P, P]
        L.dsa_topk.argtypes = [P, I, I, I, I, I, P, P, Z, P]
        L.dsa_sparse_attn.argtypes = [ctypes.POINTER(AttnArgs), I, I, I, P, I, P, P, P, Z, P]
        L.dsa_sparse_attn_noalloc.argtypes = [ctypes.POINTER(AttnArgs), I, I, I, P, I, P, P, P]
        L.dsa_forward.argtypes = [ctypes.POINTER(IndexerArgs), ctypes.POINTER(AttnArgs), I, P, P, P, P, Z, P]
        L.dsa_forward_timed.argtypes = [ctypes.POINTER(IndexerArgs), ctypes.POINTER(AttnArgs), I, P, P, P, P, P, Z,
                                        P, ctypes.POINTER(ctypes.c_void_p)]
        L.dsa_indexer_topk.argtypes = [ctypes.POINTER(IndexerArgs), I, P, P, P, Z, P]
        L.dsa_indexer_kl_loss.argtypes = [ctypes.POINTER(AttnArgs), I, I, I, P, I, P, P, P, P, P]
        L.dsa_indexer_kl_loss_selected.argtypes = [ctypes.POINTER(AttnArgs), I, I, I, P, I, P, P, P, P, P]
        L.dsa_workspace_size.argtypes = [I, I, I, I, I, I, I]
        L.dsa_workspace_size.restype = ctypes.c_size_t
        L.dsa_workspace_size_args.argtypes = [I, ctypes.POINTER(IndexerArgs), I, I, I]
        L.dsa_workspace_size_args.restype = ctypes.c_size_t
        L.dsa_status_string.argtypes = [I]
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_device_status.argtypes = [I]
        L.dsa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, P]
        for f in ("dsa_indexer_scores", "dsa_topk", "dsa_indexer_topk", "dsa_sparse_attn", "dsa_sparse_attn_noalloc",
                  "dsa_forward", "dsa_forward_timed", "dsa_indexer_kl_loss", "dsa_indexer_kl_loss_selected",
                  "dsa_device_status",
                  "dsa_selftest_wait_timeout", "dsa_version"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().dsa_status_string(int(status)).decode()
    except ImportError:
        return _STATUS.get(int(status), f"status {status}")


def version() -> int:
    return int(lib().dsa_version())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise DSAError(rc, where)


def _need(t, dtype, shape, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def _u8(t):
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


def _indexer_args(q_I, q_scale, w, k_I, k_scale, q_offset):
    q_I, k_I = _u8(q_I), _u8(k_I)
    B, Lq, H_I, d_I = q_I.shape
    Lk = k_I.shape[1]
    _need(q_I, torch.uint8, (B, Lq, H_I, d_I), "q_I")
    _need(w, torch.bfloat16, (B, Lq, H_I), "w")
    _need(k_I, torch.uint8, (B, Lk, d_I), "k_I")
    if q_scale is not None:
        _need(q_scale, torch.float32, (B, Lq), "q_scale")
    if k_scale is not None:
        _need(k_scale, torch.float32, (B, Lk), "k_scale")
    return IndexerArgs(B, Lq, Lk, int(q_offset), H_I, d_I, _ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_I),
                       _ptr(k_scale))


def _attn_args(q, kv, d_v, scale):
    B, Lq, H, D = q.shape
    _need(q, torch.bfloat16, (B, Lq, H, D), "q")
    _need(kv, torch.bfloat16, (B, kv.shape[1], D), "kv")
    return AttnArgs(H, D, int(d_v), float(scale), _ptr(q), _ptr(kv))


def workspace_size(op: int, B: int, Lq: int, Lk: int, k: int, H: int, d_v: int) -> int:
    return int(lib().dsa_workspace_size(int(op), B, Lq, Lk, k, H, d_v))


def workspace_size_args(op: int, ia: "IndexerArgs", k: int, H: int = 0, d_v: int = 0) -> int:
    """Exact workspace bytes of `op` for these indexer arguments (dsa_workspace_size_args)."""
    return int(lib().dsa_workspace_size_args(int(op), ctypes.byref(ia), int(k), int(H), int(d_v)))


def indexer_scores(q_I, q_scale, w, k_I, k_scale, q_offset=0, scores=None, stream=None):
    """fp32 [B, Lq, Lk] indexer scores, -inf above the causal boundary."""
    a = _indexer_args(q_I, q_scale, w, k_I, k_scale, q_offset)
    if scores is None:
        scores = torch.empty(a.B, a.Lq, a.Lk, dtype=torch.float32, device=w.device)
    _need(scores, torch.float32, (a.B, a.Lq, a.Lk), "scores")
    _check(lib().dsa_indexer_scores(ctypes.byref(a), _ptr(scores), _stream(stream)), "dsa_indexer_scores")
    return scores


def topk(scores, k, q_offset=0, indices=None, workspace=None, stream=None):
    """int32 [B, Lq, k] selected positions (ascending, -1 padded)."""
    B, Lq, Lk = scores.shape
    _need(scores, torch.float32, (B, Lq, Lk), "scores")
    if indices is None:
        indices = torch.empty(B, Lq, k, dtype=torch.int32, device=scores.device)
    _need(indices, torch.int32, (B, Lq, k), "indices")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().dsa_topk(_ptr(scores), B, Lq, Lk, int(q_offset), int(k), _ptr(indices), _ptr(workspace),
                          ws_bytes, _stream(stream)), "dsa_topk")
    return indices


def indexer_topk(q_I, q_scale, w, k_I, k_scale, k, q_offset=0, indices=None, sel_scores=None,
                 want_scores=True, workspace=None, stream=None):
    """Indexer with the top-k fused into it (no score matrix is written).

    Returns (indices int32 [B, Lq, k] ascending, -1 padded; sel_scores fp32 [B, Lq, k]
    or None: the score of each selected position, -inf on padding)."""
    a = _indexer_args(q_I, q_scale, w, k_I, k_scale, q_offset)
    dev = w.device
    if indices is None:
        indices = torch.empty(a.B, a.Lq, k, dtype=torch.int32, device=dev)
    _need(indices, torch.int32, (a.B, a.Lq, k), "indices")
    if sel_scores is None and want_scores:
        sel_scores = torch.empty(a.B, a.Lq, k, dtype=torch.float32, device=dev)
    if sel_scores is not None:
        _need(sel_scores, torch.float32, (a.B, a.Lq, k), "sel_scores")
    need = workspace_size_args(OP_INDEXER_TOPK, a, k)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().dsa_indexer_topk(ctypes.byref(a), int(k), _ptr(indices), _ptr(sel_scores), _ptr(workspace),
                                  nbytes, _stream(stream)), "dsa_indexer_topk")
    return indices, sel_scores


def _workspace(op, B, Lq, Lk, k, H, d_v, device, workspace, ia=None):
    need = workspace_size_args(op, ia, k, H, d_v) if ia is not None else workspace_size(op, B, Lq, Lk, k, H, d_v)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return workspace, nbytes


def sparse_attn(q, kv, indices, d_v, scale, out=None, lse=None, want_lse=True, workspace=None, stream=None):
    """bf16 [B, Lq, H, d_v] attention over the selected latent rows (+ fp32 lse [B, Lq, H])."""
    a = _attn_args(q, kv, d_v, scale)
    B, Lq, H, _ = q.shape
    Lk = kv.shape[1]
    k = indices.shape[-1]
    _need(indices, torch.int32, (B, Lq, k), "indices")
    if out is None:
        out = torch.empty(B, Lq, H, d_v, dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (B, Lq, H, d_v), "out")
    if lse is None and want_lse:
        lse = torch.empty(B, Lq, H, dtype=torch.float32, device=q.device)
    workspace, nbytes = _workspace(OP_SPARSE_ATTN, B, Lq, Lk, k, H, d_v, q.device, workspace)
    _check(lib().dsa_sparse_attn(ctypes.byref(a), B, Lq, Lk, _ptr(indices), k, _ptr(out), _ptr(lse),
                                 _ptr(workspace), nbytes, _stream(stream)), "dsa_sparse_attn")
    return out, lse


NOALLOC_SCRATCH_BYTES = 64 << 20   # DSA_NOALLOC_SCRATCH_BYTES


def sparse_attn_noalloc(q, kv, indices, d_v, scale, out, lse=None, stream=None):
    """sparse_attn into caller-provided `out` (and `lse`), with no device allocation:
    the split-k partials use the library's fixed scratch array (dsa_sparse_attn_noalloc)."""
    a = _attn_args(q, kv, d_v, scale)
    B, Lq, H, _ = q.shape
    Lk = kv.shape[1]
    k = indices.shape[-1]
    _need(indices, torch.int32, (B, Lq, k), "indices")
    _need(out, torch.bfloat16, (B, Lq, H, d_v), "out")
    if lse is not None:
        _need(lse, torch.float32, (B, Lq, H), "lse")
    _check(lib().dsa_sparse_attn_noalloc(ctypes.byref(a), B, Lq, Lk, _ptr(indices), k, _ptr(out), _ptr(lse),
                                         _stream(stream)), "dsa_sparse_attn_noalloc")
    return out, lse


def forward(q_I, q_scale, w, k_I, k_scale, q, kv, k, d_v, scale, q_offset=0, indices=None, out=None,
            lse=None, want_lse=True, workspace=None, stream=None, stage_events=None, sel_scores=None,
            low_memory=False):
    """Indexer -> top-k -> sparse attention.  Returns (indices, out, lse).

    The selection is staged (score matrix in the workspace, then the top-k
    kernel; the faster path) unless ``low_memory`` is set or the given
    ``workspace`` is too small for the score matrix, in which case it is fused
    into the indexer (dsa_indexer_topk).  Both give identical results.
    ``stage_events``: optional four torch.cuda.Event objects, recorded on the
    stream before the indexer, after the indexer, after the top-k (the same
    point when fused) and after the attention.  ``sel_scores``: optional fp32
    [B, Lq, k] tensor that receives the indexer score of every selected position.
    """
    ia = _indexer_args(q_I, q_scale, w, k_I, k_scale, q_offset)
    aa = _attn_args(q, kv, d_v, scale)
    B, Lq, Lk, H = ia.B, ia.Lq, ia.Lk, aa.H
    if indices is None:
        indices = torch.empty(B, Lq, k, dtype=torch.int32, device=q.device)
    _need(indices, torch.int32, (B, Lq, k), "indices")
    if out is None:
        out = torch.empty(B, Lq, H, d_v, dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (B, Lq, H, d_v), "out")
    if lse is None and want_lse:
        lse = torch.empty(B, Lq, H, dtype=torch.float32, device=q.device)
    if sel_scores is not None:
        _need(sel_scores, torch.float32, (B, Lq, k), "sel_scores")
    workspace, nbytes = _workspace(OP_FORWARD_LOWMEM if low_memory else OP_FORWARD, B, Lq, Lk, k, H, d_v,
                                   q.device, workspace, ia=ia)
    ev = None
    if stage_events is not None:
        if len(stage_events) != 4:
            raise ValueError("stage_events needs four events")
        for e in stage_events:          # torch creates the CUDA event on first use
            if not e.cuda_event:
                e.record(stream if stream is not None else torch.cuda.current_stream())
        ev = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in stage_events])
    _check(lib().dsa_forward_timed(ctypes.byref(ia), ctypes.byref(aa), int(k), _ptr(indices), _ptr(sel_scores),
                                   _ptr(out), _ptr(lse), _ptr(workspace), nbytes, _stream(stream), ev),
           "dsa_forward")
    return indices, out, lse


def indexer_kl_loss(q, kv, indices, lse, scores, d_v, scale, target=None, want_target=True, kl=None,
                    stream=None):
    """Forward of the indexer's training loss over the selected positions.

    Target p = the attention probabilities (from ``lse`` of sparse_attn on the same
    selection) summed over the heads and L1-normalised; loss per row =
    D_KL(p || softmax over the selected positions of ``scores``).  Returns
    (target fp32 [B, Lq, k] or None, kl fp32 [B, Lq]).
    """
    a = _attn_args(q, kv, d_v, scale)
    B, Lq, H, _ = q.shape
    Lk = kv.shape[1]
    k = indices.shape[-1]
    _need(indices, torch.int32, (B, Lq, k), "indices")
    _need(lse, torch.float32, (B, Lq, H), "lse")
    _need(scores, torch.float32, (B, Lq, Lk), "scores")
    if target is None and want_target:
        target = torch.empty(B, Lq, k, dtype=torch.float32, device=q.device)
    if target is not None:
        _need(target, torch.float32, (B, Lq, k), "target")
    if kl is None:
        kl = torch.empty(B, Lq, dtype=torch.float32, device=q.device)
    _need(kl, torch.float32, (B, Lq), "kl")
    _check(lib().dsa_indexer_kl_loss(ctypes.byref(a), B, Lq, Lk, _ptr(indices), k, _ptr(lse), _ptr(scores),
                                     _ptr(target), _ptr(kl), _stream(stream)), "dsa_indexer_kl_loss")
    return target, kl


def indexer_kl_loss_selected(q, kv, indices, lse, sel_scores, d_v, scale, target=None, want_target=True, kl=None,
                             stream=None):
    """indexer_kl_loss with the scores given per index slot (fp32 [B, Lq, k], as
    returned by indexer_topk or forward(sel_scores=...)) instead of a full matrix."""
    a = _attn_args(q, kv, d_v, scale)
    B, Lq, H, _ = q.shape
    Lk = kv.shape[1]
    k = indices.shape[-1]
    _need(indices, torch.int32, (B, Lq, k), "indices")
    _need(lse, torch.float32, (B, Lq, H), "lse")
    _need(sel_scores, torch.float32, (B, Lq, k), "sel_scores")
    if target is None and want_target:
        target = torch.empty(B, Lq, k, dtype=torch.float32, device=q.device)
    if target is not None:
        _need(target, torch.float32, (B, Lq, k), "target")
    if kl is None:
        kl = torch.empty(B, Lq, dtype=torch.float32, device=q.device)
    _need(kl, torch.float32, (B, Lq), "kl")
    _check(lib().dsa_indexer_kl_loss_selected(ctypes.byref(a), B, Lq, Lk, _ptr(indices), k, _ptr(lse),
                                              _ptr(sel_scores), _ptr(target), _ptr(kl), _stream(stream)),
           "dsa_indexer_kl_loss_selected")
    return target, kl


def device_status(clear: bool = True) -> int:
    """0 (DSA_OK) or 5 (DSA_ERR_TIMEOUT): whether a device-side wait gave up.  Synchronises."""
    return int(lib().dsa_device_status(1 if clear else 0))


def selftest_wait_timeout(spin_limit: int = 1 << 16, stream=None) -> int:
    return int(lib().dsa_selftest_wait_timeout(int(spin_limit), _stream(stream)))
