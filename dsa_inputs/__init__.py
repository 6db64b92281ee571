"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) forward pass.

This module is shared by the oracle tests, the CUDA parity tests and the
benchmark.  It only draws random numbers and stores them in the input formats
the method consumes (FP8 e4m3 indexer queries/keys with per-token fp32 scales,
bf16 indexer weights, bf16 MLA queries and latent KV rows).  It performs none of
the method's arithmetic: no scores, no selection, no attention.

Shapes follow the workloads of the DeepSeek-V3.2 technical-report summary
("DSA: внимание только к важному", lightning-indexer and top-k sections): a few
indexer heads, an FP8 indexer, k = 2048 selected positions out of a context of
up to 128K tokens, and MLA in its MQA form where one latent KV row of width
576 (512 latent + 64 rope) is shared by all 128 query heads.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    """One DSA forward problem.

    Query ``i`` of batch ``b`` sits at sequence position ``q_offset + i`` and
    may attend to keys ``0 .. q_offset + i`` (keys ``0 .. Lk-1`` exist).
    """

    name: str
    B: int
    Lq: int
    Lk: int
    q_offset: int
    H_I: int
    d_I: int
    k: int
    H: int
    D: int
    Dv: int
    scale: float
    integer_indexer: bool = False     # q_I/k_I small integers, w integers, scales 1
    salient_frac: float = 0.0         # fraction of keys whose k_I row is scaled by salient_gain
    salient_gain: float = 4.0
    chunk: int = 0                    # >0: queries are processed in chunks of this many rows
    description: str = ""

    @property
    def causal_pairs(self) -> int:
        """Number of (query, key) pairs with key position <= query position."""
        first = self.q_offset + 1
        last = self.q_offset + self.Lq
        per_batch = (first + last) * self.Lq // 2
        return per_batch * self.B

    @property
    def selected_pairs(self) -> int:
        """Number of (query, key) pairs attention runs over: min(k, t+1) per query."""
        total = 0
        for t in range(self.q_offset, self.q_offset + self.Lq):
            total += min(self.k, t + 1)
        return total * self.B

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


_SCALE = 1.0 / math.sqrt(192.0)

WORKLOADS = {
    "tiny": Workload(
        "tiny", B=1, Lq=1024, Lk=1024, q_offset=0, H_I=4, d_I=64, k=128,
        H=16, D=192, Dv=128, scale=_SCALE, integer_indexer=True,
        description="batch 1, L=1024 causal; integer-valued FP8 indexer (exact in fp32)"),
    "prefill_8k": Workload(
        "prefill_8k", B=1, Lq=8192, Lk=8192, q_offset=0, H_I=64, d_I=128, k=2048,
        H=128, D=576, Dv=512, scale=_SCALE,
        description="prefill L=8192, N(0,1) FP8 indexer with per-token scales"),
    "prefill_32k": Workload(
        "prefill_32k", B=1, Lq=32768, Lk=32768, q_offset=0, H_I=64, d_I=128, k=2048,
        H=128, D=576, Dv=512, scale=_SCALE, salient_frac=0.05,
        description="prefill L=32768, 5% salient indexer keys (norm x4)"),
    "decode_128k": Workload(
        "decode_128k", B=64, Lq=1, Lk=131072, q_offset=131071, H_I=64, d_I=128, k=2048,
        H=128, D=576, Dv=512, scale=_SCALE,
        description="decode: 64 sequences x 131072 cached tokens, 1 new query each"),
    "prefill_2k": Workload(
        "prefill_2k", B=1, Lq=2048, Lk=2048, q_offset=0, H_I=64, d_I=128, k=2048,
        H=128, D=576, Dv=512, scale=_SCALE,
        description="short prefill L=2048 = k: every position selected (dense causal attention)"),
    "prefill_128k": Workload(
        "prefill_128k", B=1, Lq=131072, Lk=131072, q_offset=0, H_I=64, d_I=128, k=2048,
        H=128, D=576, Dv=512, scale=_SCALE, salient_frac=0.05, chunk=4096,
        description="prefill L=131072 in 4096-query chunks against the growing causal key set"),
}


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    # Independent sub-stream per tensor: a fixed odd multiplier spreads the ids.
    g.manual_seed((seed * 1_000_003 + stream * 7919 + 17) % (2**63 - 1))
    return g


def quantize_e4m3_per_row(x: torch.Tensor, row_dims: int):
    """Store ``x`` as e4m3 codes with one fp32 scale per leading-``row_dims`` index.

    scale = amax / 448 over the trailing dimensions; codes = RNE(x / scale)
    saturated to +-448.  Returns (uint8 codes, fp32 scales).
    """
    lead = x.shape[:row_dims]
    flat = x.reshape(*lead, -1).float()
    amax = flat.abs().amax(dim=-1).clamp_min(1e-30)
    scale = (amax / E4M3_MAX).float()
    y = (flat / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return codes.contiguous(), scale.contiguous()


def int_to_e4m3(x: torch.Tensor) -> torch.Tensor:
    """Small integers (|x| <= 16) are exact in e4m3; return their codes."""
    return x.float().to(torch.float8_e4m3fn).view(torch.uint8).contiguous()


def salient_positions(wl: Workload, seed: int, device="cpu") -> torch.Tensor:
    """round(salient_frac * Lk) key positions drawn without replacement."""
    n = int(round(wl.salient_frac * wl.Lk))
    if n == 0:
        return torch.empty(0, dtype=torch.int64, device=device)
    g = _gen(seed, 90, "cpu")
    perm = torch.randperm(wl.Lk, generator=g)
    return perm[:n].sort().values.to(device)


def make_key_side(wl: Workload, device="cpu", seed: int = 0) -> dict:
    """Indexer keys (+scales) and latent KV rows for all Lk positions."""
    B, Lk = wl.B, wl.Lk
    out = {}
    if wl.integer_indexer:
        g = _gen(seed, 3, device)
        kint = torch.randint(-4, 5, (B, Lk, wl.d_I), generator=g, device=device)
        out["k_I"] = int_to_e4m3(kint)
        out["k_scale"] = torch.ones(B, Lk, dtype=torch.float32, device=device)
    else:
        g = _gen(seed, 3, device)
        kf = torch.randn(B, Lk, wl.d_I, generator=g, device=device, dtype=torch.float32)
        if wl.salient_frac > 0:
            pos = salient_positions(wl, seed, device)
            kf[:, pos, :] *= wl.salient_gain
        out["k_I"], out["k_scale"] = quantize_e4m3_per_row(kf, 2)
        del kf
    g = _gen(seed, 6, device)
    out["kv"] = torch.randn(B, Lk, wl.D, generator=g, device=device, dtype=torch.bfloat16)
    return out


def make_query_side(wl: Workload, device="cpu", seed: int = 0, chunk_index: int = -1,
                    Lq: int | None = None) -> dict:
    """Indexer queries (+scales), indexer weights and MLA queries.

    ``chunk_index >= 0`` draws the queries of one chunk of a chunked workload
    from its own sub-stream, so that a chunk can be regenerated on its own.
    """
    B = wl.B
    Lq = wl.Lq if Lq is None else Lq
    base = 0 if chunk_index < 0 else 1000 * (chunk_index + 1)
    out = {}
    if wl.integer_indexer:
        g = _gen(seed, base + 1, device)
        qint = torch.randint(-4, 5, (B, Lq, wl.H_I, wl.d_I), generator=g, device=device)
        out["q_I"] = int_to_e4m3(qint)
        out["q_scale"] = torch.ones(B, Lq, dtype=torch.float32, device=device)
        g = _gen(seed, base + 2, device)
        out["w"] = torch.randint(-2, 3, (B, Lq, wl.H_I), generator=g, device=device).to(torch.bfloat16)
    else:
        g = _gen(seed, base + 1, device)
        qf = torch.randn(B, Lq, wl.H_I, wl.d_I, generator=g, device=device, dtype=torch.float32)
        out["q_I"], out["q_scale"] = quantize_e4m3_per_row(qf, 2)
        del qf
        g = _gen(seed, base + 2, device)
        out["w"] = (torch.randn(B, Lq, wl.H_I, generator=g, device=device, dtype=torch.float32)
                    * math.sqrt(1.0 / 8.0)).to(torch.bfloat16)
    g = _gen(seed, base + 5, device)
    out["q"] = torch.randn(B, Lq, wl.H, wl.D, generator=g, device=device, dtype=torch.bfloat16)
    return out


def make_inputs(wl: Workload, device="cpu", seed: int = 0) -> dict:
    """All inputs of an unchunked workload."""
    d = make_key_side(wl, device, seed)
    d.update(make_query_side(wl, device, seed))
    return d


def to_host(d: dict) -> dict:
    return {k: v.detach().to("cpu").contiguous() for k, v in d.items()}
