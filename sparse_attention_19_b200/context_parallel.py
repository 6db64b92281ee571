"""Context-parallel prefill of one long sequence over several GPUs (one process each).

Query rows are independent once every key is available (the indexer, the
top-k and the attention of row t read keys 0..t only), so a long prefill splits
by query chunks.  The causal triangle makes late chunks dearer than early ones;
with the sequence cut into 2W chunks per round, rank r takes chunk r and chunk
2W-1-r of every round (zig-zag), which gives every rank the same number of
causal pairs.  Each rank holds the key side (indexer keys, their scales, latent
KV rows) of its own chunks; one exchange step, an all-gather over the process
group, assembles the whole sequence's key side on every rank, in sequence order.
Each rank then runs the single-GPU forward pass (dsa_forward) on its own query
chunks with q_offset = chunk start and the key prefix up to the chunk's end.

Only B = 1 is supported (a long single sequence, the case that needs it).  The
all-gather is torch.distributed's (NCCL on GPUs); nothing here computes any of
the method's arithmetic.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

KEY_FIELDS = ("k_I", "k_scale", "kv")


def zigzag_chunks(n_chunks: int, world: int, rank: int) -> list[int]:
    """Chunk indices (ascending) that `rank` owns out of n_chunks, a multiple of 2*world."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    if n_chunks % (2 * world):
        raise ValueError(f"n_chunks={n_chunks} must be a multiple of 2*world={2 * world}")
    out = []
    for base in range(0, n_chunks, 2 * world):
        out += [base + rank, base + 2 * world - 1 - rank]
    return sorted(out)


def causal_pairs_of(chunks, chunk: int) -> int:
    """Causal (query, key) pairs of the given query chunks: row t sees t + 1 keys."""
    total = 0
    for c in chunks:
        first, last = c * chunk + 1, (c + 1) * chunk
        total += (first + last) * chunk // 2
    return total


def local_key_side(full: dict, chunks, chunk: int) -> dict:
    """This rank's share of the key side: its chunks' rows, concatenated in chunk order."""
    return {f: torch.cat([full[f][:, c * chunk:(c + 1) * chunk] for c in chunks], dim=1).contiguous()
            for f in KEY_FIELDS}


def gather_key_side(local: dict, n_chunks: int, chunk: int, world: int, rank: int, group=None) -> dict:
    """All-gather every rank's key-side chunks into whole-sequence tensors [1, n_chunks*chunk, ...].

    ``local`` holds this rank's chunks (as ``local_key_side`` lays them out).  Each
    round of 2*world chunks takes two all-gathers per tensor: one for the ranks'
    first chunks (positions r) and one for their second chunks (positions
    2W-1-r); the received chunks land directly in their sequence positions.
    """
    mine = zigzag_chunks(n_chunks, world, rank)
    out = {}
    for f in KEY_FIELDS:
        t = local[f]
        if t.shape[0] != 1:
            raise ValueError("context parallelism supports B = 1")
        full = torch.empty((1, n_chunks * chunk) + tuple(t.shape[2:]), dtype=t.dtype, device=t.device)
        for j, base in enumerate(range(0, n_chunks, 2 * world)):
            for second in (0, 1):
                pos = [base + (2 * world - 1 - r if second else r) for r in range(world)]
                dst = [full[:, p * chunk:(p + 1) * chunk] for p in pos]
                src = t[:, (2 * j + second) * chunk:(2 * j + second + 1) * chunk].contiguous()
                if world == 1:
                    dst[0].copy_(src)
                else:
                    recv = [torch.empty_like(src) for _ in range(world)]
                    dist.all_gather(recv, src, group=group)
                    for d, r in zip(dst, recv):
                        d.copy_(r)
        out[f] = full
    return out


def cp_forward(queries: dict, local_keys: dict, n_chunks: int, chunk: int, k: int, d_v: int, scale: float,
               world: int, rank: int, group=None, stream=None):
    """Context-parallel DSA forward of this rank's query chunks.

    ``queries`` maps each chunk index this rank owns to its query side
    (q_I [1, chunk, H_I, d_I], q_scale [1, chunk], w [1, chunk, H_I],
    q [1, chunk, H, d_qk]); ``local_keys`` is this rank's key side.  Returns
    {chunk index: (indices, out, lse)}.
    """
    import sparse_attention_19_b200 as dsa
    mine = zigzag_chunks(n_chunks, world, rank)
    if sorted(queries) != mine:
        raise ValueError(f"rank {rank} owns chunks {mine}")
    keys = gather_key_side(local_keys, n_chunks, chunk, world, rank, group)
    results = {}
    for c in mine:
        qs = queries[c]
        q_offset = c * chunk
        Lk = q_offset + chunk
        results[c] = dsa.forward(qs["q_I"], qs["q_scale"], qs["w"], keys["k_I"][:, :Lk], keys["k_scale"][:, :Lk],
                                 qs["q"], keys["kv"][:, :Lk], k, d_v, scale, q_offset, stream=stream)
    return results
