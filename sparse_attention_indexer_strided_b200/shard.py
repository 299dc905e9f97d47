"""Row sharding of one top-k batch across GPUs (one process per GPU).

Rows are independent: row r's result depends on row r's logits alone (the
pages' operation is per row, addressed by the row stride; vLLM PR #42169
report, "实现拆解"). A batch therefore splits into contiguous row blocks, one
per rank, and each rank calls ``dsa_topk`` on its own block with its own
stream: there is no exchange on the data path. A rank holds the logits of its
own rows only, as an indexer rank would.

``gather_rows`` is the one optional collective: an all-gather of the int32
results for a consumer that needs every row on every rank.
"""
from __future__ import annotations

from typing import Tuple

import torch


def row_block(num_rows: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [r0, r1) of rank ``rank`` among ``world``: contiguous blocks whose
    sizes differ by at most one, in rank order, covering [0, num_rows)."""
    if world < 1 or not (0 <= rank < world) or num_rows < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, num_rows >= 0")
    return num_rows * rank // world, num_rows * (rank + 1) // world


def max_block(num_rows: int, world: int) -> int:
    """The largest block any rank gets (the padded size of an all-gather)."""
    return -(-num_rows // world) if world > 0 else 0


def gather_rows(out_block: torch.Tensor, num_rows: int, world: int, rank: int, group=None) -> torch.Tensor:
    """All-gather the ranks' ``[r1 - r0, k]`` int32 result blocks into the
    full ``[num_rows, k]`` result on every rank (blocks padded to the largest
    block for the collective, then trimmed)."""
    import torch.distributed as dist

    r0, r1 = row_block(num_rows, world, rank)
    k = int(out_block.shape[1])
    if tuple(out_block.shape) != (r1 - r0, k):
        raise ValueError("out_block must be [r1 - r0, k] for this rank")
    mb = max_block(num_rows, world)
    pad = torch.full((mb, k), -1, dtype=out_block.dtype, device=out_block.device)
    pad[: r1 - r0] = out_block
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    out = torch.empty((num_rows, k), dtype=out_block.dtype, device=out_block.device)
    for r in range(world):
        a, b = row_block(num_rows, world, r)
        out[a:b] = parts[r][: b - a]
    return out


__all__ = ["row_block", "max_block", "gather_rows"]
