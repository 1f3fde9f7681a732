"""One sequence's prefill split over several GPUs by query (one process per GPU).

The layer's rows are independent once every GPU holds the whole sequence's keys: a query row
needs the block means of all past index keys (its selection) and the K/V rows it selected, and
nothing from other query rows (Step 5 Preview pages, mo.ai.kr "Step 5 Preview agentic work
design", section "model structure and training stability": each KV group selects and attends on
its own). So the queries are split and the keys are gathered:

* zig-zag ranges: the sequence is cut into 2 * world equal chunks and rank r takes chunks r and
  2 * world - 1 - r, which balances the causal work (a late chunk attends to more history only
  up to the k/B budget, an early one to less);
* every rank produces K, V and k_idx for its own rows (in a model, the projections of its
  tokens), and one all-gather per tensor over NCCL (NVLink / NVSwitch) gives every rank the whole
  sequence, reordered from the ranks' chunk order into token order;
* each rank then runs sgqa_forward_rows for its two ranges: bit-identical to the same rows of a
  single-GPU sgqa_forward.

torch.distributed carries the collective; every computation of the layer runs in libsgqa's
kernels.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def zigzag_ranges(T: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """The two query ranges [t0, t1) of `rank`: chunks rank and 2 * world - 1 - rank of 2 * world
    equal chunks (T must be a multiple of 2 * world)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    if T % (2 * world) != 0:
        raise ValueError(f"T = {T} is not a multiple of 2 * world = {2 * world}")
    c = T // (2 * world)
    first, second = rank, 2 * world - 1 - rank
    return [(first * c, (first + 1) * c), (second * c, (second + 1) * c)]


def chunk_owner(chunk: int, world: int) -> Tuple[int, int]:
    """(rank, slot) holding chunk `chunk` of 2 * world: slot 0 is a rank's first range."""
    if chunk < world:
        return chunk, 0
    return 2 * world - 1 - chunk, 1


def gather_sequence(local: Sequence, world: int, group=None):
    """All-gather a tensor whose rows are split zig-zag over the ranks.

    local: this rank's two chunks, each [batch, chunk, ...] (contiguous, same shape on every
    rank). Returns [batch, 2 * world * chunk, ...] in token order."""
    import torch
    import torch.distributed as dist
    a, b = local
    if a.shape != b.shape:
        raise ValueError("both chunks of a rank have the same shape")
    mine = torch.stack([a, b])  # [2, batch, chunk, ...]
    parts = [torch.empty_like(mine) for _ in range(world)]
    if world > 1:
        dist.all_gather(parts, mine.contiguous(), group=group)
    else:
        parts[0].copy_(mine)
    chunks = [parts[r][s] for r, s in (chunk_owner(c, world) for c in range(2 * world))]
    return torch.cat(chunks, dim=1).contiguous()


def prefill_rows(dims, ranges, q_rows, gate_rows, q_idx_rows, k, v, k_idx, out_rows, ws, sel_rows=None, stream=None):
    """This rank's share of the layer: sgqa_forward_rows for each of its ranges.

    q_rows, gate_rows, q_idx_rows, out_rows (and sel_rows if given): one tensor per range, each
    [batch, t1 - t0, ...]; k, v, k_idx: the whole sequence (from gather_sequence)."""
    import block_sparse_long_kbar_b200 as sg
    for i, (t0, t1) in enumerate(ranges):
        sg.sgqa_forward_rows(dims, t0, t1, q_rows[i], k, v, q_idx_rows[i], k_idx, gate_rows[i], out_rows[i], ws,
                             sel_out_rows=None if sel_rows is None else sel_rows[i], stream=stream)
