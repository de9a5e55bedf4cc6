"""Splitting the decode work of one step across GPUs (one process per GPU, torch.distributed).

Two splits, both exact (the Adaptive KV Streaming + RDNA 4 announcement, wqu.guru, method
list: partial attention results over disjoint key sets are combined by online log-sum-exp):

* by unit: the (layer, KV head) units are independent, so each rank decodes a contiguous
  range of them and no data crosses between ranks (``unit_range``);
* by sequence: the pages of every unit are split into contiguous ranges, each rank decodes
  its range with ``kvattn_decode`` (its own (o, lse) per query row), the partials are
  all-gathered and merged with ``kvattn_merge_lse`` (``SequenceShardedDecode``).  Only
  (o, lse) crosses the ranks: rows x (256 + 1) floats per rank and layer.

Host logic only; every computation runs in the CUDA library.  Collectives use the caller's
process group (NCCL between GPUs); no kernel here reads another GPU's memory.
"""
from __future__ import annotations


def balanced_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of rank's share of n items split into `world` contiguous ranges whose
    sizes differ by at most one (the first n % world ranges are one longer)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad split")
    q, r = divmod(n, world)
    start = rank * q + min(rank, r)
    return start, start + q + (1 if rank < r else 0)


def unit_range(n_layers: int, n_kv_heads: int, world: int, rank: int) -> list[tuple[int, int]]:
    """The (layer, KV head) units this rank decodes, in layer-major order."""
    a, b = balanced_range(n_layers * n_kv_heads, world, rank)
    return [(u // n_kv_heads, u % n_kv_heads) for u in range(a, b)]


def page_range(n_pages: int, world: int, rank: int) -> tuple[int, int]:
    """This rank's contiguous range of a unit's page list."""
    return balanced_range(n_pages, world, rank)


def gather_partials(o, lse, group=None):
    """All-gathers every rank's (o [rows][D], lse [rows]) into (o_all [world][rows][D],
    lse_all [world][rows]) in rank order."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    o_all = torch.empty((world,) + tuple(o.shape), dtype=o.dtype, device=o.device)
    lse_all = torch.empty((world,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
    # all_gather into views of one buffer: NCCL and gloo both take this form
    dist.all_gather(list(o_all.unbind(0)), o.contiguous(), group=group)
    dist.all_gather(list(lse_all.unbind(0)), lse.contiguous(), group=group)
    return o_all, lse_all


class SequenceShardedDecode:
    """Decode of one layer with every unit's page list split across the ranks of `group`.

    The caller passes the full page list of each KV head (device int32 [H_kv][max_pages],
    logical ids optional); this rank attends over its page_range of every head's list (the
    whole list must be valid on every rank, e.g. a replicated page table) and writes the merged
    (out, lse) of all ranks."""

    def __init__(self, kv, desc, n_q: int, max_pages: int, group=None):
        import torch
        import torch.distributed as dist

        self.kv, self.desc, self.n_q, self.group = kv, desc, n_q, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.a, self.b = page_range(max_pages, self.world, self.rank)
        self.n_local = self.b - self.a
        self.rows = n_q * desc.n_q_heads
        dev = torch.device("cuda", torch.cuda.current_device())
        self.ws_bytes = kv.kvattn_decode_workspace_size(desc, n_q, max(self.n_local, 1))
        self.ws = torch.zeros(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)
        self.o_part = torch.empty((self.rows, 256), device=dev)
        self.l_part = torch.empty((self.rows,), device=dev)
        self.max_pages = max_pages

    def __call__(self, q, q_pos, page_list, page_logical, out, lse) -> None:
        import torch

        H = self.desc.n_kv_heads
        # this rank's slice of every head's list (logical ids default to the list position)
        pl = page_list[:, self.a:self.b].contiguous()
        if page_logical is None:
            page_logical = torch.arange(self.max_pages, dtype=torch.int32, device=pl.device).expand(H, -1)
        lg = page_logical[:, self.a:self.b].contiguous()
        n_pages = torch.full((H,), self.n_local, dtype=torch.int32, device=pl.device)
        self.kv.kvattn_decode(self.desc, q, self.n_q, q_pos, pl, lg, n_pages, self.n_local,
                              self.o_part.view(self.n_q, -1, 256), self.l_part.view(self.n_q, -1), self.ws,
                              self.ws_bytes)
        o_all, l_all = gather_partials(self.o_part, self.l_part, self.group)
        self.kv.kvattn_merge_lse(o_all, l_all, self.world, self.rows, 256, out, lse)
