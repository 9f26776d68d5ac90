"""Row-sharded flat prefill of one long sequence over several GPUs (one process per GPU).

The query rows of a causal prefill are independent given the keys (ADIndex §3, Eqs. (1)-(2):
row t scores keys s <= t), so one problem splits across ranks by rows with no exchange inside
the indexer. What does cross ranks:
  * the keys, once per call: a rank that holds only its slice of the sequence's keys gets the
    whole key array with one all-gather (torch.distributed, NCCL over NVLink on GPUs);
  * the Top-K rows, once at the end: every rank's rows are gathered to rank 0 (or to all).

Rows are assigned in units of `unit` consecutive rows, longest first, each unit to the rank
with the least work so far (the LPT rule): row t costs its q_pos0 + t + 1 visible keys, so
the causal triangle's long rows are spread before the short ones fill the gaps. Every rank
computes the same assignment from (T, q_pos0, world, unit); no message carries it.

The per-rank work is any callable index_fn(q_rows, w_rows, k, K, q_pos0) -> Top-K rows
[n, K] int32 (by default the library's adx_index_prefill through indexer.index_prefill); it
only ever sees whole units of consecutive rows.
"""

import heapq

import torch


def unit_cost(q_pos0, r0, r1):
    """Visible keys summed over rows r0 .. r1-1 at positions q_pos0 + r: the row's work."""
    n = r1 - r0
    return n * (q_pos0 + 1) + (r0 + r1 - 1) * n // 2


def partition_rows(T, q_pos0, world, unit=64):
    """Longest-first assignment of units of `unit` rows to `world` ranks. Returns
    (ranges, loads): ranges[rank] = ascending list of (r0, r1) row ranges; loads[rank] = the
    rank's summed cost."""
    if T <= 0 or world <= 0 or unit <= 0:
        raise ValueError("T, world and unit must be positive")
    units = [(r0, min(T, r0 + unit)) for r0 in range(0, T, unit)]
    units.sort(key=lambda u: (-unit_cost(q_pos0, *u), u[0]))
    heap = [(0, rank) for rank in range(world)]
    ranges = [[] for _ in range(world)]
    loads = [0] * world
    for r0, r1 in units:
        load, rank = heapq.heappop(heap)
        ranges[rank].append((r0, r1))
        loads[rank] = load + unit_cost(q_pos0, r0, r1)
        heapq.heappush(heap, (loads[rank], rank))
    for rs in ranges:
        rs.sort()
    return ranges, loads


def all_gather_keys(k_local, group=None):
    """The whole key array [S, d] from every rank's contiguous slice k_local [S_r, d] (ranks in
    order; slices may differ in length)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    n = torch.tensor([k_local.shape[0]], dtype=torch.int64, device=k_local.device)
    sizes = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(sizes, n, group=group)
    sizes = [int(x.item()) for x in sizes]
    most = max(sizes)
    pad = torch.zeros((most,) + tuple(k_local.shape[1:]), dtype=k_local.dtype,
                      device=k_local.device)
    pad[: k_local.shape[0]] = k_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:s] for p, s in zip(parts, sizes)], dim=0).contiguous()


def _index_prefill(q, w, k, K, q_pos0, q_scale=None, k_scale=None):
    from . import indexer
    idx, _, _ = indexer.index_prefill(q, w, k, K, q_scale=q_scale, k_scale=k_scale,
                                      q_pos0=q_pos0)
    return idx


def sharded_prefill(q, w, k, K, q_pos0=0, unit=64, index_fn=None, to_all=False, group=None,
                    q_scale=None, k_scale=None):
    """Flat prefill of the T rows of q [T, H, d] (positions q_pos0 ..) against the whole key
    array k [S, d], split over the process group's ranks. Each rank indexes its rows, then the
    rows are gathered: the full [T, K] int32 Top-K on rank 0 (on every rank with to_all), None
    on the others. Every rank must pass the same q, w (or at least their rows it owns), k, K
    and q_pos0."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    T = q.shape[0]
    ranges, _ = partition_rows(T, q_pos0, world, unit)
    if index_fn is None:
        def index_fn(qr, wr, kk, KK, p0):
            r0 = p0 - q_pos0
            qs = None if q_scale is None else q_scale[r0:r0 + qr.shape[0]]
            return _index_prefill(qr, wr, kk, KK, p0, qs, k_scale)
    mine = [index_fn(q[r0:r1], w[r0:r1], k, K, q_pos0 + r0) for r0, r1 in ranges[rank]]
    dev = q.device
    n_mine = sum(r1 - r0 for r0, r1 in ranges[rank])
    most = max(sum(r1 - r0 for r0, r1 in rs) for rs in ranges)
    buf = torch.full((most, K), -1, dtype=torch.int32, device=dev)
    if mine:
        buf[:n_mine] = torch.cat(mine, dim=0)
    if to_all:
        parts = [torch.empty_like(buf) for _ in range(world)]
        dist.all_gather(parts, buf, group=group)
    else:
        parts = [torch.empty_like(buf) for _ in range(world)] if rank == 0 else None
        dist.gather(buf, parts, dst=dist.get_global_rank(group, 0) if group else 0, group=group)
    if parts is None:
        return None
    out = torch.empty((T, K), dtype=torch.int32, device=dev)
    for rk, rs in enumerate(ranges):
        at = 0
        for r0, r1 in rs:
            out[r0:r1] = parts[rk][at:at + (r1 - r0)]
            at += r1 - r0
    return out
