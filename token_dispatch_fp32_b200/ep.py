"""Expert-parallel dispatch and combine across ranks (Kimi K2 "Add shared
output" page, moe_infer, the ep_size > 1 branch).

With ep ranks, rank r owns the routed experts [r*E_loc, (r+1)*E_loc),
E_loc = N_r / ep (the page's tokens_per_expert.view(ep_size, -1)).  One
dispatch per rank, in the page's order:

  1. counts, offsets, perm, inv of the rank's own top-k ids     (mr_dispatch)
  2. its token rows in expert-sorted order                        (mr_gather_rows)
  3. all_to_all_single of tokens_per_expert: rank r learns how many rows
     each source sends it per local expert                        (exchange_counts)
  4. the rows themselves, variable splits                         (exchange_rows)
  5. the received rows sorted by local expert, stable             (mr_ep_recv_order,
                                                                   mr_gather_rows)
and after the local experts ran on the sorted rows, the way back:

  6. the outputs back into received order (new_x[gatherd_idxs] = outs)
  7. the reverse all-to-all to the rows' sources                  (exchange_rows)
  8. the weighted combine and shared add on the source            (mr_combine)

The collectives are torch.distributed calls on the process group (NCCL over
NVLink on GPUs; any backend that has all_to_all_single works); rows travel
as raw bytes, so any row dtype goes through every backend.  As on the page,
the split sizes are read back to the host once per dispatch because the
variable-split all-to-all takes them as host integers (here one copy of
2*N_r integers).  Every local step runs in libmr.so's
kernels; this module only orders the steps, sums the split sizes on the host
and moves buffers.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist

from . import _binding as mr


def split_sizes(counts, recv_counts, ep: int):
    """Host bookkeeping of one dispatch, from this rank's tokens_per_expert
    ([N_r]) and what the count exchange delivered ([ep * E_loc], source-major),
    both flat host integer sequences: the rows this rank sends to each rank
    (tokens_per_ep_rank: its counts summed over that rank's expert block) and
    the rows it receives from each (output_splits: the received counts summed
    per source).  Returns two lists of ep ints."""
    counts = [int(c) for c in counts]
    recv = [int(c) for c in recv_counts]
    if len(counts) % ep or len(recv) != len(counts):
        raise ValueError(f"{len(counts)} experts do not split over {ep} ranks")
    E_loc = len(counts) // ep
    send_splits = [sum(counts[r * E_loc:(r + 1) * E_loc]) for r in range(ep)]
    recv_splits = [sum(recv[s * E_loc:(s + 1) * E_loc]) for s in range(ep)]
    return send_splits, recv_splits


def exchange_counts(counts: torch.Tensor, group=None):
    """all_to_all_single of tokens_per_expert ([N_r] int32): rank r receives
    from every source s that source's counts for r's local experts.
    Returns recv_counts [ep, E_loc] (on counts' device) and the host split
    sizes (send, recv), read back with one copy of 2*N_r integers."""
    ep = dist.get_world_size(group)
    if counts.numel() % ep:
        raise ValueError(f"{counts.numel()} experts do not split over {ep} ranks")
    recv = torch.empty_like(counts)
    dist.all_to_all_single(recv, counts.contiguous(), group=group)
    host = torch.cat([counts.view(-1), recv.view(-1)]).cpu().tolist()
    n = counts.numel()
    send_splits, recv_splits = split_sizes(host[:n], host[n:], ep)
    return recv.view(ep, -1), send_splits, recv_splits


def exchange_rows(rows: torch.Tensor, send_splits, recv_splits, group=None) -> torch.Tensor:
    """Variable-split all-to-all of [n, d] rows: rows[sum(send[:s]) :
    sum(send[:s+1])] go to rank s; the result holds what every source sent
    this rank, in source order.  The rows travel as bytes."""
    rows = rows.contiguous()
    if rows.numel() == 0:  # an empty tensor may carry zero strides: give it plain ones
        rows = torch.empty(rows.shape, dtype=rows.dtype, device=rows.device)
    d_bytes = rows.shape[1] * rows.element_size()
    out = torch.empty((int(sum(recv_splits)), rows.shape[1]), dtype=rows.dtype,
                      device=rows.device)
    dist.all_to_all_single(out.view(torch.uint8).view(-1, d_bytes),
                           rows.view(torch.uint8).view(-1, d_bytes),
                           output_split_sizes=list(recv_splits),
                           input_split_sizes=list(send_splits), group=group)
    return out


@dataclasses.dataclass
class EPHandle:
    """What the way back needs: the source-side dispatch (inv_perm) and the
    receive-side order and split sizes of one dispatch."""
    inv_perm: torch.Tensor
    order: torch.Tensor
    send_splits: list
    recv_splits: list


def ep_dispatch(x_rows, idx, N_r, group=None, stream=None):
    """Dispatch of this rank's tokens to the experts' owners.  x_rows [T,d]
    (bf16 or fp32), idx [T,k] int32 top-k ids.  Returns (local_rows
    [R,d] sorted by local expert, local_counts [E_loc], local_offsets
    [E_loc+1], handle)."""
    T, k = idx.shape
    counts, _, perm, inv = mr.mr_dispatch(idx, N_r, stream=stream)
    xs = mr.mr_gather_rows(x_rows, k, perm=perm, inv_perm=inv, stream=stream)
    recv_counts, send_splits, recv_splits = exchange_counts(counts, group)
    recv_rows = exchange_rows(xs, send_splits, recv_splits, group)
    R = int(sum(recv_splits))
    order, _, local_counts, local_offsets = mr.mr_ep_recv_order(recv_counts, R, stream=stream)
    local_rows = mr.mr_gather_rows(recv_rows, 1, perm=order, stream=stream)
    return local_rows, local_counts, local_offsets, EPHandle(inv, order, send_splits,
                                                             recv_splits)


def ep_combine(local_out, handle: EPHandle, w, shared=None, group=None, stream=None):
    """The way back: local expert outputs [R,d] (sorted by local expert) to
    their sources, then the weighted combine with w [T,k] and the shared
    output [T,d] (or None) on the source.  Returns y [T,d]."""
    received = mr.mr_gather_rows(local_out, 1, inv_perm=handle.order, stream=stream)
    back = exchange_rows(received, handle.recv_splits, handle.send_splits, group)
    return mr.mr_combine(back, w, handle.inv_perm, shared, stream=stream)
