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

The second half of the module does the same exchange over peer memory
(ep_dispatch_p2p / ep_combine_p2p): every rank maps the others' receive and
output buffers (PeerBuffers), an all-gather of tokens_per_expert replaces
the count all-to-all, one kernel writes each row straight into its owner's
receive buffer at its final local-expert-sorted place (steps 2, 4 and 5 in
one pass, no host read-back), and one kernel combines straight out of the
owners' output buffers (steps 6-8).  Collectives on the stream order the
ranks' steps; no kernel waits on another rank.
"""
from __future__ import annotations

import dataclasses
import threading

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


# ---- the exchange over peer memory ------------------------------------------

_opened = {}  # (device index, allocation handle) -> [base, references]
_opened_lock = threading.Lock()


def _import(handle: bytes, device):
    """Opens another process's buffer once per allocation (a second open of
    the same allocation in one process is refused by CUDA): returns (key,
    address)."""
    key = (torch.device(device).index, handle[:64])
    offset = int.from_bytes(handle[64:72], "little")  # mr_ipc_handle_t.offset
    with _opened_lock:
        ent = _opened.get(key)
        if ent is None:
            base, _, _ = mr.mr_ipc_import(handle, device)
            ent = _opened[key] = [base, 0]
        ent[1] += 1
        return key, ent[0] + offset


def _release(key, device) -> None:
    with _opened_lock:
        ent = _opened[key]
        ent[1] -= 1
        if ent[1] == 0:
            del _opened[key]
            mr.mr_ipc_close(ent[0], device)


class PeerBuffers:
    """One [rows, d] buffer per rank, all of them addressable from this
    process: this rank's own (`local`, a tensor on its device) and every
    other rank's, mapped through CUDA IPC (handles exchanged with an
    all-gather over `group`).  `ptrs[r]` is rank r's buffer as seen here.
    Ranks on different GPUs need peer access between them (NVLink/NVSwitch);
    ranks may also share a GPU."""

    def __init__(self, rows: int, d: int, dtype, group=None, device=None):
        self.rows, self.d, self.dtype = int(rows), int(d), dtype
        self.device = torch.device(device if device is not None else torch.cuda.current_device())
        self.rank = dist.get_rank(group)
        self.ep = dist.get_world_size(group)
        self.local = torch.empty((self.rows, self.d), dtype=dtype, device=self.device)
        mine = mr.mr_ipc_export(self.local)
        handles = [None] * self.ep
        dist.all_gather_object(handles, mine, group=group)
        self._keys = []
        self.ptrs = []
        for r, h in enumerate(handles):
            if r == self.rank:
                self.ptrs.append(self.local.data_ptr())
            else:
                key, ptr = _import(h, self.device)
                self._keys.append(key)
                self.ptrs.append(ptr)

    def close(self) -> None:
        """Unmaps the other ranks' buffers (call on every rank once no kernel
        uses them any more)."""
        for key in self._keys:
            _release(key, self.device)
        self._keys = []
        self.ptrs = []


def stream_barrier(group=None) -> None:
    """Orders the ranks' GPU work: with NCCL a one-element all-reduce on the
    current stream (nothing after it on any rank's stream runs before every
    rank's work before it is done); with other backends the stream is
    synchronised and the ranks meet on the host."""
    if dist.get_backend(group) == "nccl":
        t = torch.zeros(1, dtype=torch.int32, device=torch.cuda.current_device())
        dist.all_reduce(t, group=group)
    else:
        torch.cuda.current_stream().synchronize()
        dist.barrier(group=group)


def gather_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's tokens_per_expert, rank-major [ep, N_r] on counts' device
    (all-gather; on the device with NCCL, through the host otherwise)."""
    ep = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        out = torch.empty((ep, counts.numel()), dtype=counts.dtype, device=counts.device)
        dist.all_gather_into_tensor(out, counts.contiguous(), group=group)
        return out
    host = counts.cpu()
    parts = [torch.empty_like(host) for _ in range(ep)]
    dist.all_gather(parts, host, group=group)
    return torch.stack(parts).to(counts.device)


@dataclasses.dataclass
class P2PHandle:
    """What the combine needs from one dispatch over peer memory."""
    idx: torch.Tensor
    dest: torch.Tensor
    N_r: int


def ep_dispatch_p2p(x_rows, idx, N_r, recv: PeerBuffers, group=None):
    """Dispatch of this rank's tokens straight into the owners' receive
    buffers, on the current stream.  x_rows [T,d], idx [T,k] int32.  Returns (rows, local_counts,
    local_offsets, handle): rows = this rank's receive buffer, whose first
    local_offsets[-1] rows are what it received, sorted by local expert
    (stable), local_counts [E_loc] / local_offsets [E_loc+1] on the device.
    No host synchronisation: the expert layer reads the offsets on the
    device (mr_expert_gemm_gather with perm=None)."""
    counts, offsets, _, inv = mr.mr_dispatch(idx, N_r)
    counts_all = gather_counts(counts, group)
    dest, local_counts, local_offsets = mr.mr_ep_dispatch_p2p(
        x_rows, idx, inv, offsets, counts_all, recv.rank, recv.ptrs, recv.rows)
    stream_barrier(group)  # every source's rows are in
    return recv.local, local_counts, local_offsets, P2PHandle(idx, dest, N_r)


def ep_combine_p2p(out: PeerBuffers, handle: P2PHandle, w, shared=None, group=None):
    """The weighted combine (+ shared [T,d]) of this rank's tokens, on the
    current stream, reading
    the expert outputs straight out of the owners' output buffers (row i of
    owner r's `out` buffer is the output of its receive row i).  Returns y
    [T,d].  The next ep_dispatch_p2p's count all-gather keeps the owners
    from overwriting their outputs before every rank has combined."""
    stream_barrier(group)  # every owner's outputs are complete
    return mr.mr_ep_combine_p2p(out.ptrs, w, handle.idx, handle.dest, handle.N_r, out.rows,
                                out.d, out.dtype, shared)
