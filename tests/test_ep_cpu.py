"""Expert-parallel dispatch and combine (Kimi K2 "Add shared output" page,
moe_infer, ep_size > 1) on CPU ranks over gloo: the package's exchange steps
(count all-to-all, host split sizes, variable-split row all-to-all there and
back) composed with the oracle's local steps (router, dispatch, gather,
receive-side order, combine) must give, on every rank, exactly the result
of the single-rank path with the same expert function.  The split sizes are
also checked against the oracle's restatement of the page's bookkeeping, and
the received rows against an all-to-all emulated from every rank's rows."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads as wl  # noqa: E402
from token_dispatch_fp32_b200 import ep  # noqa: E402

BASE = wl.Workload("ep_cpu_N64", T=50, d=40, N_r=64, n_group=4, topk_group=2, k=4,
                   route_scale=2.5, mask_mode=0, seed=70, io_dtype="f32")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def expert_fn(e_global, rows):
    """Synthetic expert: the row scaled by a factor of its expert (fp32),
    so a row sent to the wrong expert changes the result."""
    return (rows * np.float32(1.0 + e_global / 64.0)).astype(np.float32)


def rank_inputs(r, skew):
    w = BASE.replace(T=BASE.T - 13 * r, seed=BASE.seed + r)  # ragged per rank
    if skew:
        w = w.replace(hot_experts=8, hot_bias=1.0)
    d = wl.gen_router_inputs(w)
    return w, d


def _rank_main(rank, world, port, out_dir, skew):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, d = rank_inputs(rank, skew)
        r = oracle.router(d["x_f32"], d["W"], d["b"], w.n_group, w.topk_group, w.k,
                          w.route_scale, w.mask_mode)
        idx, wt = r["idx"], r["w"].astype(np.float32)
        counts, offsets, perm, inv = oracle.dispatch(idx, w.N_r)
        xs = oracle.gather(d["x_f32"], w.k, perm)
        shared = wl.gen_shared(w)
        # the package's exchange steps
        recv_counts, send_splits, recv_splits = ep.exchange_counts(torch.from_numpy(counts))
        recv_rows = ep.exchange_rows(torch.from_numpy(xs), send_splits, recv_splits).numpy()
        # the oracle's restatement of the bookkeeping, from every rank's counts
        all_counts = [torch.zeros(w.N_r, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(all_counts, torch.from_numpy(counts))
        o_send, o_recv_counts, o_recv = oracle.ep_splits(np.stack([c.numpy() for c in all_counts]),
                                                         rank)
        assert list(o_send) == send_splits and list(o_recv) == recv_splits
        assert np.array_equal(recv_counts.numpy(), o_recv_counts)
        # the received rows against an all-to-all emulated from every rank's rows
        blocks = [None] * world
        dist.all_gather_object(blocks, (xs, send_splits))
        send_blocks = [np.split(b, np.cumsum(sp)[:-1]) for b, sp in blocks]
        assert np.array_equal(recv_rows, oracle.all_to_all(send_blocks)[rank])
        # receive side: sort by local expert, run the experts, scatter back
        order, local_counts = oracle.ep_recv_order(recv_counts.numpy())
        local_rows = oracle.gather(recv_rows, 1, order)
        E_loc = w.N_r // world
        labels = np.repeat(np.arange(E_loc), local_counts) + rank * E_loc
        local_out = np.concatenate([expert_fn(e, local_rows[i:i + 1])
                                    for i, e in enumerate(labels)]) if len(labels) else \
            np.zeros((0, w.d), np.float32)
        new_x = np.empty_like(local_out)
        new_x[order] = local_out                      # new_x[gatherd_idxs] = outs
        back = ep.exchange_rows(torch.from_numpy(new_x), recv_splits, send_splits).numpy()
        y, _ = oracle.combine(back, wt, inv, shared, w.k)
        # the single-rank path with the same experts
        experts = idx.reshape(-1)[perm]
        E_ref = np.concatenate([expert_fn(e, xs[i:i + 1]) for i, e in enumerate(experts)])
        assert np.array_equal(back, E_ref)
        y_ref, _ = oracle.combine(E_ref, wt, inv, shared, w.k)
        assert np.array_equal(y, y_ref)
        with open(os.path.join(out_dir, f"ok{rank}"), "w") as f:
            f.write(f"{sum(send_splits)} {sum(recv_splits)}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,skew", [(2, False), (2, True), (4, True)])
def test_ep_exchange_matches_single_rank_path(tmp_path, world, skew):
    tmp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), skew), nprocs=world,
              join=True)
    sent = recv = 0
    for r in range(world):
        a, b = open(tmp_path / f"ok{r}").read().split()
        sent, recv = sent + int(a), recv + int(b)
    assert sent == recv  # every row sent was received once


def test_split_sizes_host_bookkeeping():
    counts = [3, 0, 2, 1, 5, 0]
    recv = [1, 1, 0, 4, 2, 2]  # [ep=3][E_loc=2], source-major
    assert ep.split_sizes(counts, recv, 3) == ([3, 3, 5], [2, 4, 4])
    with pytest.raises(ValueError):
        ep.split_sizes(counts[:5], recv[:5], 3)
