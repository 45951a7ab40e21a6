"""Expert-parallel dispatch and combine on the GPU (Kimi K2 "Add shared output"
page, moe_infer, ep_size > 1).

* mr_ep_recv_order (the receive-side order, local counts and offsets) against
  the oracle, bit for bit, on many count patterns;
* ranks emulated on one GPU: each emulated rank routes, dispatches and
  gathers its own batch with libmr.so; the all-to-all is done by slicing
  and concatenating device buffers (the collective's definition, no kernel
  waits on another); the receive side sorts with mr_ep_recv_order +
  mr_gather_rows, runs a synthetic expert, scatters back, and the source
  combines -- the result must equal the single-rank path bit for bit;
* the package's ep_dispatch / ep_combine over a one-rank NCCL group equal
  the single-rank path."""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr
import workloads as wl
from parity import router_inputs, to_dev
from token_dispatch_fp32_b200 import ep

pytestmark = pytest.mark.gpu


def _counts(ep_, E_loc, seed, zeros=0.3, hot=False):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 700, size=(ep_, E_loc)).astype(np.int32)
    c[rng.random((ep_, E_loc)) < zeros] = 0
    if hot:
        c[:, :2] *= 20
    return c


CASES = [(1, 64, 0, False), (2, 128, 1, False), (4, 64, 2, True), (8, 32, 3, True),
         (8, 128, 4, False), (16, 64, 5, True), (3, 5, 6, False), (64, 16, 7, False)]


@pytest.mark.parametrize("ep_,E_loc,seed,hot", CASES,
                         ids=[f"ep{c[0]}_E{c[1]}" for c in CASES])
def test_recv_order_matches_oracle(ep_, E_loc, seed, hot):
    rc = _counts(ep_, E_loc, seed, hot=hot)
    R = int(rc.sum())
    fill = lambda n: torch.full((n,), -7, dtype=torch.int32, device="cuda")  # noqa: E731
    order, inv, lc, lo = mr.mr_ep_recv_order(to_dev(rc), R, order=fill(R), inv_order=fill(R),
                                             local_counts=fill(E_loc),
                                             local_offsets=fill(E_loc + 1))
    assert mr.mr_get_error() == mr.MR_OK
    o_order, o_local = oracle.ep_recv_order(rc)
    assert np.array_equal(order.cpu().numpy(), o_order)
    assert np.array_equal(lc.cpu().numpy(), o_local)
    assert np.array_equal(lo.cpu().numpy(), np.concatenate([[0], np.cumsum(o_local)]))
    inv_h = inv.cpu().numpy()
    assert np.array_equal(inv_h[o_order], np.arange(R))


def test_recv_order_empty_and_bad_counts():
    rc = np.zeros((4, 8), np.int32)
    order, inv, lc, lo = mr.mr_ep_recv_order(to_dev(rc), 0)
    assert mr.mr_get_error() == mr.MR_OK
    assert (lc.cpu().numpy() == 0).all() and (lo.cpu().numpy() == 0).all()
    rc[1, 3] = 5
    lc = torch.full((8,), -7, dtype=torch.int32, device="cuda")
    mr.mr_ep_recv_order(to_dev(rc), 4, local_counts=lc)  # R disagrees with the counts
    assert mr.mr_get_error() == mr.MR_ERR_DEVICE
    assert (lc.cpu().numpy() == -7).all()  # nothing written


def _expert(rows, experts, N_r):
    """Synthetic expert outputs: each row scaled by a factor of its expert,
    in fp32, rounded back to the row type."""
    scale = (1.0 + torch.arange(N_r, device=rows.device, dtype=torch.float32) / N_r)
    return (rows.float() * scale[experts.long()].unsqueeze(1)).to(rows.dtype)


def _route(w):
    d = router_inputs(w)
    xb = to_dev(d["x_bf16"], "bf16")
    ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                     device="cuda")
    idx, wt = mr.mr_router_forward_ex(xb, to_dev(d["W"]), to_dev(d["b"]), w.n_group,
                                      w.topk_group, w.k, w.route_scale, w.mask_mode,
                                      precision=mr.MR_PREC_BF16X3, workspace=ws)
    shared = torch.randn((w.T, w.d), generator=torch.Generator("cuda").manual_seed(w.seed),
                         device="cuda").to(torch.bfloat16)
    return xb, idx, wt, shared


def _single_rank(w, xb, idx, wt, shared):
    counts, offsets, perm, inv = mr.mr_dispatch(idx, w.N_r)
    xs = mr.mr_gather_rows(xb, w.k, perm=perm, inv_perm=inv)
    experts = idx.view(-1)[perm.long()]
    return mr.mr_combine(_expert(xs, experts, w.N_r), wt, inv, shared)


@pytest.mark.parametrize("ep_", [2, 4, 8])
def test_emulated_ranks_equal_single_rank_path(ep_):
    base = wl.V3_PREFILL.replace(T=1500, d=1024)
    ranks = [base.replace(T=base.T - 211 * r, seed=base.seed + 17 * r,
                          hot_experts=32 if r % 2 else 0, hot_bias=1.0) for r in range(ep_)]
    E_loc = base.N_r // ep_
    src = []
    for w in ranks:
        xb, idx, wt, shared = _route(w)
        counts, offsets, perm, inv = mr.mr_dispatch(idx, w.N_r)
        xs = mr.mr_gather_rows(xb, w.k, perm=perm, inv_perm=inv)
        src.append(dict(w=w, xb=xb, idx=idx, wt=wt, shared=shared, counts=counts, inv=inv,
                        xs=xs, send=counts.view(ep_, E_loc).sum(1).tolist()))
    # the count all-to-all and the row all-to-all, by their definition
    recv_counts = [torch.stack([s["counts"].view(ep_, E_loc)[r] for s in src]) for r in range(ep_)]
    starts = [np.concatenate([[0], np.cumsum(s["send"])]) for s in src]
    recv_rows = [torch.cat([s["xs"][starts[i][r]:starts[i][r + 1]] for i, s in enumerate(src)])
                 for r in range(ep_)]
    # receive side on every emulated rank: sort, run the experts, scatter back
    back_parts = []
    for r in range(ep_):
        R = recv_rows[r].shape[0]
        assert R == int(recv_counts[r].sum())
        order, _, lc, lo = mr.mr_ep_recv_order(recv_counts[r].contiguous(), R)
        o_order, o_local = oracle.ep_recv_order(recv_counts[r].cpu().numpy())
        assert np.array_equal(order.cpu().numpy(), o_order)
        local = mr.mr_gather_rows(recv_rows[r], 1, perm=order)
        experts = r * E_loc + torch.repeat_interleave(
            torch.arange(E_loc, device="cuda"), lc.long())
        out = _expert(local, experts, base.N_r)
        received = mr.mr_gather_rows(out, 1, inv_perm=order)
        recv_splits = recv_counts[r].sum(1).tolist()
        rs = np.concatenate([[0], np.cumsum(recv_splits)])
        back_parts.append([received[rs[i]:rs[i + 1]] for i in range(ep_)])
    assert mr.mr_get_error() == mr.MR_OK
    # the reverse all-to-all and the combine on every source
    for i, s in enumerate(src):
        back = torch.cat([back_parts[r][i] for r in range(ep_)])
        y = mr.mr_combine(back, s["wt"], s["inv"], s["shared"])
        y_ref = _single_rank(s["w"], s["xb"], s["idx"], s["wt"], s["shared"])
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), f"rank {i}"
    assert mr.mr_get_error() == mr.MR_OK


def _free_port():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def test_ep_driver_one_rank_nccl_equals_single_rank_path():
    """ep_dispatch / ep_combine through a real NCCL process group of one rank
    (the collectives are identities there) give the single-rank result."""
    import torch.distributed as dist
    w = wl.V3_PREFILL.replace(T=777, d=1024, hot_experts=32, hot_bias=1.0)
    xb, idx, wt, shared = _route(w)
    y_ref = _single_rank(w, xb, idx, wt, shared)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        local, lc, lo, h = ep.ep_dispatch(xb, idx, w.N_r)
        experts = torch.repeat_interleave(torch.arange(w.N_r, device="cuda"), lc.long())
        y = ep.ep_combine(_expert(local, experts, w.N_r), h, wt, shared)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert mr.mr_get_error() == mr.MR_OK
    assert h.send_splits == h.recv_splits == [w.T * w.k]
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
