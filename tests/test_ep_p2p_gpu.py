"""Expert-parallel exchange over peer memory on the GPU (Kimi K2 "Add shared
output" page, moe_infer, ep_size > 1): mr_ep_dispatch_p2p writes every row
straight into its owner's receive buffer at its final local-expert-sorted
place; mr_ep_combine_p2p combines straight out of the owners' output buffers.

Ranks are emulated in one process on one GPU: one buffer per emulated rank,
the kernels of one rank after another (none waits on another), the
all-gather of the counts done by stacking them.
* the destinations, local counts and offsets against the oracle (which runs
  the page's all-to-all and stable label sort on slot labels), bit for bit;
  every received row against its token row, bit for bit; the rows past what
  an owner receives untouched;
* a whole expert layer (the grouped expert GEMM on each owner's received
  rows) combined over peer memory equals the single-rank path bit for bit;
* fp32 rows and rows without 16-byte vectors;
* the capacity limit (rows past it dropped, reported, never written) and
  inconsistent counts (nothing placed, reported);
* two processes on one GPU sharing their buffers through CUDA IPC run the
  package's ep_dispatch_p2p / ep_combine_p2p over a gloo group (host
  barriers between the steps, no kernel waits on another process)."""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr
import workloads as wl
from parity import to_dev

pytestmark = pytest.mark.gpu


def _idx(T, N_r, k, seed, hot=0):
    """k distinct expert ids per token (hot experts favoured when hot > 0)."""
    g = torch.Generator("cuda").manual_seed(seed)
    s = torch.rand((T, N_r), generator=g, device="cuda")
    if hot:
        s[:, :hot] += 0.5
    return s.topk(k, dim=1).indices.to(torch.int32).contiguous()


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def _ranks(ep_, T0, d, N_r, k, dtype, seed):
    """Per emulated rank: rows, ids and the rank's own dispatch (ragged batch
    sizes, the last rank with no tokens)."""
    out = []
    for r in range(ep_):
        T = 0 if r == ep_ - 1 and ep_ > 1 else T0 - 37 * r
        g = torch.Generator("cuda").manual_seed(seed + r)
        x = torch.randn((T, d), generator=g, device="cuda").to(dtype)
        idx = _idx(T, N_r, k, seed + 100 + r, hot=8 if r % 2 else 0) if T else \
            torch.zeros((0, k), dtype=torch.int32, device="cuda")
        counts, offsets, perm, inv = mr.mr_dispatch(idx, N_r)
        out.append(dict(T=T, x=x, idx=idx, counts=counts, offsets=offsets, perm=perm, inv=inv))
    return out


def _dispatch_all(src, N_r, cap, d, dtype, guard=3, sentinel=-3):
    """Runs every emulated rank's mr_ep_dispatch_p2p into one buffer per rank
    ([cap + guard, d], filled with a sentinel bit pattern)."""
    ep_ = len(src)
    counts_all = torch.stack([s["counts"] for s in src]).contiguous()
    itype = torch.int16 if dtype == torch.bfloat16 else torch.int32
    bufs = [torch.full((cap + guard, d), sentinel, dtype=itype, device="cuda").view(dtype)
            for _ in range(ep_)]
    for r, s in enumerate(src):
        s["dest"], s["lc"], s["lo"] = mr.mr_ep_dispatch_p2p(
            s["x"], s["idx"], s["inv"], s["offsets"], counts_all, r, bufs, cap)
    return bufs, counts_all


CASES = [(2, 256, 8, 1024, torch.bfloat16), (4, 256, 8, 7168, torch.bfloat16),
         (8, 256, 8, 1024, torch.bfloat16), (8, 384, 8, 512, torch.bfloat16),
         (3, 48, 6, 1000, torch.float32), (4, 64, 4, 7, torch.bfloat16),
         (2, 16, 3, 5, torch.float32), (1, 64, 8, 256, torch.bfloat16)]


@pytest.mark.parametrize("ep_,N_r,k,d,dtype", CASES,
                         ids=[f"ep{c[0]}_N{c[1]}_k{c[2]}_d{c[3]}_{str(c[4])[6:]}" for c in CASES])
def test_dispatch_p2p_matches_oracle(ep_, N_r, k, d, dtype):
    src = _ranks(ep_, 700, d, N_r, k, dtype, seed=ep_ * 1000 + N_r + d)
    E_loc = N_r // ep_
    o_dest, o_local = oracle.ep_dest([s["idx"].cpu().numpy() for s in src], N_r)
    R = [int(l.sum()) for l in o_local]
    cap = max(R) + 5
    bufs, _ = _dispatch_all(src, N_r, cap, d, dtype)
    assert mr.mr_get_error() == mr.MR_OK
    for r, s in enumerate(src):
        assert np.array_equal(s["dest"].cpu().numpy(), o_dest[r]), f"rank {r} dest"
        assert np.array_equal(s["lc"].cpu().numpy(), o_local[r])
        assert np.array_equal(s["lo"].cpu().numpy(), np.concatenate([[0], np.cumsum(o_local[r])]))
    for s in src:  # every slot's row holds its token row, in its owner's buffer
        if s["T"] == 0:
            continue
        owner = (s["idx"].view(-1) // E_loc).long()
        tok = torch.arange(s["T"] * k, device="cuda") // k
        for r in range(ep_):
            m = owner == r
            got = bufs[r][s["dest"][m].long()]
            assert torch.equal(_bits(got), _bits(s["x"][tok[m]]))
    for r in range(ep_):  # nothing past what the owner receives
        assert (_bits(bufs[r][R[r]:]) == -3).all()


def _single_rank_layer(s, W, N_r, k):
    counts, offsets, perm, inv = mr.mr_dispatch(s["idx"], N_r)
    out = mr.mr_expert_gemm_gather(s["x"], k, perm, offsets, W)
    return mr.mr_combine(out, s["w"], inv, s["shared"])


@pytest.mark.parametrize("ep_", [2, 4, 8])
def test_expert_layer_over_peer_memory_equals_single_rank(ep_):
    """Router weights from the fused router, one linear expert per expert
    (bf16 weights), the shared add: every source's y equals the single-rank
    path (dispatch + gather-fused expert GEMM + combine) bit for bit."""
    base = wl.V3_PREFILL.replace(T=900, d=1024)
    N_r, k, n_out = base.N_r, base.k, 256
    E_loc = N_r // ep_
    W = to_dev(wl.gen_expert_W(base, n_out), "bf16")
    src = []
    for r in range(ep_):
        w = base.replace(T=base.T - 113 * r, seed=base.seed + 17 * r,
                         hot_experts=32 if r % 2 else 0, hot_bias=1.0)
        d_in = wl.gen_router_inputs(w)
        x = to_dev(d_in["x_bf16"], "bf16")
        ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                         device="cuda")
        idx, wt = mr.mr_router_forward_ex(x, to_dev(d_in["W"]), to_dev(d_in["b"]), w.n_group,
                                          w.topk_group, w.k, w.route_scale, w.mask_mode,
                                          precision=mr.MR_PREC_BF16X3, workspace=ws)
        shared = torch.randn((w.T, n_out), generator=torch.Generator("cuda").manual_seed(w.seed),
                             device="cuda").to(torch.bfloat16)
        counts, offsets, perm, inv = mr.mr_dispatch(idx, N_r)
        src.append(dict(T=w.T, x=x, idx=idx, w=wt, shared=shared, counts=counts,
                        offsets=offsets, inv=inv))
    cap = sum(s["T"] for s in src) * k  # never overflows
    recv, _ = _dispatch_all(src, N_r, cap, base.d, torch.bfloat16)
    outs = [torch.zeros((cap, n_out), dtype=torch.bfloat16, device="cuda") for _ in range(ep_)]
    for r in range(ep_):  # each owner's experts on its received rows
        mr.mr_expert_gemm_gather(recv[r][:cap], 1, None, src[r]["lo"],
                                 W[r * E_loc:(r + 1) * E_loc].contiguous(), out=outs[r])
    for r, s in enumerate(src):
        y = mr.mr_ep_combine_p2p(outs, s["w"], s["idx"], s["dest"], N_r, cap, n_out,
                                 torch.bfloat16, s["shared"])
        y_ref = _single_rank_layer(s, W, N_r, k)
        assert torch.equal(_bits(y), _bits(y_ref)), f"rank {r}"
    assert mr.mr_get_error() == mr.MR_OK


@pytest.mark.parametrize("d,dtype,shared", [(1000, torch.float32, True),
                                            (7, torch.bfloat16, True),
                                            (5, torch.float32, False),
                                            (1024, torch.bfloat16, False)])
def test_combine_p2p_equals_combine(d, dtype, shared):
    """Identity experts (each owner's output buffer is its receive buffer):
    the combine over peer memory equals mr_combine of the rank's own gathered
    rows, bit for bit, on the vector and the element paths."""
    ep_, N_r, k = 4, 64, 6
    src = _ranks(ep_, 500, d, N_r, k, dtype, seed=d * 7)
    cap = sum(s["T"] for s in src) * k
    bufs, _ = _dispatch_all(src, N_r, cap, d, dtype)
    for r, s in enumerate(src):
        g = torch.Generator("cuda").manual_seed(r)
        w = torch.rand((s["T"], k), generator=g, device="cuda")
        sh = torch.randn((s["T"], d), generator=g, device="cuda").to(dtype) if shared else None
        y = mr.mr_ep_combine_p2p(bufs, w, s["idx"], s["dest"], N_r, cap, d, dtype, sh)
        xs = mr.mr_gather_rows(s["x"], k, perm=s["perm"], inv_perm=s["inv"]) if s["T"] else \
            s["x"].new_empty((0, d))
        y_ref = mr.mr_combine(xs, w, s["inv"], sh) if s["T"] else y
        assert torch.equal(_bits(y), _bits(y_ref)), f"rank {r}"
    assert mr.mr_get_error() == mr.MR_OK


def test_capacity_overflow_drops_rows_and_reports():
    ep_, N_r, k, d = 4, 64, 8, 256
    src = _ranks(ep_, 600, d, N_r, k, torch.bfloat16, seed=5)
    o_dest, o_local = oracle.ep_dest([s["idx"].cpu().numpy() for s in src], N_r)
    R = [int(l.sum()) for l in o_local]
    cap = min(R) - 50  # every owner loses rows
    assert cap > 0
    bufs, _ = _dispatch_all(src, N_r, cap, d, torch.bfloat16, guard=64)
    assert mr.mr_get_error() == mr.MR_ERR_OVERFLOW
    E_loc = N_r // ep_
    for r, s in enumerate(src):
        want = np.where(o_dest[r] < cap, o_dest[r], -1)
        assert np.array_equal(s["dest"].cpu().numpy(), want)
        lo = np.minimum(np.concatenate([[0], np.cumsum(o_local[r])]), cap)
        assert np.array_equal(s["lo"].cpu().numpy(), lo)
        assert np.array_equal(s["lc"].cpu().numpy(), np.diff(lo))
    for r in range(ep_):  # the guard rows past the capacity were never written
        assert (bufs[r][cap:].view(torch.int16) == -3).all()
    for s in src:  # the rows that fit are in place
        if s["T"] == 0:
            continue
        ok = s["dest"] >= 0
        owner = (s["idx"].view(-1) // E_loc).long()
        tok = torch.arange(s["T"] * k, device="cuda") // k
        for r in range(ep_):
            m = ok & (owner == r)
            assert torch.equal(_bits(bufs[r][s["dest"][m].long()]), _bits(s["x"][tok[m]]))


def test_inconsistent_counts_place_nothing():
    ep_, N_r, k, d = 2, 32, 4, 64
    src = _ranks(ep_, 300, d, N_r, k, torch.bfloat16, seed=9)
    counts_all = torch.stack([s["counts"] for s in src]).contiguous()
    counts_all[0, 3] += 1  # rank 0's row disagrees with its own offsets
    buf = [torch.full((5000, d), -3, dtype=torch.int16, device="cuda").view(torch.bfloat16)
           for _ in range(ep_)]
    s = src[0]
    dest, lc, lo = mr.mr_ep_dispatch_p2p(s["x"], s["idx"], s["inv"], s["offsets"], counts_all, 0,
                                         buf, 5000)
    assert mr.mr_get_error() == mr.MR_ERR_DEVICE
    assert (dest == -1).all() and (lc == 0).all() and (lo == 0).all()
    assert all((b.view(torch.int16) == -3).all() for b in buf)


def test_argument_checks():
    x = torch.zeros((4, 8), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    counts, offsets, perm, inv = mr.mr_dispatch(idx, 6)
    ca = torch.stack([counts, counts, counts])
    with pytest.raises(ValueError):  # 3 receive buffers for 3 ranks, 6 experts: fine; 2: not
        mr.mr_ep_dispatch_p2p(x, idx, inv, offsets, ca, 0, [x, x], 4)
    with pytest.raises(mr.MRError):  # rank out of range
        mr.mr_ep_dispatch_p2p(x, idx, inv, offsets, ca, 3, [x, x, x], 4)
    with pytest.raises(mr.MRError):  # a null buffer
        mr.mr_ep_dispatch_p2p(x, idx, inv, offsets, ca, 0, [x, 0, x], 4)


# ---- two processes, one GPU, buffers shared through CUDA IPC -----------------

def _free_port():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _ipc_rank(rank, world, port):
    import torch.distributed as dist

    from token_dispatch_fp32_b200 import ep
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=120))
    N_r, k, d, n_out = 64, 6, 512, 128
    E_loc = N_r // world
    T = 300 + 77 * rank
    g = torch.Generator("cuda").manual_seed(40 + rank)
    x = torch.randn((T, d), generator=g, device="cuda").to(torch.bfloat16)
    idx = _idx(T, N_r, k, 50 + rank, hot=4 * rank)
    w = torch.rand((T, k), generator=g, device="cuda")
    shared = torch.randn((T, n_out), generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn((N_r, n_out, d), generator=torch.Generator("cuda").manual_seed(7),
                     device="cuda") / 16).to(torch.bfloat16)
    cap = 2 * 400 * k
    recv = ep.PeerBuffers(cap, d, torch.bfloat16)
    out = ep.PeerBuffers(cap, n_out, torch.bfloat16)
    rows, lc, lo, h = ep.ep_dispatch_p2p(x, idx, N_r, recv)
    mr.mr_expert_gemm_gather(rows, 1, None, lo, W[rank * E_loc:(rank + 1) * E_loc].contiguous(),
                             out=out.local)
    y = ep.ep_combine_p2p(out, h, w, shared)
    torch.cuda.synchronize()
    dist.barrier()  # every rank finished reading the others' buffers
    status = mr.mr_get_error()
    recv.close()
    out.close()
    counts, offsets, perm, inv = mr.mr_dispatch(idx, N_r)
    y_ref = mr.mr_combine(mr.mr_expert_gemm_gather(x, k, perm, offsets, W), w, inv, shared)
    dist.destroy_process_group()
    assert status == mr.MR_OK, f"rank {rank}: status {status}"
    assert int(lo[-1].item()) > 0
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), \
        f"rank {rank}: y differs from the single-rank path"


def test_two_processes_share_buffers_through_ipc():
    import torch.multiprocessing as tmp
    tmp.spawn(_ipc_rank, args=(2, _free_port()), nprocs=2, join=True)


def test_package_p2p_over_one_rank_nccl_equals_single_rank():
    """ep.ep_dispatch_p2p / ep.ep_combine_p2p through a real NCCL process
    group of one rank: the count all-gather on the device, the stream-ordered
    barriers (one-element all-reduces) and PeerBuffers with this rank's own
    buffer only; a whole expert layer equals the single-rank path."""
    import torch.distributed as dist

    from token_dispatch_fp32_b200 import ep
    N_r, k, d, n_out, T = 64, 6, 512, 128, 700
    g = torch.Generator("cuda").manual_seed(11)
    x = torch.randn((T, d), generator=g, device="cuda").to(torch.bfloat16)
    idx = _idx(T, N_r, k, 12, hot=4)
    w = torch.rand((T, k), generator=g, device="cuda")
    shared = torch.randn((T, n_out), generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn((N_r, n_out, d), generator=g, device="cuda") / 16).to(torch.bfloat16)
    counts, offsets, perm, inv = mr.mr_dispatch(idx, N_r)
    y_ref = mr.mr_combine(mr.mr_expert_gemm_gather(x, k, perm, offsets, W), w, inv, shared)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        recv = ep.PeerBuffers(T * k, d, torch.bfloat16)
        out = ep.PeerBuffers(T * k, n_out, torch.bfloat16)
        assert recv.ptrs == [recv.local.data_ptr()]
        rows, lc, lo, h = ep.ep_dispatch_p2p(x, idx, N_r, recv)
        mr.mr_expert_gemm_gather(rows, 1, None, lo, W, out=out.local)
        y = ep.ep_combine_p2p(out, h, w, shared)
        torch.cuda.synchronize()
        recv.close()
        out.close()
    finally:
        dist.destroy_process_group()
    assert mr.mr_get_error() == mr.MR_OK
    assert int(lo[-1].item()) == T * k
    assert torch.equal(lc, counts)
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
