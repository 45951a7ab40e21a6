"""The whole hot path on the GPU, chained through the C ABI exactly as the
benchmark runs it: router -> dispatch -> gather -> (synthetic experts) ->
combine.  Each stage is checked against the oracle fed with the GPU's own
upstream outputs (so dispatch/gather are bit-exact with no exclusions), the
router against the oracle on the raw inputs, and the identity-expert closed
form (y = route_scale * x) on every token."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr
import workloads as wl
from parity import (compare_combine, compare_router, oracle_router, router_inputs, row_inputs,
                    sample_tokens, to_dev, widen)

pytestmark = pytest.mark.gpu


def _host_rows(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def run_path(w: wl.Workload, E_dev, shared_dev):
    d = router_inputs(w)
    x32 = to_dev(d["x_f32"])
    x_rows = to_dev(d["x_bf16"], "bf16") if w.io_dtype == "bf16" else x32
    # outputs start as values no kernel writes: a skipped element cannot pass
    # on the stale result of an earlier call
    fill = lambda shape, dt, v: torch.full(shape, v, dtype=dt, device="cuda")  # noqa: E731
    T, k, N, dd = w.T, w.k, w.N_r, w.d
    idx, wt = mr.mr_router_forward(x32, to_dev(d["W"]), to_dev(d["b"]), w.n_group,
                                   w.topk_group, w.k, w.route_scale, w.mask_mode,
                                   idx_out=fill((T, k), torch.int32, -1),
                                   w_out=fill((T, k), torch.float32, float("nan")))
    counts, offsets, perm, inv = mr.mr_dispatch(
        idx, N, counts=fill((N,), torch.int32, -7), offsets=fill((N + 1,), torch.int32, -7),
        perm=fill((T * k,), torch.int32, -7), inv_perm=fill((T * k,), torch.int32, -7))
    xs = mr.mr_gather_rows(x_rows, w.k, perm=perm, inv_perm=inv,
                           xs=fill((T * k, dd), x_rows.dtype, float("nan")))
    y = mr.mr_combine(E_dev if E_dev is not None else xs, wt, inv, shared_dev,
                      y=fill((T, dd), x_rows.dtype, float("nan")))
    assert mr.mr_get_error() == mr.MR_OK
    return dict(idx=idx, w=wt, counts=counts, offsets=offsets, perm=perm, inv=inv, xs=xs, y=y,
                x_rows=x_rows)


@pytest.mark.parametrize("w", [wl.TINY, wl.V3_FULL], ids=["tiny", "v3_full"])
def test_full_path(w):
    rows = row_inputs(w)
    dt = "bf16" if w.io_dtype == "bf16" else None
    out = run_path(w, to_dev(rows["E"], dt), to_dev(rows["shared"], dt))
    idx = out["idx"].cpu().numpy()
    wt = out["w"].cpu().numpy()
    # router on sampled tokens
    tok = sample_tokens(w.T, 256, seed=w.seed)
    stats = compare_router(idx[tok], wt[tok], oracle_router(w, tok, want_logits=False))
    # dispatch on the GPU's idx: bit-exact, every entry
    rc, ro, rp, ri = oracle.dispatch(idx, w.N_r)
    assert (out["counts"].cpu().numpy() == rc).all()
    assert (out["offsets"].cpu().numpy() == ro).all()
    assert (out["perm"].cpu().numpy() == rp).all()
    assert (out["inv"].cpu().numpy() == ri).all()
    # gather: bit-exact on sampled sorted rows (all rows for small T)
    x_host = rows_x = router_inputs(w)["x_bf16" if w.io_dtype == "bf16" else "x_f32"]
    nrows = w.T * w.k
    srows = sample_tokens(nrows, 4096, seed=1).astype(np.int32)
    xs = out["xs"][torch.from_numpy(srows).long().cuda()]
    assert np.array_equal(_host_rows(xs), oracle.gather(x_host, w.k, rp, srows))
    # combine on sampled tokens with the GPU's weights and inverse permutation
    ry, rr = oracle.combine(rows["E"], wt, ri, rows["shared"], w.k,
                            tokens=tok.astype(np.int32))
    gy = widen(_host_rows(out["y"][torch.from_numpy(tok).cuda()]))
    cstats = compare_combine(gy, ry, rr, widen(rows["shared"][tok]))
    print(w.name, stats, cstats, "hot-expert counts", rc[:4])
    del rows_x


@pytest.mark.parametrize("w", [wl.TINY, wl.V3_FULL], ids=["tiny", "v3_full"])
def test_identity_experts_closed_form_every_token(w):
    """Experts = identity and no shared expert: y_t = sum_j w_tj x_t =
    route_scale * x_t (weights sum to the route scale), on every token."""
    out = run_path(w, None, None)
    x = out["x_rows"].float()
    y = out["y"].float()
    wsum = out["w"].sum(1, keepdim=True)
    exact = x.double() * wsum.double()
    err = (y.double() - exact).abs()
    if w.io_dtype == "bf16":  # one rounding to bf16 (half an ulp) plus fp32 sums
        ulp = torch.exp2(torch.floor(torch.log2(exact.abs().clamp_min(1e-30))) - 7)
        assert (err <= 0.5 * ulp + 1e-5 * exact.abs() + 1e-30).all()
    else:
        assert (err <= 1e-6 * exact.abs() + 1e-7).all()
    assert torch.allclose(wsum, torch.full_like(wsum, w.route_scale), rtol=2e-6)
