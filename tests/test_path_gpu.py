"""The whole hot path on the GPU, chained through the C ABI exactly as the
benchmark runs it: router -> dispatch -> gather -> (synthetic experts) ->
combine, on all five workloads.  Every stage is compared with the oracle on
every token and every row:
  * the router on the raw inputs (selection exact outside near-ties, weights
    within 1e-5 relative, logits within 2e-5);
  * dispatch and gather fed the GPU's own idx, so they are bit-exact with no
    exclusions;
  * combine fed the GPU's own weights and inverse permutation, within the
    combine tolerance;
plus the identity-expert closed form (y = route_scale * x) on every token.
With MR_PARITY_OUT set, each comparison appends its figures (near-ties,
largest errors) to that file, one JSON line per workload and stage."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr
import workloads as wl
from parity import (compare_combine, compare_router, oracle_router, record, router_inputs,
                    row_inputs, to_dev, widen)

pytestmark = pytest.mark.gpu

ALL = [wl.TINY, wl.V3_PREFILL, wl.K2_PREFILL, wl.V3_DECODE, wl.V3_FULL]
CHUNK_ROWS = 1 << 14  # rows compared per host round trip (bounds host memory)


def _host_rows(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bench_router(w: wl.Workload, x32, x_rows, Wd, bd, idx, wt, logits=None):
    """The router as the benchmark launches it for this workload: bf16 rows
    above 256 tokens take the bf16x3 kernel with a workspace; decode-size and
    fp32 batches take the plain entry point on the fp32 rows (split-K for
    T <= 256, with no workspace)."""
    if w.io_dtype == wl.BF16 and w.T > 256:
        ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                         device="cuda")
        mr.mr_router_forward_ex(x_rows, Wd, bd, w.n_group, w.topk_group, w.k, w.route_scale,
                                w.mask_mode, precision=mr.MR_PREC_BF16X3, idx_out=idx,
                                w_out=wt, logits_out=logits, workspace=ws)
        return "bf16x3 fused (mr_router_forward_ex)"
    mr.mr_router_forward(x32, Wd, bd, w.n_group, w.topk_group, w.k, w.route_scale,
                         w.mask_mode, idx_out=idx, w_out=wt)
    return "plain mr_router_forward (fp32 rows)"


def run_path(w: wl.Workload, E_dev, shared_dev):
    d = router_inputs(w)
    x32 = to_dev(d["x_f32"])
    x_rows = to_dev(d["x_bf16"], "bf16") if w.io_dtype == "bf16" else x32
    # outputs start as values no kernel writes: a skipped element cannot pass
    # on the stale result of an earlier call
    fill = lambda shape, dt, v: torch.full(shape, v, dtype=dt, device="cuda")  # noqa: E731
    T, k, N, dd = w.T, w.k, w.N_r, w.d
    idx, wt = fill((T, k), torch.int32, -1), fill((T, k), torch.float32, float("nan"))
    how = bench_router(w, x32, x_rows, to_dev(d["W"]), to_dev(d["b"]), idx, wt)
    counts, offsets, perm, inv = mr.mr_dispatch(
        idx, N, counts=fill((N,), torch.int32, -7), offsets=fill((N + 1,), torch.int32, -7),
        perm=fill((T * k,), torch.int32, -7), inv_perm=fill((T * k,), torch.int32, -7))
    xs = mr.mr_gather_rows(x_rows, w.k, perm=perm, inv_perm=inv,
                           xs=fill((T * k, dd), x_rows.dtype, float("nan")))
    y = mr.mr_combine(E_dev if E_dev is not None else xs, wt, inv, shared_dev,
                      y=fill((T, dd), x_rows.dtype, float("nan")))
    assert mr.mr_get_error() == mr.MR_OK
    return dict(idx=idx, w=wt, counts=counts, offsets=offsets, perm=perm, inv=inv, xs=xs, y=y,
                x_rows=x_rows, router=how)


@pytest.mark.parametrize("w", ALL, ids=[w.name for w in ALL])
def test_full_path_every_token(w):
    rows = row_inputs(w)
    dt = "bf16" if w.io_dtype == "bf16" else None
    out = run_path(w, to_dev(rows["E"], dt), to_dev(rows["shared"], dt))
    idx = out["idx"].cpu().numpy()
    wt = out["w"].cpu().numpy()
    # router: every token
    stats = compare_router(idx, wt, oracle_router(w, np.arange(w.T), want_logits=False))
    stats["router"] = out["router"]
    record(w.name, "router", stats)
    # dispatch on the GPU's idx: bit-exact, every entry
    rc, ro, rp, ri = oracle.dispatch(idx, w.N_r)
    assert (out["counts"].cpu().numpy() == rc).all()
    assert (out["offsets"].cpu().numpy() == ro).all()
    assert (out["perm"].cpu().numpy() == rp).all()
    assert (out["inv"].cpu().numpy() == ri).all()
    record(w.name, "dispatch", {"entries": int(w.T * w.k), "mismatches": 0,
                                "hot_expert_max_count": int(rc.max())})
    # gather: bit-exact, every sorted row
    x_host = router_inputs(w)["x_bf16" if w.io_dtype == "bf16" else "x_f32"]
    nrows = w.T * w.k
    for r0 in range(0, nrows, CHUNK_ROWS):
        r1 = min(nrows, r0 + CHUNK_ROWS)
        sel = np.arange(r0, r1, dtype=np.int32)
        want = oracle.gather(x_host, w.k, rp, sel)
        assert np.array_equal(_host_rows(out["xs"][r0:r1]), want), f"gather rows {r0}..{r1}"
    record(w.name, "gather", {"rows": nrows, "mismatches": 0})
    # combine: every token, with the GPU's weights and inverse permutation
    worst = {"y_max_abs": 0.0, "y_row_rel_l2_max": 0.0, "y_max_err_over_tol": 0.0,
             "y_differ_elems": 0, "y_beyond_1e-2_rel": 0}
    tstep = max(1, CHUNK_ROWS // w.k)
    for t0 in range(0, w.T, tstep):
        t1 = min(w.T, t0 + tstep)
        tok = np.arange(t0, t1, dtype=np.int32)
        ry, rr = oracle.combine(rows["E"], wt, ri, rows["shared"], w.k, tokens=tok)
        gy = widen(_host_rows(out["y"][t0:t1]))
        c = compare_combine(gy, ry, rr, widen(rows["shared"][t0:t1]),
                            bf16=w.io_dtype == wl.BF16)
        for key in worst:
            summed = key in ("y_differ_elems", "y_beyond_1e-2_rel")
            worst[key] = worst[key] + c[key] if summed else max(worst[key], c[key])
    worst["tokens"] = w.T
    worst["elems"] = w.T * w.d
    record(w.name, "combine", worst)
    print(w.name, out["router"], stats, worst, "hot-expert counts", rc[:4])


@pytest.mark.parametrize("w", ALL, ids=[w.name for w in ALL])
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
