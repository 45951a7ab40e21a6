"""One expert layer over the expert-sorted rows with the row gather fused into
the GEMM (mr_expert_gemm_gather; Kimi K2 "Add shared output" page, moe_infer:
sorted_tokens = x[idxs // k], expert(sorted_tokens[start_idx:end_idx])),
against the oracle's binary64 restatement.

Tolerance: each bf16 x bf16 product is exact in fp32; the tensor core adds
them into an fp32 accumulator rounding toward zero, one rounding per
16-deep MMA step, so the accumulated value is within (d/16 + 2) * 2^-23 *
sum_c |x_c W_c| of the exact dot product; the result is then rounded to bf16,
which can land one bf16 ulp away where the exact value sits on a rounding
boundary.  Hence |out - exact| <= ulp_bf16(exact) + (d/16 + 2) 2^-23 sum|xW|.
Rows past the expert segments (dropped ids) must stay untouched."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr
import workloads as wl
from parity import bf16_ulp, record

pytestmark = pytest.mark.gpu


def _ids(T, k, N_r, seed, skew):
    rng = np.random.default_rng(seed)
    if skew:
        return np.where(rng.random((T, k)) < 0.7, rng.integers(0, 8, (T, k)),
                        rng.integers(0, N_r, (T, k))).astype(np.int32)
    return np.stack([rng.permutation(N_r)[:k] for _ in range(T)]).astype(np.int32)


def _dev_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()


CASES = [
    # T, d, N_r, k, n_out, skew, n_check (None: every row)
    (100, 256, 16, 4, 256, False, None),
    (257, 200, 32, 3, 144, True, None),      # K tail (200 % 32), partial N tile
    (64, 7168, 256, 8, 512, False, None),    # decode-size batch, most experts one block
    (1000, 512, 64, 8, 256, True, None),     # skewed: experts with many blocks
    (4096, 7168, 256, 8, 2048, False, 768),  # DeepSeek-V3 prefill batch, sampled rows
]


@pytest.mark.parametrize("bk", ["64", "64tma", "32"])
@pytest.mark.parametrize("T,d,N_r,k,n_out,skew,n_check", CASES,
                         ids=[f"T{c[0]}_d{c[1]}_E{c[2]}_n{c[4]}" for c in CASES])
def test_expert_gemm_gather_matches_oracle(T, d, N_r, k, n_out, skew, n_check, bk,
                                           monkeypatch):
    """Both K-chunk widths: 64 bf16 (128-byte rows, the default; rows copied
    by the epilogue warps, or by TMA gathers when pinned) and 32 (TMA
    gathers)."""
    monkeypatch.setenv("MR_EG_BK", bk[:2])
    if bk == "64tma":
        monkeypatch.setenv("MR_EG_GATHER", "tma")
    if bk != "64" and n_check is not None:
        pytest.skip("the full-size case runs with the default width")
    w = wl.Workload(f"expert_T{T}_d{d}", T=T, d=d, N_r=N_r, n_group=1, topk_group=1, k=k,
                    route_scale=1.0, mask_mode=0, seed=T + d + N_r)
    rng = np.random.default_rng(w.seed)
    x = wl.to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    W = wl.gen_expert_W(w, n_out)
    idx = _ids(T, k, N_r, w.seed, skew)
    counts, offsets, perm, inv = oracle.dispatch(idx, N_r)
    out = torch.full((T * k, n_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    mr.mr_expert_gemm_gather(_dev_bits(x), k, torch.from_numpy(perm).cuda(),
                             torch.from_numpy(offsets).cuda(), _dev_bits(W), out=out)
    assert mr.mr_get_error() == mr.MR_OK
    if n_check is None:
        rows = np.arange(T * k, dtype=np.int32)
    else:  # spread over the experts, with every segment's first and last row
        ends = np.concatenate([offsets[:-1], offsets[1:] - 1])
        ends = ends[(ends >= 0) & (ends < T * k)]
        rows = np.unique(np.concatenate([ends, rng.choice(T * k, n_check, replace=False)]))
        rows = rows.astype(np.int32)
    ref = oracle.expert_gemm(x, k, perm, offsets, W, rows=rows)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)[rows]
    got = wl.bf16_bits_to_f32(got).astype(np.float64)
    xf = np.abs(wl.bf16_bits_to_f32(x).astype(np.float64))
    Wf = np.abs(wl.bf16_bits_to_f32(W).astype(np.float64))
    e_of = np.searchsorted(offsets, rows, side="right") - 1
    absdot = np.stack([xf[perm[j] // k] @ Wf[e].T for j, e in zip(rows, e_of)])
    tol = bf16_ulp(ref) + (d / 16 + 2) * 2.0 ** -23 * absdot
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert (err <= tol).all(), f"row {rows[worst[0]]} col {worst[1]}: {got[worst]} vs {ref[worst]}"
    stats = {"rows_checked": int(len(rows)), "rows": int(T * k), "max_abs_err": float(err.max()),
             "max_err_over_tol": float((err / tol).max()),
             "differ_from_rounded_exact": int((got != oracle.round_bf16(ref)).sum())}
    record(w.name, f"expert_gemm_gather_bk{bk}", stats)
    print(w.name, stats)


def test_expert_gemm_gather_leaves_dropped_rows_alone():
    """Ids outside [0, N_r) are dropped by the dispatch; the rows past
    offsets[N_r] keep whatever the output held."""
    T, d, N_r, k, n_out = 50, 64, 8, 2, 32
    rng = np.random.default_rng(5)
    idx = _ids(T, k, N_r, 5, False)
    idx[3, 1] = N_r + 2
    idx_d = torch.from_numpy(idx).cuda()
    counts, offsets, perm, inv = mr.mr_dispatch(idx_d, N_r)
    assert mr.mr_get_error() == mr.MR_ERR_DEVICE
    x = wl.to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    W = wl.to_bf16_bits(rng.standard_normal((N_r, n_out, d)).astype(np.float32) * 0.1)
    out = torch.full((T * k, n_out), 7.0, dtype=torch.bfloat16, device="cuda")
    mr.mr_expert_gemm_gather(_dev_bits(x), k, perm, offsets, _dev_bits(W), out=out)
    assert mr.mr_get_error() == mr.MR_OK
    n_valid = int(offsets[-1])
    assert n_valid == T * k - 1
    assert (out[n_valid:].float() == 7.0).all()
    ref = oracle.expert_gemm(x, k, perm.cpu().numpy(), offsets.cpu().numpy(), W)
    got = out[:n_valid].float().cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= bf16_ulp(ref) + 1e-3).all()


@pytest.mark.parametrize("T,d,N_r,k,n_out", [(257, 200, 32, 3, 144), (300, 7168, 64, 8, 512),
                                             (100, 520, 16, 4, 256)])
def test_expert_gemm_packed_weights_bit_identical(T, d, N_r, k, n_out):
    """The packed weight layout changes only where the weights are read:
    the results equal the plain layout's bit for bit (K tails and partial
    output tiles included)."""
    w = wl.Workload(f"expert_packed_T{T}", T=T, d=d, N_r=N_r, n_group=1, topk_group=1, k=k,
                    route_scale=1.0, mask_mode=0, seed=3 * T + d)
    rng = np.random.default_rng(w.seed)
    x = _dev_bits(wl.to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32)))
    W = _dev_bits(wl.gen_expert_W(w, n_out))
    counts, offsets, perm, inv = mr.mr_dispatch(torch.from_numpy(_ids(T, k, N_r, w.seed, True))
                                                .cuda(), N_r)
    plain = mr.mr_expert_gemm_gather(x, k, perm, offsets, W)
    Wp = mr.mr_expert_pack_weights(W)
    packed = mr.mr_expert_gemm_gather_packed(x, k, perm, offsets, Wp, N_r, n_out)
    assert mr.mr_get_error() == mr.MR_OK
    assert torch.equal(plain.view(torch.int16), packed.view(torch.int16))


def test_expert_gemm_on_sorted_rows_equals_fused_gather():
    """Without perm the GEMM reads already-sorted rows (e.g. from
    mr_gather_rows) with tiled copies: the same rows, the same arithmetic,
    so the same bits as the fused gather."""
    T, d, N_r, k, n_out = 300, 7168, 64, 8, 256
    w = wl.Workload("expert_sorted_T300", T=T, d=d, N_r=N_r, n_group=1, topk_group=1, k=k,
                    route_scale=1.0, mask_mode=0, seed=77)
    rng = np.random.default_rng(w.seed)
    x = _dev_bits(wl.to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32)))
    W = _dev_bits(wl.gen_expert_W(w, n_out))
    counts, offsets, perm, inv = mr.mr_dispatch(torch.from_numpy(_ids(T, k, N_r, 7, True))
                                                .cuda(), N_r)
    fused = mr.mr_expert_gemm_gather(x, k, perm, offsets, W)
    xs = mr.mr_gather_rows(x, k, perm=perm, inv_perm=inv)
    plain = mr.mr_expert_gemm_gather(xs, k, None, offsets, W)
    packed = mr.mr_expert_gemm_gather_packed(xs, k, None, offsets,
                                             mr.mr_expert_pack_weights(W), N_r, n_out)
    assert mr.mr_get_error() == mr.MR_OK
    assert torch.equal(fused.view(torch.int16), plain.view(torch.int16))
    assert torch.equal(fused.view(torch.int16), packed.view(torch.int16))


# ---- the combine fused into the expert layer's epilogue ---------------------

def _combine_case(T, d, N_r, k, n_out, seed, skew, integer, with_shared, drop=0.0):
    """Inputs of one fused-combine case (bf16 bits, fp32 weights) and the
    dispatch of its ids (oracle); `drop` > 0 puts that fraction of the slots
    (and every slot of token 0) out of range, which dispatch drops."""
    rng = np.random.default_rng(seed)
    if integer:
        # small integers: every product and every d-term sum is exact in fp32,
        # so the tensor core's expert outputs are the rounded exact values
        x = wl.to_bf16_bits(rng.integers(-2, 3, (T, d)).astype(np.float32))
        W = wl.to_bf16_bits(rng.integers(-2, 3, (N_r, n_out, d)).astype(np.float32))
    else:
        x = wl.to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
        W = wl.gen_expert_W(wl.Workload(f"ecomb{seed}", T=T, d=d, N_r=N_r, n_group=1,
                                        topk_group=1, k=k, route_scale=1.0, mask_mode=0,
                                        seed=seed), n_out)
    idx = _ids(T, k, N_r, seed, skew)
    if drop > 0:
        idx = np.where(rng.random((T, k)) < drop, N_r + 1, idx).astype(np.int32)
        idx[0, :] = N_r + 3
    w = rng.uniform(0.05, 1.0, (T, k)).astype(np.float32)
    sh = (wl.to_bf16_bits(rng.standard_normal((T, n_out)).astype(np.float32))
          if with_shared else None)
    return x, W, idx, w, sh


def _combine_reference(x, W, idx, w, sh, k, N_r, integer):
    """The oracle's y and routed sums for the fused layer, and a per-element
    bound on |y_gpu - y|: the expert outputs (tensor core, fp32 accumulation,
    bf16 rounding) are within 2 ulp_bf16 + (d/16 + 2) 2^-23 sum|x W| of the
    oracle's rounded exact ones (0 for integer inputs: exact accumulation);
    the weighted sum adds fp32 products in some order ((k + 1) 2^-23 of
    sum|w E|); the two bf16 roundings can each land one ulp away."""
    T, d = x.shape
    n_out = W.shape[1]
    valid = (idx >= 0) & (idx < N_r)
    # dropped slots go to an extra expert N_r: the stable sort keeps the valid
    # slots first, in the order dispatch gives them
    _, offsets, perm, inv = oracle.dispatch(np.where(valid, idx, N_r).astype(np.int32),
                                            N_r + 1)
    offsets = offsets[:N_r + 1]
    n_valid = int(offsets[-1])
    ref = oracle.expert_gemm(x, k, perm, offsets, W)  # [n_valid, n_out] exact
    E_ref = oracle.round_bf16(ref)
    if integer:
        e_err = np.zeros_like(ref)
    else:
        xf = np.abs(wl.bf16_bits_to_f32(x).astype(np.float64))
        Wf = np.abs(wl.bf16_bits_to_f32(W).astype(np.float64))
        absdot = np.empty_like(ref)
        for e in range(N_r):
            lo, hi = offsets[e], offsets[e + 1]
            if hi > lo:
                absdot[lo:hi] = xf[perm[lo:hi] // k] @ Wf[e].T
        e_err = 2 * bf16_ulp(ref) + (d / 16 + 2) * 2.0 ** -23 * absdot
    w0 = np.where(valid, w, np.float32(0)).astype(np.float32)
    inv0 = np.where(valid.reshape(-1), inv, 0).astype(np.int32)
    E_full = np.zeros((T * k, n_out), np.float64)
    E_full[:n_valid] = E_ref
    err_full = np.zeros_like(E_full)
    err_full[:n_valid] = e_err
    E_bits = wl.to_bf16_bits(E_full.astype(np.float32))
    ry, rr = oracle.combine(E_bits, w0, inv0, sh, k)
    aw = np.abs(w0).astype(np.float64)[:, :, None]
    s_err = (aw * err_full[inv0].reshape(T, k, n_out)).sum(1)
    s_abs = (aw * np.abs(E_full[inv0]).reshape(T, k, n_out)).sum(1)
    tol = bf16_ulp(rr) + bf16_ulp(ry) + 1.01 * (s_err + (k + 1) * 2.0 ** -23 * s_abs)
    return ry, rr, tol


COMBINE_CASES = [
    # T, d, N_r, k, n_out, skew, integer, shared, packed, gather, drop
    (300, 512, 32, 4, 256, False, True, True, False, "lsu", 0.0),
    (257, 200, 32, 3, 144, True, True, True, True, "tma", 0.0),   # K tail, partial N tile
    (257, 200, 32, 3, 144, True, False, False, False, "tma", 0.0),
    (1000, 512, 64, 8, 256, True, False, True, True, "lsu", 0.0),  # skewed: many blocks
    (256, 7168, 256, 8, 512, False, False, True, True, "lsu", 0.0),  # DeepSeek-V3 shapes
    (600, 256, 16, 4, 256, False, False, True, False, "lsu", 0.1),  # dropped slots
]


@pytest.mark.parametrize("T,d,N_r,k,n_out,skew,integer,with_shared,packed,gather,drop",
                         COMBINE_CASES,
                         ids=[f"T{c[0]}_d{c[1]}_E{c[2]}_n{c[4]}_{'int' if c[6] else 'rand'}"
                              f"{'_packed' if c[8] else ''}_{c[9]}{'_drop' if c[10] else ''}"
                              for c in COMBINE_CASES])
def test_expert_gemm_gather_combine_matches_oracle(T, d, N_r, k, n_out, skew, integer,
                                                   with_shared, packed, gather, drop,
                                                   monkeypatch):
    """y of the fused layer against the oracle (expert layer rounded to bf16,
    then the pages' weighted sum and shared add) within the derived bound of
    _combine_reference; tokens without a routed slot get the shared row."""
    if gather == "tma":
        monkeypatch.setenv("MR_EG_GATHER", "tma")
    seed = 11 * T + d + n_out
    x, W, idx, w, sh = _combine_case(T, d, N_r, k, n_out, seed, skew, integer, with_shared,
                                     drop)
    counts, offsets, perm, inv = mr.mr_dispatch(torch.from_numpy(idx).cuda(), N_r)
    assert mr.mr_get_error() == (mr.MR_ERR_DEVICE if drop > 0 else mr.MR_OK)
    Wd = _dev_bits(W)
    if packed:
        Wd = mr.mr_expert_pack_weights(Wd)
    acc = torch.full((T, n_out), float("nan"), dtype=torch.float32, device="cuda")
    y = mr.mr_expert_gemm_gather_combine(_dev_bits(x), k, perm, offsets, Wd,
                                         torch.from_numpy(w).cuda(),
                                         None if sh is None else _dev_bits(sh), N_r=N_r,
                                         n_out=n_out, packed=packed, acc=acc)
    assert mr.mr_get_error() == mr.MR_OK
    got = wl.bf16_bits_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16))
    got = got.astype(np.float64)
    ry, rr, tol = _combine_reference(x, W, idx, w, sh, k, N_r, integer)
    err = np.abs(got - ry)
    assert np.isfinite(got).all()
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert (err <= tol).all(), f"token {worst[0]} col {worst[1]}: {got[worst]} vs {ry[worst]}"
    if drop > 0:  # token 0 has no routed slot: y = bf16(0 + shared) = shared
        want = sh[0] if sh is not None else np.zeros(n_out, np.uint16)
        assert np.array_equal(y[0].view(torch.int16).cpu().numpy().view(np.uint16), want)
    stats = {"elems": int(err.size), "max_abs_err": float(err.max()),
             "max_err_over_tol": float((err / tol).max()),
             "y_differ_elems": int((err > 0).sum())}
    record(f"expert_combine_T{T}_d{d}_E{N_r}_n{n_out}_{'int' if integer else 'rand'}"
           f"{'_drop' if drop else ''}", "expert_gemm_gather_combine", stats)
    print(stats)


def test_expert_gemm_gather_combine_equals_layer_then_combine_within_bound():
    """The fused layer against the two-step path on the same GPU (the expert
    layer written out, then mr_combine): the same expert outputs, added in
    another order and without the FMA.  The two fp32 sums are each within
    (k + 1) 2^-24 sum|w E| of the exact one; each bf16 rounding can then land
    one ulp apart."""
    T, d, N_r, k, n_out = 512, 1024, 64, 8, 512
    x, W, idx, w, sh = _combine_case(T, d, N_r, k, n_out, 5, True, False, True)
    counts, offsets, perm, inv = mr.mr_dispatch(torch.from_numpy(idx).cuda(), N_r)
    xd, Wd, wd, shd = _dev_bits(x), _dev_bits(W), torch.from_numpy(w).cuda(), _dev_bits(sh)
    acc = torch.empty((T, n_out), dtype=torch.float32, device="cuda")
    fused = mr.mr_expert_gemm_gather_combine(xd, k, perm, offsets, Wd, wd, shd, acc=acc)
    E = mr.mr_expert_gemm_gather(xd, k, perm, offsets, Wd)
    two = mr.mr_combine(E, wd, inv, shd)
    assert mr.mr_get_error() == mr.MR_OK
    a = fused.float().cpu().numpy().astype(np.float64)
    b = two.float().cpu().numpy().astype(np.float64)
    Ef = E.float().cpu().numpy().astype(np.float64)
    s_abs = (np.abs(w).astype(np.float64)[:, :, None]
             * np.abs(Ef[inv.cpu().numpy()]).reshape(T, k, n_out)).sum(1)
    D = 2 * (k + 1) * 2.0 ** -24 * s_abs
    r = np.abs(acc.cpu().numpy().astype(np.float64)) + D
    tol = D + 2 * bf16_ulp(r) + 2 * bf16_ulp(np.abs(b) + D + 2 * bf16_ulp(r))
    assert (np.abs(a - b) <= tol).all()
    assert (a == b).mean() > 0.95  # most elements round identically
