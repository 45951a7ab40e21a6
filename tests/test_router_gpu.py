"""Router parity on the GPU: libmr.so (through its C ABI) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr
import workloads as wl
from parity import compare_router, oracle_router, record, router_inputs, to_dev

pytestmark = pytest.mark.gpu

W = wl.Workload
SMALL = [
    wl.TINY,
    W("v3_like_T300_d1000", T=300, d=1000, N_r=256, n_group=8, topk_group=4, k=8,
      route_scale=2.5, mask_mode=0, seed=11),
    W("k2_like_T200", T=200, d=7168, N_r=384, n_group=1, topk_group=1, k=8,
      route_scale=2.827, mask_mode=1, seed=12),
    W("zero_mask_negative_bias_T256", T=256, d=512, N_r=128, n_group=4, topk_group=2, k=8,
      route_scale=2.5, mask_mode=1, seed=13, bias_lo=-1.5, bias_hi=-0.6, io_dtype="f32"),
    W("no_bias_T129", T=129, d=256, N_r=64, n_group=8, topk_group=3, k=6, route_scale=1.0,
      mask_mode=0, seed=14, with_bias=False, io_dtype="f32"),
    W("k1_T100", T=100, d=128, N_r=32, n_group=2, topk_group=1, k=1, route_scale=2.5,
      mask_mode=0, seed=15, io_dtype="f32"),
    W("k3_N16_T77", T=77, d=64, N_r=16, n_group=2, topk_group=1, k=3, route_scale=2.5,
      mask_mode=0, seed=16, io_dtype="f32"),
    W("N512_T160", T=160, d=520, N_r=512, n_group=16, topk_group=4, k=8, route_scale=2.5,
      mask_mode=0, seed=17, io_dtype="f32"),
    W("N320_G10_T140", T=140, d=300, N_r=320, n_group=10, topk_group=3, k=5,
      route_scale=2.5, mask_mode=1, seed=18, io_dtype="f32"),
    # every biased score < 0 = the masked groups' fill: the top-k is mostly
    # masked experts (ties at 0.0 resolved by index), and the kept groups'
    # top-2 bound lies below every candidate
    W("zero_mask_all_negative_T200", T=200, d=256, N_r=256, n_group=8, topk_group=4, k=8,
      route_scale=2.5, mask_mode=1, seed=19, bias_lo=-1.5, bias_hi=-1.1, io_dtype="f32"),
]
FULL = [wl.V3_PREFILL, wl.K2_PREFILL, wl.V3_DECODE, wl.V3_FULL]


def _poisoned(T, k):
    """Output buffers filled with values no kernel writes, so a token the
    kernel skips cannot pass on a stale result of an earlier call."""
    return (torch.full((T, k), -1, dtype=torch.int32, device="cuda"),
            torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda"))


def _run(w, precision, x_dtype="f32", want_logits=True, api="ex"):
    d = router_inputs(w)
    io, wo = _poisoned(w.T, w.k)
    x = to_dev(d["x_bf16"], "bf16") if x_dtype == "bf16" else to_dev(d["x_f32"])
    Wd, b = to_dev(d["W"]), to_dev(d["b"])
    if api == "plain":
        idx, wt = mr.mr_router_forward(x, Wd, b, w.n_group, w.topk_group, w.k, w.route_scale,
                                       w.mask_mode, idx_out=io, w_out=wo)
        logits = None
    else:
        logits = torch.full((w.T, w.N_r), float("nan"), device="cuda") \
            if want_logits else None
        idx, wt = mr.mr_router_forward_ex(x, Wd, b, w.n_group, w.topk_group, w.k,
                                          w.route_scale, w.mask_mode, precision=precision,
                                          idx_out=io, w_out=wo, logits_out=logits)
    torch.cuda.synchronize()
    assert mr.mr_get_error() == mr.MR_OK
    return idx.cpu().numpy(), wt.cpu().numpy(), None if logits is None else logits.cpu().numpy()


@pytest.mark.parametrize("precision", [mr.MR_PREC_3XTF32, mr.MR_PREC_FFMA], ids=["3xtf32", "ffma"])
@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_router_small_all_tokens(w, precision):
    idx, wt, logits = _run(w, precision)
    ref = oracle_router(w, np.arange(w.T))
    stats = compare_router(idx, wt, ref, logits)
    print(w.name, precision, stats)


# Plain TF32 (one tensor-core product per multiply-add).  The tensor core
# reads each fp32 operand with its 13 low mantissa bits dropped (truncation,
# pinned by test_tf32_operand_low_bits_probe), so each operand carries a relative
# error below 2^-10 and a product x_j W_ij one below 2^-9 + 2^-20.  With fp32
# accumulation (round toward zero inside 128-K intervals, rounded sums
# between them: below 128 * 2^-23 + 2^-24 relative) every logit satisfies
#     |L_tf32 - L| <= TF32_LOGIT_COEF * sum_j |x_j W_ij|,
# TF32_LOGIT_COEF = 2^-9 + 2^-20 + 129 * 2^-23 < 1.97e-3.
TF32_LOGIT_COEF = 2.0 ** -9 + 2.0 ** -20 + 129 * 2.0 ** -23


def tf32_check(w, x_f32, idx, wt, logits, tag):
    """TF32 router output against the oracle: the logits within the bound
    above; the selection and weights exactly what the method gives for the
    GPU's own logits (the oracle fed those logits as x with W = identity,
    so its logits equal them), outside the usual 1e-5 near-tie band; and
    the number of tokens whose selection differs from the fp64 selection
    on the true inputs (reported: the cost of the cheaper arithmetic)."""
    d = router_inputs(w)
    ref = oracle_router(w, np.arange(w.T))
    L = ref["logits"]
    absdot = np.abs(np.asarray(x_f32, np.float64)) @ np.abs(d["W"].astype(np.float64)).T
    err = np.abs(logits.astype(np.float64) - L)
    assert (err <= TF32_LOGIT_COEF * absdot).all(), \
        f"TF32 logit error {(err / absdot).max():.3g} x sum|xW| > {TF32_LOGIT_COEF:.3g}"
    eye = np.eye(w.N_r, dtype=np.float32)
    own = oracle.router(logits.astype(np.float32), eye, d["b"], w.n_group, w.topk_group, w.k,
                        w.route_scale, w.mask_mode)
    stats = compare_router(idx, wt, own)
    changed = int((np.sort(idx, 1) != np.sort(ref["idx"], 1)).any(1).sum())
    stats.update({"logit_max_abs_err": float(err.max()),
                  "logit_err_over_bound_max": float((err / (TF32_LOGIT_COEF * absdot)).max()),
                  "selection_changed_vs_fp64": changed})
    record(w.name, tag, stats)
    return stats


@pytest.mark.parametrize("w", SMALL[:4], ids=[w.name for w in SMALL[:4]])
def test_router_plain_tf32_parity(w):
    """One-product TF32, reported separately: logits within the derived TF32
    bound, selection and weights exact given its logits."""
    idx, wt, logits = _run(w, mr.MR_PREC_TF32)
    stats = tf32_check(w, router_inputs(w)["x_f32"], idx, wt, logits, "router_tf32")
    print(w.name, "tf32", stats)


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_router_plain_tf32_full_size(w):
    """The TF32 variant on the full workloads (fused kernel; split-K for the
    64-token decode batch), every token."""
    d = router_inputs(w)
    ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                     device="cuda")
    lg = torch.full((w.T, w.N_r), float("nan"), device="cuda")
    io, wo = _poisoned(w.T, w.k)
    idx, wt = mr.mr_router_forward_ex(to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"]),
                                      w.n_group, w.topk_group, w.k, w.route_scale, w.mask_mode,
                                      precision=mr.MR_PREC_TF32, idx_out=io, w_out=wo,
                                      logits_out=lg, workspace=ws)
    assert mr.mr_get_error() == mr.MR_OK
    stats = tf32_check(w, d["x_f32"], idx.cpu().numpy(), wt.cpu().numpy(), lg.cpu().numpy(),
                       "router_tf32")
    print(w.name, "tf32", stats)


@pytest.mark.parametrize("cs", ["1", "2"])
@pytest.mark.parametrize("w", [SMALL[1], SMALL[3], SMALL[4]], ids=lambda w: w.name)
def test_router_cluster_size_pinned(w, cs, monkeypatch):
    """Both tile shapes of the tensor-core kernel (one CTA with all experts,
    or two CTAs splitting them) on the same inputs."""
    monkeypatch.setenv("MR_TC_CLUSTER", cs)
    idx, wt, logits = _run(w, mr.MR_PREC_3XTF32)
    compare_router(idx, wt, oracle_router(w, np.arange(w.T)), logits)


def test_router_default_entry_point_matches_ex():
    w = SMALL[1]
    a = _run(w, mr.MR_PREC_3XTF32, want_logits=False)
    b = _run(w, None, api="plain")
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()


def test_router_ffma_fallback_shapes():
    """Shapes the tensor-core path does not take (N_r % 16, d % 4) run on the
    CUDA-core path through the default entry point."""
    w = W("ragged_N40_d37_T33", T=33, d=37, N_r=40, n_group=4, topk_group=2, k=4,
          route_scale=2.5, mask_mode=0, seed=19, io_dtype="f32")
    idx, wt, _ = _run(w, None, api="plain")
    compare_router(idx, wt, oracle_router(w, np.arange(w.T), want_logits=False))
    d = router_inputs(w)
    with pytest.raises(mr.MRError) as e:
        mr.mr_router_forward_ex(to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"]), 4, 2, 4,
                                2.5, 0, precision=mr.MR_PREC_3XTF32)
    assert e.value.status == mr.MR_ERR_UNSUPPORTED


def test_router_bf16_input_equals_widened_fp32():
    w = SMALL[1].replace(io_dtype="bf16")
    a = _run(w, mr.MR_PREC_FFMA, x_dtype="bf16")
    b = _run(w, mr.MR_PREC_FFMA, x_dtype="f32")
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all() and (a[2] == b[2]).all()


def test_router_deterministic():
    w = SMALL[2]
    a = _run(w, mr.MR_PREC_3XTF32)
    b = _run(w, mr.MR_PREC_3XTF32)
    for u, v in zip(a, b):
        assert (u == v).all()


def test_router_empty_batch():
    Wd = torch.zeros((64, 128), device="cuda")
    x = torch.zeros((0, 128), device="cuda")
    idx, wt = mr.mr_router_forward(x, Wd, None, 8, 4, 8, 2.5, 0)
    assert idx.shape == (0, 8)


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_router_full_size_every_token(w):
    """The fp32-row (3xTF32) router at full size against the oracle on every
    token: selection, weights and logits."""
    idx, wt, logits = _run(w, mr.MR_PREC_3XTF32)
    ref = oracle_router(w, np.arange(w.T))
    stats = compare_router(idx, wt, ref, logits)
    record(w.name, "router_3xtf32_fp32_rows", stats)
    # properties that hold for every token
    assert (idx >= 0).all() and (idx < w.N_r).all()
    assert all(len(set(r)) == w.k for r in idx[:: max(1, w.T // 512)])
    np.testing.assert_allclose(wt.sum(1), w.route_scale, rtol=2e-6)
    if w.mask_mode == 0 and w.n_group > 1:
        S = w.N_r // w.n_group
        assert max(len(set(r)) for r in (idx // S).tolist()) <= w.topk_group
    print(w.name, stats)


SPLITK = [
    W("splitk_T1", T=1, d=7168, N_r=256, n_group=8, topk_group=4, k=8, route_scale=2.5,
      mask_mode=0, seed=21),
    W("splitk_T7_N384", T=7, d=7168, N_r=384, n_group=1, topk_group=1, k=8,
      route_scale=2.827, mask_mode=1, seed=22),
    W("splitk_T200_d1000", T=200, d=1000, N_r=256, n_group=8, topk_group=4, k=8,
      route_scale=2.5, mask_mode=0, seed=23),
    W("splitk_T256_N64", T=256, d=516, N_r=64, n_group=4, topk_group=2, k=4, route_scale=2.5,
      mask_mode=1, seed=24, io_dtype="f32"),
    wl.V3_DECODE,
]


SPLITK_CASES = [(w, "f32") for w in SPLITK] + [(w, "bf16") for w in SPLITK
                                                if w.io_dtype == "bf16"]


@pytest.mark.parametrize("routing", ["default", "cta"])
@pytest.mark.parametrize("w,rows", SPLITK_CASES, ids=[f"{w.name}-{r}" for w, r in SPLITK_CASES])
def test_router_splitk_small_batches(w, rows, routing, monkeypatch):
    """Batches of up to 256 tokens with a workspace take the split-K path
    (K-sliced tensor-core GEMM over all SMs, cluster reduction, reduce-and-
    route), for fp32 rows and for bf16 rows (staged as bf16, widened in
    shared memory).  d = 7168 and 1000 reduce the K slices in clusters of 8;
    d = 516 has too few K chunks for that and writes every slice.  The
    slices are reduced and routed by the routing kernel where its lane
    layout fits (default) or, pinned by MR_ROUTE_KERNEL=0, by one CTA per
    token (the kernel shapes without a lane layout take)."""
    if routing == "cta":
        monkeypatch.setenv("MR_ROUTE_KERNEL", "0")
    n = mr.mr_router_workspace_size(w.T, w.d, w.N_r)
    assert n > 0
    d = router_inputs(w)
    x = to_dev(d["x_bf16"], "bf16") if rows == "bf16" else to_dev(d["x_f32"])
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    logits = torch.full((w.T, w.N_r), float("nan"), device="cuda")
    io, wo = _poisoned(w.T, w.k)
    l0 = mr.mr_launch_count()
    idx, wt = mr.mr_router_forward_ex(x, to_dev(d["W"]), to_dev(d["b"]),
                                      w.n_group, w.topk_group, w.k, w.route_scale, w.mask_mode,
                                      idx_out=io, w_out=wo, logits_out=logits, workspace=ws)
    assert mr.mr_launch_count() - l0 == 2  # GEMM + reduce/route
    assert mr.mr_get_error() == mr.MR_OK
    ref = oracle_router(w, np.arange(w.T))
    stats = compare_router(idx.cpu().numpy(), wt.cpu().numpy(), ref, logits.cpu().numpy())
    print(w.name, rows, stats)
    # deterministic: slices are summed in a fixed order
    idx2, wt2 = mr.mr_router_forward_ex(x, to_dev(d["W"]), to_dev(d["b"]),
                                        w.n_group, w.topk_group, w.k, w.route_scale,
                                        w.mask_mode, workspace=ws)
    assert torch.equal(idx, idx2) and torch.equal(wt, wt2)
    if rows == "bf16":
        # the same logits as the fp32 cast of the rows, bit for bit: both
        # stage the same fp32 values and a bf16 row has no tf32 residual
        lf = torch.full_like(logits, float("nan"))
        mr.mr_router_forward_ex(to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"]), w.n_group,
                                w.topk_group, w.k, w.route_scale, w.mask_mode,
                                logits_out=lf, workspace=ws)
        assert torch.equal(lf, logits)


# Routing shapes of the decode reduce-and-route kernel: whole-CTA routing
# with groups of 1, 2 and 4 warps or none, a partial last warp, a single warp,
# and the cases that hand the token to the one-warp routine (the kept groups'
# top-2 pairs give fewer than k values; ties at the 0.0 fill of masked
# experts beat the bound).
ROUTE_SHAPES = [
    W("route_g4_two_warps_per_group", T=96, d=512, N_r=256, n_group=4, topk_group=2, k=8,
      route_scale=2.5, mask_mode=0, seed=61),
    W("route_g2_four_warps_per_group", T=96, d=512, N_r=256, n_group=2, topk_group=1, k=6,
      route_scale=1.0, mask_mode=0, seed=62),
    W("route_no_groups_N256_zero_fill", T=96, d=512, N_r=256, n_group=1, topk_group=1, k=8,
      route_scale=2.827, mask_mode=1, seed=63),
    W("route_no_groups_N208", T=96, d=512, N_r=208, n_group=1, topk_group=1, k=8,
      route_scale=1.0, mask_mode=0, seed=64),
    W("route_no_groups_N32", T=96, d=512, N_r=32, n_group=1, topk_group=1, k=4,
      route_scale=1.0, mask_mode=0, seed=65),
    W("route_g8_keep2_too_few_pairs", T=96, d=512, N_r=256, n_group=8, topk_group=2, k=8,
      route_scale=2.5, mask_mode=0, seed=66),
    W("route_zero_fill_negative_bias", T=96, d=512, N_r=256, n_group=8, topk_group=4, k=8,
      route_scale=2.5, mask_mode=1, seed=67, bias_lo=-0.95, bias_hi=-0.8),
]


@pytest.mark.parametrize("routing", ["default", "cta"])
@pytest.mark.parametrize("w", ROUTE_SHAPES, ids=[w.name for w in ROUTE_SHAPES])
def test_router_splitk_routing_shapes(w, routing, monkeypatch):
    """Every token of each routing shape of the split-K path against the
    oracle (expert sets exact outside near-ties, weights within tolerance),
    reduced and routed by the routing kernel where its lane layout fits and
    by one CTA per token (MR_ROUTE_KERNEL=0)."""
    if routing == "cta":
        monkeypatch.setenv("MR_ROUTE_KERNEL", "0")
    d = router_inputs(w)
    ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                     device="cuda")
    logits = torch.full((w.T, w.N_r), float("nan"), device="cuda")
    io, wo = _poisoned(w.T, w.k)
    l0 = mr.mr_launch_count()
    idx, wt = mr.mr_router_forward_ex(to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"]),
                                      w.n_group, w.topk_group, w.k, w.route_scale, w.mask_mode,
                                      idx_out=io, w_out=wo, logits_out=logits, workspace=ws)
    assert mr.mr_launch_count() - l0 == 2  # the split-K GEMM + reduce-and-route
    assert mr.mr_get_error() == mr.MR_OK
    ref = oracle_router(w, np.arange(w.T))
    stats = compare_router(idx.cpu().numpy(), wt.cpu().numpy(), ref, logits.cpu().numpy())
    print(w.name, stats)


def test_router_workspace_for_large_batches_holds_w_planes():
    # three bf16 planes of W (which also covers W's fp32 tf32-residuals)
    # and, for a K-split batch, room after them for the partial sums the
    # routing kernel adds (4096 tokens: 4 slices)
    planes = 3 * 2 * 7168 * 256
    assert mr.mr_router_workspace_size(16384, 7168, 256) == planes
    assert mr.mr_router_workspace_size(4096, 7168, 256) >= planes + 4 * 4096 * 256 * 4


@pytest.mark.parametrize("w", [SMALL[1], SMALL[2].replace(name="k2_like_T300", T=300),
                               wl.V3_PREFILL], ids=lambda w: w.name)
def test_router_with_precomputed_residuals_is_identical(w):
    """Above 256 tokens a workspace makes the fused path read W's tf32
    residuals precomputed (one extra launch; a K-split batch also hands its
    partial sums to the routing kernel, one more); results are bit-identical
    (the slices are added in the same order either way)."""
    assert w.T > 256  # (smaller batches take the split-K path instead)
    d = router_inputs(w)
    args = (to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"]), w.n_group, w.topk_group, w.k,
            w.route_scale, w.mask_mode)
    ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                     device="cuda")
    l0 = mr.mr_launch_count()
    a = mr.mr_router_forward_ex(*args, workspace=ws)
    assert mr.mr_launch_count() - l0 in (2, 3)
    b = mr.mr_router_forward_ex(*args)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert mr.mr_get_error() == mr.MR_OK


def test_tf32_operand_low_bits_probe():
    """The tensor core reads an fp32 operand of kind::tf32 with its 13 low
    mantissa bits ignored (truncation).  The 3xTF32 kernels rely on it: the
    staged fp32 tile serves as the hi operand and only lo = v - trunc(v) is
    materialised."""
    d, N = 32, 16
    x = torch.zeros((1, d), device="cuda")
    x[0, 0] = 1.0
    ulp = 2.0 ** -10
    vals = np.array([1.0 + j * ulp / 8 + 2.0 ** -22 for j in range(N)], np.float32)
    W = torch.zeros((N, d), device="cuda")
    W[:, 0] = torch.from_numpy(vals).cuda()
    logits = torch.empty((1, N), device="cuda")
    mr.mr_router_forward_ex(x, W, None, 1, 1, 1, 1.0, 0, precision=mr.MR_PREC_TF32,
                            logits_out=logits)
    got = logits.cpu().numpy()[0].astype(np.float64)
    u = vals.view(np.uint32)
    trunc = (u & np.uint32(0xFFFFE000)).view(np.float32).astype(np.float64)
    rn = np.array([np.round(v / ulp) * ulp for v in vals.astype(np.float64)])
    kind = "truncate" if np.array_equal(got, trunc) else "round" if np.array_equal(got, rn) \
        else "other"
    print("tf32 operand low bits:", kind, got[:10])
    # The 3xTF32 kernels stage raw fp32 tiles as the hi operand and rely on it.
    assert kind == "truncate"


BF16X3 = [
    SMALL[1],                                              # V3-like, ragged T and K tail
    SMALL[2].replace(name="k2_like_T300", T=300),          # 384 experts, 2-CTA split
    W("bf16x3_N16_T77", T=77, d=64, N_r=16, n_group=2, topk_group=1, k=3, route_scale=2.5,
      mask_mode=0, seed=31),
    W("bf16x3_N320_G10_T140", T=140, d=304, N_r=320, n_group=10, topk_group=3, k=5,
      route_scale=2.5, mask_mode=1, seed=32, bias_lo=-0.8, bias_hi=-0.2),
    W("bf16x3_no_bias_T129", T=129, d=256, N_r=64, n_group=8, topk_group=3, k=6,
      route_scale=1.0, mask_mode=0, seed=33, with_bias=False),
    W("bf16x3_zero_mask_all_negative_T300", T=300, d=512, N_r=256, n_group=8, topk_group=4,
      k=8, route_scale=2.5, mask_mode=1, seed=34, bias_lo=-1.5, bias_hi=-1.1),
]


def _run_bf16x3(w, precision=mr.MR_PREC_BF16X3, logits=True):
    d = router_inputs(w)
    ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                     device="cuda")
    lg = torch.full((w.T, w.N_r), float("nan"), device="cuda") if logits else None
    io, wo = _poisoned(w.T, w.k)
    idx, wt = mr.mr_router_forward_ex(to_dev(d["x_bf16"], "bf16"), to_dev(d["W"]),
                                      to_dev(d["b"]), w.n_group, w.topk_group, w.k,
                                      w.route_scale, w.mask_mode, precision=precision,
                                      idx_out=io, w_out=wo, logits_out=lg, workspace=ws)
    assert mr.mr_get_error() == mr.MR_OK
    return idx.cpu().numpy(), wt.cpu().numpy(), None if lg is None else lg.cpu().numpy()


@pytest.mark.parametrize("w", BF16X3, ids=[w.name for w in BF16X3])
def test_router_bf16x3_small_all_tokens(w):
    """bf16 activations: W split into three bf16 planes, exact products,
    fp32 accumulation -- same tolerances as the fp32 path."""
    assert w.io_dtype == "bf16"
    idx, wt, logits = _run_bf16x3(w)
    stats = compare_router(idx, wt, oracle_router(w, np.arange(w.T)), logits)
    print(w.name, "bf16x3", stats)


@pytest.mark.parametrize("cs", ["1", "2", "P"])
@pytest.mark.parametrize("w", [SMALL[1], BF16X3[5]], ids=lambda w: w.name)
def test_router_bf16x3_cluster_size_pinned(w, cs, monkeypatch):
    """Every way the bf16x3 kernel can cover a tile: one CTA, two CTAs
    splitting the experts, or a 2-SM pair running one M = 256 MMA (T = 300
    gives an odd tile count, so a pair's second tile lies past T)."""
    monkeypatch.setenv("MR_TC_CLUSTER", cs)
    idx, wt, logits = _run_bf16x3(w)
    compare_router(idx, wt, oracle_router(w, np.arange(w.T)), logits)


@pytest.mark.parametrize("w", [wl.V3_PREFILL, wl.K2_PREFILL, wl.V3_DECODE, wl.V3_FULL],
                         ids=lambda w: w.name)
def test_router_bf16x3_full_size_every_token(w):
    """bf16 rows (the benchmark's router arithmetic) at full size against the
    oracle on every token, logits included (T <= 256 runs split-K)."""
    idx, wt, logits = _run_bf16x3(w)
    stats = compare_router(idx, wt, oracle_router(w, np.arange(w.T)), logits)
    np.testing.assert_allclose(wt.sum(1), w.route_scale, rtol=2e-6)
    record(w.name, "router_bf16_rows", stats)
    print(w.name, "bf16x3", stats)


def test_router_bf16_input_needs_workspace_on_tensor_cores():
    w = SMALL[1]
    d = router_inputs(w)
    with pytest.raises(mr.MRError) as e:
        mr.mr_router_forward_ex(to_dev(d["x_bf16"], "bf16"), to_dev(d["W"]), to_dev(d["b"]),
                                w.n_group, w.topk_group, w.k, w.route_scale, w.mask_mode,
                                precision=mr.MR_PREC_BF16X3)
    assert e.value.status == mr.MR_ERR_UNSUPPORTED


# --------------------------------------------------------------------------
# Scoring variants of the DeepSeek-V3.2-Exp Gate (softmax scores without
# renormalisation, largest-score group score, no 1e-20), on every path.

VARIANTS = {
    "softmax": (mr.MR_SCORE_SOFTMAX, dict(score="softmax")),
    "group_max": (mr.MR_GROUP_MAX, dict(group_score="max")),
    "no_eps": (mr.MR_NORM_NO_EPS, dict(eps=False)),
    "v32_softmax_nobias": (mr.MR_SCORE_SOFTMAX | mr.MR_GROUP_MAX | mr.MR_NORM_NO_EPS,
                           dict(score="softmax", group_score="max", eps=False)),
}

VAR_W = [
    W("var_v3_T300", T=300, d=512, N_r=256, n_group=8, topk_group=4, k=8, route_scale=2.5,
      mask_mode=0, seed=41),
    W("var_k2_T260", T=260, d=256, N_r=384, n_group=1, topk_group=1, k=8, route_scale=2.827,
      mask_mode=1, seed=42),
    W("var_zero_mask_T200", T=200, d=256, N_r=128, n_group=4, topk_group=2, k=6, route_scale=2.5,
      mask_mode=1, seed=43, bias_lo=-0.6, bias_hi=0.1),
]


def _variant_ref(w, tok, okw, no_bias):
    d = router_inputs(w)
    b = None if no_bias else d["b"]
    return oracle.router(d["x_f32"][tok], d["W"], b, w.n_group, w.topk_group, w.k,
                         w.route_scale, w.mask_mode, want_logits=True, **okw)


def _variant_run(w, flags, rows, precision, no_bias, ws=True):
    d = router_inputs(w)
    x = to_dev(d["x_bf16"], "bf16") if rows == "bf16" else to_dev(d["x_f32"])
    b = None if no_bias else to_dev(d["b"])
    wsb = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                      device="cuda") if ws else None
    lg = torch.full((w.T, w.N_r), float("nan"), device="cuda")
    io, wo = _poisoned(w.T, w.k)
    idx, wt = mr.mr_router_forward_ex(x, to_dev(d["W"]), b, w.n_group, w.topk_group, w.k,
                                      w.route_scale, w.mask_mode, precision=precision,
                                      idx_out=io, w_out=wo, logits_out=lg, workspace=wsb,
                                      flags=flags)
    assert mr.mr_get_error() == mr.MR_OK
    return idx.cpu().numpy(), wt.cpu().numpy(), lg.cpu().numpy()


@pytest.mark.parametrize("var", sorted(VARIANTS))
@pytest.mark.parametrize("path", ["fused_bf16x3", "fused_3xtf32", "splitk_bf16", "ffma"])
@pytest.mark.parametrize("w", VAR_W, ids=[w.name for w in VAR_W])
def test_router_scoring_variants(w, path, var):
    flags, okw = VARIANTS[var]
    no_bias = var == "v32_softmax_nobias"
    if path == "splitk_bf16":
        w = w.replace(T=100)
    tok = np.arange(w.T)
    rows = "f32" if path in ("fused_3xtf32",) else "bf16"
    prec = {"fused_bf16x3": mr.MR_PREC_BF16X3, "fused_3xtf32": mr.MR_PREC_3XTF32,
            "splitk_bf16": mr.MR_PREC_BF16X3, "ffma": mr.MR_PREC_FFMA}[path]
    if path == "ffma":
        w = w.replace(T=96)
        tok = np.arange(w.T)
    idx, wt, lg = _variant_run(w, flags, rows, prec, no_bias, ws=path != "ffma")
    ref = _variant_ref(w, tok, okw, no_bias)
    # softmax scores are O(1/N_r), so the absolute 1e-5 near-tie band (made for
    # O(1) sigmoid scores) holds a few percent of the tokens; they are still
    # counted and excluded from the exact comparison only
    tie_frac = 0.05 if okw.get("score") == "softmax" else 0.01
    stats = compare_router(idx, wt, ref, lg, allow_tie_frac=tie_frac)
    if var in ("softmax", "v32_softmax_nobias"):
        assert (wt.sum(1) < w.route_scale).all()  # not renormalised
    else:
        np.testing.assert_allclose(wt.sum(1), w.route_scale, rtol=2e-6)
    print(w.name, path, var, stats)


@pytest.mark.parametrize("cs", ["1", "2", "P"])
def test_router_softmax_every_tile_shape(cs, monkeypatch):
    """Softmax needs each token's largest logit and sum of exponentials over
    all experts: over the two column halves, and with CS = 2 over the two
    CTAs that split the experts."""
    monkeypatch.setenv("MR_TC_CLUSTER", cs)
    w = VAR_W[0]
    flags, okw = VARIANTS["softmax"]
    idx, wt, lg = _variant_run(w, flags, "bf16", mr.MR_PREC_BF16X3, False)
    compare_router(idx, wt, _variant_ref(w, np.arange(w.T), okw, False), lg, allow_tie_frac=0.05)


def test_router_no_eps_underflow_gives_nan_like_the_page():
    """Every chosen sigmoid score underflows to 0: with the 1e-20 the weights
    are 0, without it 0/0 -- both as the oracle computes them."""
    T, d, N = 4, 64, 64
    x = torch.zeros((T, d), device="cuda")
    x[:, 0] = 1.0
    Wt = torch.zeros((N, d), device="cuda")
    Wt[:, 0] = -1000.0
    for flags, want_nan in ((0, False), (mr.MR_NORM_NO_EPS, True)):
        _, wt = mr.mr_router_forward_ex(x, Wt, None, 1, 1, 4, 2.5, 0, flags=flags)
        got = wt.cpu().numpy()
        assert np.isnan(got).all() if want_nan else (got == 0).all()


@pytest.mark.parametrize("w", SPLITK, ids=[w.name for w in SPLITK])
def test_router_plain_entry_point_picks_splitk_for_small_batches(w):
    """The plain entry point (no workspace argument) runs batches of up to 256
    tokens on the split-K path -- two launches, its partials in the library's
    own array -- with the same results as mr_router_forward_ex given a
    workspace, and parity with the oracle on every token."""
    d = router_inputs(w)
    x, Wd, b = to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"])
    io, wo = _poisoned(w.T, w.k)
    l0 = mr.mr_launch_count()
    idx, wt = mr.mr_router_forward(x, Wd, b, w.n_group, w.topk_group, w.k, w.route_scale,
                                   w.mask_mode, idx_out=io, w_out=wo)
    assert mr.mr_launch_count() - l0 == 2  # split-K GEMM + reduce/route
    assert mr.mr_get_error() == mr.MR_OK
    ref = oracle_router(w, np.arange(w.T), want_logits=False)
    print(w.name, compare_router(idx.cpu().numpy(), wt.cpu().numpy(), ref))
    ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                     device="cuda")
    idx2, wt2 = mr.mr_router_forward_ex(x, Wd, b, w.n_group, w.topk_group, w.k, w.route_scale,
                                        w.mask_mode, workspace=ws)
    assert torch.equal(idx, idx2) and torch.equal(wt, wt2)


def test_router_plain_small_batches_on_two_streams():
    """Calls of the plain entry point on two streams share its split-K array;
    the library orders them, so interleaved calls on unordered streams each
    get their own batch's result."""
    ws_ = [SPLITK[0], SPLITK[2], wl.V3_DECODE]
    ins = []
    for w in ws_:
        d = router_inputs(w)
        ins.append((w, to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"])))
    refs = [mr.mr_router_forward(x, Wd, b, w.n_group, w.topk_group, w.k, w.route_scale,
                                 w.mask_mode) for w, x, Wd, b in ins]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for rep in range(6):
        for j, (w, x, Wd, b) in enumerate(ins):
            s = streams[(rep + j) % 2]
            outs.append((j, mr.mr_router_forward(x, Wd, b, w.n_group, w.topk_group, w.k,
                                                  w.route_scale, w.mask_mode, stream=s)))
    torch.cuda.synchronize()
    assert mr.mr_get_error() == mr.MR_OK
    for j, (idx, wt) in outs:
        assert torch.equal(idx, refs[j][0]) and torch.equal(wt, refs[j][1])


def test_router_plain_large_batches_stay_fused():
    """Above 256 tokens the plain entry point runs the fused kernel (one
    launch: no W residual pass without a workspace)."""
    w = SMALL[1]
    d = router_inputs(w)
    l0 = mr.mr_launch_count()
    idx, wt = mr.mr_router_forward(to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"]),
                                   w.n_group, w.topk_group, w.k, w.route_scale, w.mask_mode)
    assert mr.mr_launch_count() - l0 == 1
    assert mr.mr_get_error() == mr.MR_OK
    compare_router(idx.cpu().numpy(), wt.cpu().numpy(),
                   oracle_router(w, np.arange(w.T), want_logits=False))
    assert mr.mr_router_forward_max_scratch() == 2 << 20


# --------------------------------------------------------------------------
# Gate weight stored in bf16 (mr_router_forward_bf16w).  The oracle gets the
# widened bf16 values of W; with bf16 rows every product is exact in fp32, so
# the tolerances of the fp32 path hold.

BF16W = [
    SMALL[1],                                              # fused, ragged T and K tail
    SMALL[2].replace(name="k2_like_bf16w_T300", T=300),    # 384 experts, 2-CTA split
    BF16X3[2],                                             # N_r = 16, k = 3
    BF16X3[3],                                             # 320 experts in 10 groups, zero mask
    BF16X3[5],                                             # all biased scores negative
    SPLITK[0], SPLITK[1], SPLITK[2], wl.V3_DECODE,         # decode sizes: split-K
]


def _bf16w_ref(w, tok):
    d = router_inputs(w)
    Wf = wl.gen_W_bf16(w)["W_f32"]
    return oracle.router(d["x_f32"][tok], Wf, d["b"], w.n_group, w.topk_group, w.k,
                         w.route_scale, w.mask_mode, want_logits=True)


def _bf16w_run(w, rows="bf16", workspace=True):
    d = router_inputs(w)
    Wb = to_dev(wl.gen_W_bf16(w)["W_bf16"], "bf16")
    x = to_dev(d["x_bf16"], "bf16") if rows == "bf16" else to_dev(d["x_f32"])
    ws = torch.empty(mr.mr_router_workspace_size(w.T, w.d, w.N_r), dtype=torch.uint8,
                     device="cuda") if workspace else None
    lg = torch.full((w.T, w.N_r), float("nan"), device="cuda")
    io, wo = _poisoned(w.T, w.k)
    l0 = mr.mr_launch_count()
    idx, wt = mr.mr_router_forward_bf16w(x, Wb, to_dev(d["b"]), w.n_group, w.topk_group, w.k,
                                         w.route_scale, w.mask_mode, idx_out=io, w_out=wo,
                                         logits_out=lg, workspace=ws)
    launches = mr.mr_launch_count() - l0
    assert mr.mr_get_error() == mr.MR_OK
    return idx.cpu().numpy(), wt.cpu().numpy(), lg.cpu().numpy(), launches


@pytest.mark.parametrize("w", BF16W, ids=[w.name for w in BF16W])
def test_router_bf16_weights_all_tokens(w):
    """bf16 rows x bf16-stored W on the tensor cores (fused kernel with one
    bf16 plane, or split-K with kind::f16 for <= 256 tokens) against the
    oracle on the widened W: every token, fp32 tolerances."""
    assert w.io_dtype == "bf16"
    idx, wt, lg, launches = _bf16w_run(w)
    assert launches == (2 if w.T <= 256 else 1)
    stats = compare_router(idx, wt, _bf16w_ref(w, np.arange(w.T)), lg)
    record(w.name, "router_bf16_weights", stats)
    print(w.name, "bf16 W", stats)


def test_router_bf16_weights_without_workspace_and_fp32_rows():
    """Decode-size batch without a workspace (the library's split-K array),
    and fp32 rows (CUDA-core path on the widened W): same results as the
    oracle."""
    w = wl.V3_DECODE
    ref = _bf16w_ref(w, np.arange(w.T))
    idx, wt, lg, launches = _bf16w_run(w, workspace=False)
    assert launches == 2
    compare_router(idx, wt, ref, lg)
    w2 = SMALL[1]
    idx, wt, lg, launches = _bf16w_run(w2, rows="f32", workspace=False)
    assert launches == 1
    compare_router(idx, wt, _bf16w_ref(w2, np.arange(w2.T)), lg)


@pytest.mark.parametrize("cs", ["1", "2", "P"])
def test_router_bf16_weights_every_tile_shape(cs, monkeypatch):
    monkeypatch.setenv("MR_TC_CLUSTER", cs)
    w = BF16X3[5]
    idx, wt, lg, _ = _bf16w_run(w)
    compare_router(idx, wt, _bf16w_ref(w, np.arange(w.T)), lg)


@pytest.mark.parametrize("w", [wl.V3_PREFILL, wl.K2_PREFILL, wl.V3_FULL], ids=lambda w: w.name)
def test_router_bf16_weights_full_size_every_token(w):
    idx, wt, lg, launches = _bf16w_run(w)
    assert launches == 1
    stats = compare_router(idx, wt, _bf16w_ref(w, np.arange(w.T)), lg)
    np.testing.assert_allclose(wt.sum(1), w.route_scale, rtol=2e-6)
    record(w.name, "router_bf16_weights", stats)
    print(w.name, "bf16 W", stats)


# --------------------------------------------------------------------------
# K-split clusters: 2 or 4 CTAs share one 128-token tile's K loop and meet
# through distributed shared memory (the default for batches with few tiles).

@pytest.mark.parametrize("ks", ["K2", "K4"])
@pytest.mark.parametrize("path", ["3xtf32", "tf32", "bf16x3", "bf16w", "softmax"])
def test_router_ksplit_shapes(ks, path, monkeypatch):
    monkeypatch.setenv("MR_TC_CLUSTER", ks)
    if path == "3xtf32":
        w = SMALL[1]  # T = 300: ragged last tile, d = 1000: K tail
        idx, wt, lg = _run(w, mr.MR_PREC_3XTF32)
        compare_router(idx, wt, oracle_router(w, np.arange(w.T)), lg)
    elif path == "tf32":
        w = SMALL[3]
        idx, wt, lg = _run(w, mr.MR_PREC_TF32)
        tf32_check(w, router_inputs(w)["x_f32"], idx, wt, lg, "router_tf32_ksplit")
    elif path == "bf16x3":
        w = BF16X3[5]  # zero mask, every biased score negative
        idx, wt, lg = _run_bf16x3(w)
        compare_router(idx, wt, oracle_router(w, np.arange(w.T)), lg)
    elif path == "bf16w":
        w = BF16X3[0]
        idx, wt, lg, launches = _bf16w_run(w)
        assert launches == 1
        compare_router(idx, wt, _bf16w_ref(w, np.arange(w.T)), lg)
    else:
        w = VAR_W[0]
        flags, okw = VARIANTS["softmax"]
        idx, wt, lg = _variant_run(w, flags, "bf16", mr.MR_PREC_BF16X3, False)
        compare_router(idx, wt, _variant_ref(w, np.arange(w.T), okw, False), lg,
                       allow_tie_frac=0.05)


def test_router_ksplit_is_deterministic_and_matches_one_cta():
    """The K-split sums the slices in a fixed order: repeated calls agree bit
    for bit, and the selection equals one CTA per tile's (the logits may
    differ in the last bits: the summation order differs)."""
    w = wl.V3_PREFILL.replace(name="v3_T1000", T=1000)
    a = _run_bf16x3(w)
    b = _run_bf16x3(w)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    ref = oracle_router(w, np.arange(w.T))
    compare_router(a[0], a[1], ref, a[2])


# ---- routing after the GEMM: the routing kernel and the GEMM's epilogue ----
# With a workspace of mr_router_workspace_size bytes, the CTAs of a K-split
# tile (or of an expert split) write their partial sums (their logits) to the
# workspace and a routing kernel of P lanes per token adds them and routes;
# MR_ROUTE_KERNEL=0 keeps the exchanges through distributed shared memory and
# the routing in the GEMM's epilogue (=1 routes every shape after the GEMM),
# MR_ROUTE_LANES pins P, MR_TC_CLUSTER=K2 / K4 forces the K split.

def _launches(fn):
    n0 = mr.mr_launch_count()
    out = fn()
    torch.cuda.synchronize()
    return out, mr.mr_launch_count() - n0


@pytest.mark.parametrize("route", ["kernel", "epilogue"])
def test_router_routing_kernel_launches(route, monkeypatch):
    """bf16x3 fused, K split: W split + GEMM + routing kernel (3 launches);
    the epilogue routing: 2."""
    monkeypatch.setenv("MR_TC_CLUSTER", "K2")
    if route == "epilogue":
        monkeypatch.setenv("MR_ROUTE_KERNEL", "0")
    w = SMALL[1]
    (idx, wt, lg), n = _launches(lambda: _run_bf16x3(w))
    assert n == (3 if route == "kernel" else 2)
    compare_router(idx, wt, oracle_router(w, np.arange(w.T)), lg)


# shapes of the small cases with more than 256 tokens (smaller batches take
# split-K): groups of 8, 16 and 32 experts, 2 or 4 lanes per group, no groups,
# 64 to 512 experts, the zero fill, and N = 320 in groups of 32 split over
# two CTAs (160 experts each), which no lane layout fits (epilogue routing)
ROUTE_W = [SMALL[1], SMALL[3].replace(name="zero_mask_N128_T333", T=333, io_dtype="bf16"),
           SMALL[4].replace(name="no_bias_N64_G8_T301", T=301, io_dtype="bf16"),
           SMALL[7].replace(name="N512_G16_T290", T=290, io_dtype="bf16"),
           BF16X3[3].replace(name="N320_G10_T280", T=280), BF16X3[5],
           wl.K2_PREFILL.replace(name="k2_T300", T=300),
           wl.V3_PREFILL.replace(name="v3_T777", T=777)]


@pytest.mark.parametrize("lanes", ["8", "16", "32"])
@pytest.mark.parametrize("w", ROUTE_W, ids=lambda w: w.name)
def test_router_routing_kernel_every_lane_layout(w, lanes, monkeypatch):
    """Every lane layout the shape allows (8, 16 or 32 lanes per token) gives
    the oracle's routing, after a K split or (more than 256 experts) two CTAs
    splitting the experts; a layout that does not fit is routed by the
    epilogue (2 launches) with the same result."""
    monkeypatch.setenv("MR_TC_CLUSTER", "K2")
    monkeypatch.setenv("MR_ROUTE_LANES", lanes)
    (idx, wt, lg), n = _launches(lambda: _run_bf16x3(w))
    assert n in (2, 3)
    compare_router(idx, wt, oracle_router(w, np.arange(w.T)), lg)


@pytest.mark.parametrize("var", sorted(VARIANTS))
@pytest.mark.parametrize("route", ["kernel", "epilogue"])
@pytest.mark.parametrize("w", VAR_W, ids=[w.name for w in VAR_W])
def test_router_scoring_variants_both_routings(w, route, var, monkeypatch):
    monkeypatch.setenv("MR_TC_CLUSTER", "K2")
    if route == "epilogue":
        monkeypatch.setenv("MR_ROUTE_KERNEL", "0")
    flags, okw = VARIANTS[var]
    no_bias = var == "v32_softmax_nobias"
    idx, wt, lg = _variant_run(w, flags, "bf16", mr.MR_PREC_BF16X3, no_bias)
    tie_frac = 0.05 if okw.get("score") == "softmax" else 0.01
    compare_router(idx, wt, _variant_ref(w, np.arange(w.T), okw, no_bias), lg,
                   allow_tie_frac=tie_frac)


@pytest.mark.parametrize("ks", ["1", "K2", "K4"])
@pytest.mark.parametrize("route", ["kernel", "epilogue"])
def test_router_ksplit_both_routings(ks, route, monkeypatch):
    """K-split partial sums meet either in the routing kernel (slices added in
    order from the workspace) or through distributed shared memory."""
    monkeypatch.setenv("MR_TC_CLUSTER", ks)
    if route == "epilogue":
        monkeypatch.setenv("MR_ROUTE_KERNEL", "0")
    for w in (SMALL[1], BF16X3[5]):
        idx, wt, lg = _run_bf16x3(w)
        compare_router(idx, wt, oracle_router(w, np.arange(w.T)), lg)
        a = _run_bf16x3(w)
        assert np.array_equal(a[0], idx) and np.array_equal(a[1], wt)


@pytest.mark.parametrize("route", ["0", "1"], ids=["epilogue", "routing_kernel"])
@pytest.mark.parametrize("w", [wl.V3_PREFILL, wl.K2_PREFILL, wl.V3_FULL], ids=lambda w: w.name)
def test_router_both_routings_full_size_every_token(w, route, monkeypatch):
    """Each routing for every full-size batch (whichever the default takes),
    every token."""
    monkeypatch.setenv("MR_ROUTE_KERNEL", route)
    idx, wt, logits = _run_bf16x3(w)
    compare_router(idx, wt, oracle_router(w, np.arange(w.T)), logits)
