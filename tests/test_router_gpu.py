"""Router parity on the GPU: libmr.so (through its C ABI) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr
import workloads as wl
from parity import compare_router, oracle_router, router_inputs, sample_tokens, to_dev

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
]
FULL = [wl.V3_PREFILL, wl.K2_PREFILL, wl.V3_DECODE, wl.V3_FULL]


def _run(w, precision, x_dtype="f32", want_logits=True, api="ex"):
    d = router_inputs(w)
    x = to_dev(d["x_bf16"], "bf16") if x_dtype == "bf16" else to_dev(d["x_f32"])
    Wd, b = to_dev(d["W"]), to_dev(d["b"])
    if api == "plain":
        idx, wt = mr.mr_router_forward(x, Wd, b, w.n_group, w.topk_group, w.k, w.route_scale,
                                       w.mask_mode)
        logits = None
    else:
        logits = torch.empty((w.T, w.N_r), dtype=torch.float32, device="cuda") \
            if want_logits else None
        idx, wt = mr.mr_router_forward_ex(x, Wd, b, w.n_group, w.topk_group, w.k,
                                          w.route_scale, w.mask_mode, precision=precision,
                                          logits_out=logits)
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


@pytest.mark.parametrize("w", SMALL[:4], ids=[w.name for w in SMALL[:4]])
def test_router_plain_tf32_logits(w):
    """One-product TF32 is reported separately: logits within ~1e-3, not 2e-5."""
    idx, wt, logits = _run(w, mr.MR_PREC_TF32)
    ref = oracle_router(w, np.arange(w.T))
    err = np.abs(logits - ref["logits"]) / np.maximum(np.abs(ref["logits"]), 1.0)
    assert err.max() < 2e-2
    assert (idx >= 0).all() and (idx < w.N_r).all()
    np.testing.assert_allclose(wt.sum(1), w.route_scale, rtol=1e-5)
    print(w.name, "tf32 logit max err", err.max())


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
def test_router_full_size_sampled(w):
    """Every token runs on the GPU in the configuration the benchmark uses;
    the oracle checks a sample of tokens (incl. the first and last)."""
    idx, wt, logits = _run(w, mr.MR_PREC_3XTF32)
    tok = sample_tokens(w.T, 256, seed=w.seed)
    ref = oracle_router(w, tok)
    stats = compare_router(idx[tok], wt[tok], ref, logits[tok])
    # properties that hold for every token
    assert (idx >= 0).all() and (idx < w.N_r).all()
    assert all(len(set(r)) == w.k for r in idx[:: max(1, w.T // 512)])
    np.testing.assert_allclose(wt.sum(1), w.route_scale, rtol=2e-6)
    if w.mask_mode == 0 and w.n_group > 1:
        S = w.N_r // w.n_group
        assert max(len(set(r)) for r in (idx // S).tolist()) <= w.topk_group
    print(w.name, stats)
