"""Shared helpers of the GPU parity tests: cached seeded inputs, oracle runs on
(sampled) tokens and the comparison rules.

Comparison rules (tolerances the routing path is specified with):
  * selection: the set of k expert ids per token is bit-exact wherever the
    oracle's selection and group margins exceed 1e-5 ("near-tie" tokens are
    counted and reported, not hidden); the slot order is bit-exact wherever
    the gaps between consecutive selected scores exceed 1e-5 as well.
  * weights: within 1e-5 relative of the oracle (matched by expert id).
  * logits: |dL| <= 2e-5 * max(|L|, 1).
  * dispatch and gather: bit-exact.
  * combine: |dy| <= 1e-2 * max(|y|, |routed|, |shared|) + 1e-5, plus one
    bf16 ulp of the routed sum for bf16 rows (compare_combine); the 1e-5
    bounds the fp32 accumulation error of k fused multiply-adds
    (k * 2^-24 * sum_j |w_j e_j| <= 8 * 6e-8 * 15 for N(0,1) rows and weights
    summing to <= 2.827), which a bf16 rounding boundary can expose.
"""
from __future__ import annotations

import functools
import json
import os

import numpy as np
import torch

import oracle
import workloads as wl

SEL_EPS = 1e-5
W_RTOL = 1e-5
LOGIT_TOL = 2e-5
Y_RTOL = 1e-2
Y_ATOL = 1e-5


@functools.lru_cache(maxsize=4)
def router_inputs(w: wl.Workload):
    return wl.gen_router_inputs(w)


@functools.lru_cache(maxsize=2)
def row_inputs(w: wl.Workload):
    return {"E": wl.gen_E(w), "shared": wl.gen_shared(w)}


def to_dev(a, dtype=None):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.cuda()


def bf16_dev_to_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    """n tokens spread over [0, T) plus the first and last rows (ragged tail)."""
    if T <= n:
        return np.arange(T, dtype=np.int64)
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, size=n - 2, replace=False).tolist()) | {0, T - 1}
    return np.array(sorted(s), dtype=np.int64)


def oracle_router(w: wl.Workload, tokens: np.ndarray, want_logits=True):
    d = router_inputs(w)
    return oracle.router(d["x_f32"][tokens], d["W"], d["b"], w.n_group, w.topk_group, w.k,
                         w.route_scale, w.mask_mode, want_logits=want_logits)


def compare_router(gidx, gw, ref, glogits=None, logit_tol=LOGIT_TOL, allow_tie_frac=0.01):
    """Compare GPU idx/w (numpy, rows matching ref) with an oracle result."""
    gidx = np.asarray(gidx)
    gw = np.asarray(gw, dtype=np.float64)
    ridx, rw = ref["idx"], ref["w"]
    n = len(ridx)
    # A margin of exactly 0 is an exact tie (e.g. two experts masked to 0.0):
    # both sides break it toward the lower index, so it is compared exactly.
    mg = ref["margins"]
    m_sel = np.minimum(mg[:, 0], mg[:, 1])
    tie = (m_sel <= SEL_EPS) & (m_sel > 0)
    otie = tie | ((mg[:, 2] <= SEL_EPS) & (mg[:, 2] > 0))
    ok = ~tie
    gs, rs = np.sort(gidx, 1), np.sort(ridx, 1)
    bad = ok & (gs != rs).any(1)
    assert not bad.any(), (
        f"{bad.sum()} of {ok.sum()} non-tie tokens select different experts; first: "
        f"row {np.argmax(bad)} gpu {gidx[np.argmax(bad)]} oracle {ridx[np.argmax(bad)]}")
    og, orr = np.argsort(gidx, 1, kind="stable"), np.argsort(ridx, 1, kind="stable")
    wg = np.take_along_axis(gw, og, 1)[ok]
    wr = np.take_along_axis(rw, orr, 1)[ok]
    rel = np.abs(wg - wr) / np.abs(wr)
    assert rel.size == 0 or rel.max() <= W_RTOL, f"weight rel err {rel.max():.3g}"
    okk = ~otie
    assert (gidx[okk] == ridx[okk]).all(), "slot order differs on tokens with clear gaps"
    stats = {"tokens": n, "near_ties": int(tie.sum()), "order_ties": int(otie.sum()),
             "w_max_rel": float(rel.max()) if rel.size else 0.0}
    if glogits is not None and ref["logits"] is not None:
        L = ref["logits"]
        err = np.abs(np.asarray(glogits, np.float64) - L) / np.maximum(np.abs(L), 1.0)
        stats["logit_max_err"] = float(err.max())
        assert err.max() <= logit_tol, f"logit error {err.max():.3g} > {logit_tol}"
    assert tie.sum() <= max(2, allow_tie_frac * n), f"too many near-ties: {tie.sum()} of {n}"
    return stats


def bf16_ulp(a):
    """Spacing of bf16 values at |a| (8 significant bits): 2^(e - 8) for
    |a| = m * 2^e, 0.5 <= m < 1; the subnormal spacing 2^-133 at the bottom."""
    a = np.abs(np.asarray(a, np.float64))
    _, e = np.frexp(a)
    return np.where(a == 0, 2.0 ** -133, np.ldexp(1.0, np.maximum(e - 8, -133)))


def compare_combine(gy, ry, rrouted, shared, bf16=True):
    """gy: GPU y as float64 numpy; ry/rrouted from the oracle; shared float64 or None.

    bf16 rows: the pages round the fp32 routed sum to bf16, then round the
    sum with the shared row again.  The GPU's fp32 sum differs from the exact
    sum by far less than half a bf16 ulp, yet where the exact value sits on a
    rounding boundary the first rounding can land one bf16 ulp of the routed
    sum away from the oracle's, and the second rounding can add one ulp of y
    (< 2^-7 |y|, inside the relative term).  Hence the tolerance
    1e-2 * max(|y|, |routed|, |shared|) + ulp_bf16(routed) + 1e-5."""
    scale = np.maximum(np.abs(ry), np.abs(rrouted))
    if shared is not None:
        scale = np.maximum(scale, np.abs(shared))
    err = np.abs(gy - ry)
    tol = Y_RTOL * scale + Y_ATOL
    if bf16:
        tol = tol + bf16_ulp(rrouted)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert (err <= tol).all(), (f"combine error at {worst}: gpu {gy[worst]} oracle {ry[worst]} "
                                f"tol {tol[worst]}")
    rel_l2 = np.linalg.norm(gy - ry, axis=1) / np.maximum(np.linalg.norm(ry, axis=1), 1e-30)
    return {"y_max_abs": float(err.max()), "y_row_rel_l2_max": float(rel_l2.max()),
            "y_max_err_over_tol": float((err / tol).max()),
            "y_differ_elems": int((err > 0).sum()),
            "y_beyond_1e-2_rel": int((err > Y_RTOL * scale + Y_ATOL).sum())}


def widen(a):
    """bf16 bits (uint16) or fp32 numpy array -> float64."""
    if a.dtype == np.uint16:
        return wl.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def record(config: str, stage: str, stats: dict) -> None:
    """Append one JSON line {config, stage, **stats} to the file named by the
    environment variable MR_PARITY_OUT (nothing when it is unset): the
    per-config parity figures (near-ties, largest errors) of a test run."""
    path = os.environ.get("MR_PARITY_OUT")
    if not path:
        return
    row = {"config": config, "stage": stage}
    row.update({k: (float(v) if isinstance(v, (np.floating,)) else
                    int(v) if isinstance(v, (np.integer,)) else v) for k, v in stats.items()})
    with open(path, "a") as f:
        f.write(json.dumps(row) + "\n")
