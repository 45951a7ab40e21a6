"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a hand-derived case, a brute-force search, a closed form, a
library routine (BLAS, numpy sorting, torch's bf16 cast) or an invariant the
pages state.  Each is chosen so that a plausible slip in the oracle (dropped
bias, bias in the weights, wrong group score, wrong mask value, transposed
perm/inverse, wrong tie order, missing rounding) fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import expit

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _frac(v):
    return Fraction(v) if isinstance(v, str) else Fraction(v)


def _one_hot_logits(s_list):
    """Token x = e_0 with W[:,0] = logit(s): logits are exactly W[:,0]."""
    L = np.array([math.log(float(s) / (1 - float(s))) for s in s_list], np.float64)
    N = len(L)
    x = np.zeros((1, 4), np.float32)
    x[0, 0] = 1.0
    W = np.zeros((N, 4), np.float32)
    W[:, 0] = L.astype(np.float32)
    return x, W


def _rand_problem(rng, T, d, N_r, bias_scale=0.1):
    x = rng.standard_normal((T, d)).astype(np.float32)
    W = (rng.standard_normal((N_r, d)) / math.sqrt(d)).astype(np.float32)
    b = rng.uniform(-bias_scale, bias_scale, N_r).astype(np.float32)
    return x, W, b


# --------------------------------------------------------------------------
# Hand-derived cases (tests/golden/hand_cases.json)

with open(GOLDEN) as f:
    _G = json.load(f)


@pytest.mark.parametrize("case", _G["router"], ids=[c["name"] for c in _G["router"]])
def test_router_hand_cases(case):
    x, W = _one_hot_logits([_frac(s) for s in case["s"]])
    b = np.array([float(_frac(v)) for v in case["bias"]], np.float32)
    r = oracle.router(x, W, b, case["n_group"], case["topk_group"], case["k"],
                      float(_frac(case["route_scale"])), case["mask_mode"])
    assert r["idx"][0].tolist() == case["expect_idx"]
    np.testing.assert_allclose(r["w"][0], [float(_frac(v)) for v in case["expect_w"]],
                               rtol=2e-6, atol=0)


@pytest.mark.parametrize("case", _G["dispatch"], ids=[c["name"] for c in _G["dispatch"]])
def test_dispatch_hand_cases(case):
    idx = np.array(case["idx"], np.int32)
    counts, offsets, perm, inv = oracle.dispatch(idx, case["N_r"])
    assert counts.tolist() == case["expect_counts"]
    assert offsets.tolist() == case["expect_offsets"]
    assert perm.tolist() == case["expect_perm"]
    assert inv.tolist() == case["expect_inv"]
    assert (perm // idx.shape[1]).tolist() == case["expect_tokens"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", _G["combine"], ids=[c["name"] for c in _G["combine"]])
def test_combine_hand_cases(case, dtype):
    def arr(v):
        return np.array([[float(_frac(e)) for e in row] for row in v], np.float32)

    E, shared = arr(case["E"]), arr(case["shared"])
    if dtype == "bf16":  # every value in the case is exact in bf16
        E = (E.view(np.uint32) >> 16).astype(np.uint16)
        shared = (shared.view(np.uint32) >> 16).astype(np.uint16)
    y, routed = oracle.combine(E, arr(case["w"]), np.array(case["inv"], np.int32),
                               shared, case["k"])
    assert routed.tolist() == arr(case["expect_routed"]).tolist()
    assert y.tolist() == arr(case["expect_y"]).tolist()


# --------------------------------------------------------------------------
# Logits: BLAS (an independent library) on fp64 copies.

def test_logits_match_blas():
    rng = np.random.default_rng(10)
    x, W, b = _rand_problem(rng, 37, 300, 24)
    r = oracle.router(x, W, b, 4, 2, 3, 2.5, 0, want_logits=True)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_allclose(r["logits"], ref, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# Special case: one group and no bias reduces to plain top-k of the scores,
# i.e. of the logits (sigmoid is monotone) -- the unbiased top-K_r form of
# the DeepSeek-V3 "MoE Router" note.

@pytest.mark.parametrize("use_none", [True, False])
def test_unbiased_ungrouped_is_plain_topk(use_none):
    rng = np.random.default_rng(11)
    x, W, _ = _rand_problem(rng, 200, 64, 40)
    b = None if use_none else np.zeros(40, np.float32)
    k = 6
    r = oracle.router(x, W, b, 1, 1, k, 1.0, 0, want_logits=True)
    L = x.astype(np.float64) @ W.astype(np.float64).T
    ref = np.argsort(-L, axis=1, kind="stable")[:, :k]
    assert (r["idx"] == ref).all()
    # renormalised gates: g = s / sum(s) over the K_r survivors (library expit)
    s = expit(np.take_along_axis(L, ref, 1))
    np.testing.assert_allclose(r["w"], s / s.sum(1, keepdims=True), rtol=1e-12)


# --------------------------------------------------------------------------
# Brute force on tiny inputs: the chosen experts maximise the sum of masked
# scores over all k-subsets, where the mask keeps the topk_group groups that
# maximise the sum of group scores, and a group score is the best pair sum
# in the group.  Ties go to the lexicographically smallest index tuple.

def _brute(c, G, Gk, k, mask_mode):
    N = len(c)
    S = N // G
    if G > 1:
        gs = [max(c[g * S + a] + c[g * S + b] for a, b in itertools.combinations(range(S), 2))
              for g in range(G)]
        keep = min(itertools.combinations(range(G), Gk),
                   key=lambda sub: (-math.fsum(gs[g] for g in sub), sub))
        fill = -math.inf if mask_mode == 0 else 0.0
        m = [c[i] if (i // S) in keep else fill for i in range(N)]
    else:
        m = list(c)
    best = min(itertools.combinations(range(N), k),
               key=lambda sub: (-math.fsum(m[i] for i in sub), sub))
    return set(best), m


@pytest.mark.parametrize("N_r,G,Gk,k,mask_mode,bias_lo,bias_hi", [
    (12, 1, 1, 4, 0, -0.1, 0.1),
    (12, 2, 1, 3, 0, -0.1, 0.1),
    (12, 3, 2, 4, 0, -0.1, 0.1),
    (12, 4, 2, 3, 0, -0.1, 0.1),
    (12, 4, 3, 4, 1, -0.1, 0.1),
    (12, 4, 2, 4, 1, -1.5, -0.6),  # zero mask with negative biased scores
    (12, 3, 1, 4, 1, -1.5, -0.6),  # k > group size: masked zeros must fill in
    (8, 4, 2, 2, 0, -0.5, 0.5),
    (10, 5, 2, 4, 0, -0.2, 0.2),
    (9, 3, 3, 2, 0, -0.1, 0.1),
])
def test_router_brute_force(N_r, G, Gk, k, mask_mode, bias_lo, bias_hi):
    rng = np.random.default_rng(1000 + N_r * 100 + G * 10 + Gk + k + mask_mode)
    T = 300
    x, W, _ = _rand_problem(rng, T, 16, N_r)
    b = rng.uniform(bias_lo, bias_hi, N_r).astype(np.float32)
    r = oracle.router(x, W, b, G, Gk, k, 2.5, mask_mode)
    L = x.astype(np.float64) @ W.astype(np.float64).T
    c = expit(L) + b.astype(np.float64)
    for t in range(T):
        want, m = _brute(list(c[t]), G, Gk, k, mask_mode)
        got = r["idx"][t].tolist()
        assert set(got) == want, (t, got, sorted(want))
        # canonical slot order: masked score descending, index ascending
        keys = [(-m[i], i) for i in got]
        assert keys == sorted(keys)


# --------------------------------------------------------------------------
# Invariants the pages state.

def _problem_v3(seed, T=400):
    rng = np.random.default_rng(seed)
    return _rand_problem(rng, T, 96, 64)


def test_weights_sum_to_route_scale():
    x, W, b = _problem_v3(1)
    for scale in (1.0, 2.5, 2.827):
        r = oracle.router(x, W, b, 8, 4, 8, scale, 0)
        np.testing.assert_allclose(r["w"].sum(1), scale, rtol=1e-13)


def test_weights_linear_in_route_scale():
    x, W, b = _problem_v3(2)
    r1 = oracle.router(x, W, b, 8, 4, 8, 1.25, 0)
    r2 = oracle.router(x, W, b, 8, 4, 8, 2.5, 0)
    assert (r1["idx"] == r2["idx"]).all()
    assert (r2["w"] == 2.0 * r1["w"]).all()  # exact: scaling by a power of two


def test_chosen_experts_in_at_most_topk_group_groups():
    # node-limited routing: a token reaches at most topk_group groups
    x, W, b = _problem_v3(3, T=2000)
    for G, Gk in ((8, 4), (8, 1), (4, 2), (16, 3)):
        r = oracle.router(x, W, b, G, Gk, min(8, Gk * (64 // G)), 2.5, 0)
        S = 64 // G
        ngroups = np.array([len(set((r["idx"][t] // S).tolist())) for t in range(len(x))])
        assert ngroups.max() <= Gk


def test_weights_use_unbiased_scores():
    x, W, b = _problem_v3(4)
    L = x.astype(np.float64) @ W.astype(np.float64).T
    s = expit(L)
    # a large bias on a few experts pulls them into the selection ...
    b2 = b.copy()
    b2[[3, 17, 40]] += 5.0
    r = oracle.router(x, W, b2, 1, 1, 8, 2.5, 0)
    assert all({3, 17, 40} <= set(row.tolist()) for row in r["idx"])
    # ... but every weight is still route_scale * s / sum(s) of the unbiased s
    sg = np.take_along_axis(s, r["idx"].astype(np.int64), 1)
    np.testing.assert_allclose(r["w"], 2.5 * sg / sg.sum(1, keepdims=True), rtol=1e-12)


def test_uniform_bias_shift_changes_nothing():
    x, W, b = _problem_v3(5)
    r1 = oracle.router(x, W, b, 8, 4, 8, 2.5, 0)
    r2 = oracle.router(x, W, (b + np.float32(0.25)).astype(np.float32), 8, 4, 8, 2.5, 0)
    ok = ~(oracle.near_tie(r1["margins"], 1e-9))
    assert (r1["idx"][ok] == r2["idx"][ok]).all()
    np.testing.assert_allclose(r1["w"][ok], r2["w"][ok], rtol=1e-15)


def test_permutation_within_groups_is_equivariant():
    x, W, b = _problem_v3(6)
    G, S = 8, 8
    rng = np.random.default_rng(7)
    p = np.concatenate([g * S + rng.permutation(S) for g in range(G)])  # new i <- old p[i]
    r1 = oracle.router(x, W, b, G, 4, 8, 2.5, 0)
    r2 = oracle.router(x, W[p], b[p], G, 4, 8, 2.5, 0)
    ok = ~oracle.order_tie(r1["margins"], 1e-12)
    mapped = p[r2["idx"]]  # back to old expert ids
    assert (mapped[ok] == r1["idx"][ok]).all()
    np.testing.assert_allclose(r2["w"][ok], r1["w"][ok], rtol=1e-14)


def test_margins_are_score_gaps():
    x, W, b = _problem_v3(8, T=50)
    k = 8
    r = oracle.router(x, W, b, 1, 1, k, 2.5, 0)
    c = expit(x.astype(np.float64) @ W.astype(np.float64).T) + b
    srt = -np.sort(-c, axis=1)
    np.testing.assert_allclose(r["margins"][:, 0], srt[:, k - 1] - srt[:, k], atol=1e-14)
    assert np.isinf(r["margins"][:, 1]).all()
    np.testing.assert_allclose(r["margins"][:, 2], np.diff(-srt[:, :k], axis=1).min(1),
                               atol=1e-14)


def test_router_rejects_bad_arguments():
    x, W, b = _problem_v3(9, T=4)
    with pytest.raises(ValueError):
        oracle.router(x, W, b, 7, 2, 4, 2.5, 0)   # 64 % 7 != 0
    with pytest.raises(ValueError):
        oracle.router(x, W, b, 8, 9, 4, 2.5, 0)   # topk_group > n_group
    with pytest.raises(ValueError):
        oracle.router(x, W, b, 8, 1, 9, 2.5, 0)   # k > kept experts under -inf
    with pytest.raises(ValueError):
        oracle.router(x, W, b, 64, 2, 2, 2.5, 0)  # group of one expert


# --------------------------------------------------------------------------
# Dispatch against numpy (bincount, stable argsort).

@pytest.mark.parametrize("skew", [False, True])
def test_dispatch_matches_numpy(skew):
    rng = np.random.default_rng(12)
    T, k, N_r = 3000, 8, 256
    if skew:
        idx = np.where(rng.random((T, k)) < 0.9, rng.integers(0, 32, (T, k)),
                       rng.integers(0, N_r, (T, k))).astype(np.int32)
    else:
        idx = rng.integers(0, N_r, (T, k)).astype(np.int32)
    counts, offsets, perm, inv = oracle.dispatch(idx, N_r)
    flat = idx.reshape(-1)
    assert (counts == np.bincount(flat, minlength=N_r)).all()
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert (np.diff(offsets) == counts).all()
    assert (perm == np.argsort(flat, kind="stable")).all()
    assert (inv[perm] == np.arange(T * k)).all()
    assert (np.diff(flat[perm]) >= 0).all()


def test_dispatch_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[0, 5]], np.int32), 5)
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[0, -1]], np.int32), 5)


# --------------------------------------------------------------------------
# Gather against numpy fancy indexing.

@pytest.mark.parametrize("dt", [np.float32, np.uint16])
def test_gather_matches_fancy_indexing(dt):
    rng = np.random.default_rng(13)
    T, k, d = 50, 4, 33
    x = rng.integers(0, 60000, (T, d)).astype(dt)
    idx = rng.integers(0, 16, (T, k)).astype(np.int32)
    _, _, perm, _ = oracle.dispatch(idx, 16)
    xs = oracle.gather(x, k, perm)
    assert (xs == x[perm // k]).all()
    rows = np.array([0, 7, T * k - 1], np.int32)
    assert (oracle.gather(x, k, perm, rows) == x[perm[rows] // k]).all()


# --------------------------------------------------------------------------
# bf16 rounding against torch's float32 -> bfloat16 cast (round to nearest
# even), and the two ties that decide "to even".

def test_round_bf16_matches_torch():
    import torch
    rng = np.random.default_rng(14)
    v = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000),
                        [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2.0 ** -130,
                         3.3e38, -0.0]]).astype(np.float32)
    got = oracle.round_bf16(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy().astype(np.float64)
    assert np.array_equal(got, ref)
    assert got[-6] == 1.0 and got[-5] == 1 + 2 ** -6


# --------------------------------------------------------------------------
# Combine: closed forms.

def test_combine_identity_experts_gives_route_scale_times_x():
    """Experts = identity (E = gathered x rows), no shared expert:
    y_t = sum_j w_tj x_t = route_scale * x_t since the weights sum to the
    route scale ("Normalize weights" pages)."""
    rng = np.random.default_rng(15)
    x, W, b = _rand_problem(rng, 120, 64, 32)
    r = oracle.router(x, W, b, 4, 2, 4, 2.5, 0)
    w32 = r["w"].astype(np.float32)
    _, _, perm, inv = oracle.dispatch(r["idx"], 32)
    # fp32 rows: exact value of sum_j w_j x = x * sum_j w_j (fp32 weights)
    y, _ = oracle.combine(oracle.gather(x, 4, perm), w32, inv, None, 4)
    np.testing.assert_allclose(y, x.astype(np.float64) * w32.astype(np.float64).sum(1)[:, None],
                               rtol=1e-14, atol=1e-300)
    # bf16 rows: within half a bf16 ulp of the bf16-rounded route_scale * x
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    xbf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    yb, _ = oracle.combine(oracle.gather(xb, 4, perm), w32, inv, None, 4)
    ulp = 2.0 ** (np.floor(np.log2(np.abs(2.5 * xbf) + 1e-300)) - 7)
    assert (np.abs(yb - 2.5 * xbf) <= 0.5 * ulp + 1e-300).all()


def test_combine_scatter_back_direction():
    """One-hot weights pick one slot: y_t = E[inv[t*k + j0]] -- the row the
    scatter-back new_x[idxs] = outs puts at slot (t, j0)."""
    rng = np.random.default_rng(16)
    T, k, N_r = 40, 3, 10
    idx = np.stack([rng.permutation(N_r)[:k] for _ in range(T)]).astype(np.int32)
    _, _, perm, inv = oracle.dispatch(idx, N_r)
    E = np.repeat(np.arange(T * k, dtype=np.float32)[:, None], 2, 1)  # row i holds i
    for j0 in range(k):
        w = np.zeros((T, k), np.float32)
        w[:, j0] = 1.0
        y, _ = oracle.combine(E, w, inv, None, k)
        assert (y[:, 0] == inv.reshape(T, k)[:, j0]).all()
        # and perm is the inverse of inv: the sorted row came from slot t*k+j0
        assert (perm[y[:, 0].astype(np.int64)] == np.arange(T) * k + j0).all()


def test_combine_shared_add_rounds_twice():
    """bf16 rows: routed sum rounded to bf16, then shared added and rounded
    again (the two casts back to the row dtype)."""
    T, k, d = 1, 1, 1
    w = np.array([[1.0]], np.float32)
    inv = np.array([0], np.int32)
    one = np.array([[0x3F80]], np.uint16)                 # 1.0
    tiny = np.array([[0x3B80]], np.uint16)                # 2^-8: half a ulp of 1.0
    y, routed = oracle.combine(one, w, inv, tiny, k)
    assert routed[0, 0] == 1.0 and y[0, 0] == 1.0          # tie -> even (1.0)
    three = np.array([[0x3C40]], np.uint16)               # 3 * 2^-8 = 0.01171875
    y, _ = oracle.combine(one, w, inv, three, k)
    assert y[0, 0] == 1 + 2 ** -6                          # 1 + 1.5 ulp -> up to even


def test_combine_routed_rounding_is_observable():
    """Routed sum exactly halfway (1 + 2^-8) rounds to 1.0 before the shared
    add; adding 2^-8 to the unrounded sum would reach 1 + 2^-7 instead."""
    w = np.array([[1 + 2 ** -8]], np.float32)
    one = np.array([[0x3F80]], np.uint16)                 # 1.0
    tiny = np.array([[0x3B80]], np.uint16)                # 2^-8
    y, routed = oracle.combine(one, w, np.array([0], np.int32), tiny, 1)
    assert routed[0, 0] == 1.0
    assert y[0, 0] == 1.0


# --------------------------------------------------------------------------
# Scoring variants (DeepSeek-V3.2-Exp "Normalize weights" page, Gate.forward):
# softmax scores used as weights without renormalisation, the group's largest
# biased score as its group score, renormalisation without the 1e-20.

def _softmax64(L):
    z = L - L.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def test_softmax_all_experts_gives_scaled_softmax():
    """G = 1, no bias, k = N_r: every expert is chosen and its weight is
    route_scale * softmax(L) (scipy's softmax on BLAS logits), summing to the
    route scale."""
    from scipy.special import softmax
    rng = np.random.default_rng(71)
    x, W, _ = _rand_problem(rng, 64, 48, 12)
    r = oracle.router(x, W, None, 1, 1, 12, 2.5, 0, score="softmax")
    L = x.astype(np.float64) @ W.astype(np.float64).T
    ref = 2.5 * softmax(L, axis=1)
    for t in range(64):
        got = np.zeros(12)
        got[r["idx"][t]] = r["w"][t]
        np.testing.assert_allclose(got, ref[t], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r["w"].sum(1), 2.5, rtol=1e-12)


def test_softmax_weights_are_not_renormalised():
    """k < N_r: the top-k of softmax(L) are the top-k logits (softmax is
    monotone) and their weights are the scaled scores themselves, so they sum
    to less than the route scale."""
    rng = np.random.default_rng(72)
    x, W, _ = _rand_problem(rng, 200, 32, 16)
    r = oracle.router(x, W, None, 1, 1, 4, 2.5, 0, score="softmax")
    L = x.astype(np.float64) @ W.astype(np.float64).T
    p = _softmax64(L)
    want = np.argsort(-L, axis=1, kind="stable")[:, :4]
    assert np.array_equal(r["idx"], want)
    np.testing.assert_allclose(r["w"], 2.5 * np.take_along_axis(p, want, 1), rtol=1e-12)
    assert (r["w"].sum(1) < 2.5 - 1e-6).all()


@pytest.mark.parametrize("group_score", ["top2", "max"])
@pytest.mark.parametrize("score", ["sigmoid", "softmax"])
def test_variants_brute_force(score, group_score):
    """Brute force on tiny inputs for each scoring variant: scores from the
    closed forms (expit / softmax of BLAS logits), group scores as the best
    pair sum or the best single score, then the best k-subset."""
    rng = np.random.default_rng(73 + 2 * (score == "softmax") + (group_score == "max"))
    T, N_r, G, Gk, k = 250, 12, 4, 2, 3
    x, W, _ = _rand_problem(rng, T, 16, N_r)
    b = rng.uniform(-0.05, 0.05, N_r).astype(np.float32)
    r = oracle.router(x, W, b, G, Gk, k, 2.5, 0, score=score, group_score=group_score)
    L = x.astype(np.float64) @ W.astype(np.float64).T
    s = expit(L) if score == "sigmoid" else _softmax64(L)
    c = s + b.astype(np.float64)
    S = N_r // G
    for t in range(T):
        if group_score == "top2":
            want, _ = _brute(list(c[t]), G, Gk, k, 0)
        else:
            gs = [max(c[t, g * S:(g + 1) * S]) for g in range(G)]
            keep = min(itertools.combinations(range(G), Gk),
                       key=lambda sub: (-math.fsum(gs[g] for g in sub), sub))
            m = [c[t, i] if (i // S) in keep else -math.inf for i in range(N_r)]
            want = set(min(itertools.combinations(range(N_r), k),
                           key=lambda sub: (-math.fsum(m[i] for i in sub), sub)))
        assert set(r["idx"][t].tolist()) == want, (t, r["idx"][t], sorted(want))
        sel = s[t, r["idx"][t]]
        w = 2.5 * sel if score == "softmax" else 2.5 * sel / (sel.sum() + 1e-20)
        np.testing.assert_allclose(r["w"][t], w, rtol=1e-12)


def test_group_max_differs_from_top2_sum():
    """A token whose best single score and best pair sum sit in different
    groups: the two group scores keep different groups."""
    # group 0: (0.9, 0.1)  -> max 0.9, pair 1.0; group 1: (0.6, 0.55) -> max 0.6, pair 1.15
    x, W = _one_hot_logits(["0.9", "0.1", "0.6", "0.55"])
    top2 = oracle.router(x, W, None, 2, 1, 1, 1.0, 0)
    amax = oracle.router(x, W, None, 2, 1, 1, 1.0, 0, group_score="max")
    assert top2["idx"][0].tolist() == [2]
    assert amax["idx"][0].tolist() == [0]


def test_renormalisation_epsilon_only_matters_when_scores_underflow():
    """With or without the 1e-20 the weights agree for ordinary scores; when
    every chosen sigmoid score underflows to 0 the epsilon gives 0 weights and
    the plain sum gives 0/0."""
    rng = np.random.default_rng(74)
    x, W, b = _rand_problem(rng, 100, 32, 16)
    a = oracle.router(x, W, b, 4, 2, 4, 2.5, 0)
    n = oracle.router(x, W, b, 4, 2, 4, 2.5, 0, eps=False)
    assert np.array_equal(a["idx"], n["idx"])
    np.testing.assert_allclose(a["w"], n["w"], rtol=1e-15)
    # logits of -1000: exp(1000) overflows, sigmoid is exactly 0
    xz = np.zeros((1, 4), np.float32)
    xz[0, 0] = 1.0
    Wz = np.zeros((8, 4), np.float32)
    Wz[:, 0] = -1000.0
    az = oracle.router(xz, Wz, None, 1, 1, 2, 2.5, 0)
    nz = oracle.router(xz, Wz, None, 1, 1, 2, 2.5, 0, eps=False)
    assert (az["w"] == 0).all()
    assert np.isnan(nz["w"]).all()


# --------------------------------------------------------------------------
# Expert-parallel bookkeeping (Kimi K2 "Add shared output" page, moe_infer,
# ep_size > 1).

def _ep_counts(ep, N_r, seed, zeros=0.3):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 9, size=(ep, N_r)).astype(np.int32)
    c[rng.random((ep, N_r)) < zeros] = 0
    return c


@pytest.mark.parametrize("ep,N_r", [(1, 8), (2, 8), (4, 64), (8, 256), (3, 12)])
def test_ep_splits_are_the_transposed_blocks(ep, N_r):
    """send_splits = block sums of the rank's own counts; recv_counts[s] = the
    block of source s's counts that belongs to this rank (the count
    all-to-all); recv_splits = its row sums; and over all ranks every row
    sent is received once."""
    c = _ep_counts(ep, N_r, ep * 100 + N_r)
    E_loc = N_r // ep
    sent = np.zeros((ep, ep), np.int64)
    for r in range(ep):
        send, rc, recv = oracle.ep_splits(c, r)
        for s in range(ep):
            assert send[s] == c[r, s * E_loc:(s + 1) * E_loc].sum()
            assert np.array_equal(rc[s], c[s, r * E_loc:(r + 1) * E_loc])
            assert recv[s] == rc[s].sum()
            sent[r, s] = send[s]
    for r in range(ep):
        _, _, recv = oracle.ep_splits(c, r)
        assert np.array_equal(recv, sent[:, r])  # what s sends r is what r receives from s


@pytest.mark.parametrize("ep,E_loc", [(1, 4), (2, 32), (4, 16), (8, 32), (5, 3)])
def test_ep_recv_order_is_a_stable_argsort_of_the_labels(ep, E_loc):
    """The receive order against numpy: the page's labels (i % experts_per_rank
    over the (source, expert) segments, built here with numpy.repeat) and
    numpy's stable argsort; the local counts are the column sums."""
    rc = _ep_counts(ep, E_loc, 7 * ep + E_loc)
    order, local = oracle.ep_recv_order(rc)
    labels = np.repeat(np.tile(np.arange(E_loc), ep), rc.reshape(-1))
    assert np.array_equal(order, np.argsort(labels, kind="stable"))
    assert np.array_equal(local, rc.sum(0))


def test_ep_recv_order_hand_case():
    """Two sources, two local experts: source 0 sends 2 rows of expert 0 and 1
    of expert 1, source 1 sends 3 rows of expert 1.  Sorted by expert, keeping
    arrival order: rows 0, 1 (expert 0), then 2, 3, 4, 5 (expert 1)."""
    order, local = oracle.ep_recv_order(np.array([[2, 1], [0, 3]], np.int32))
    assert order.tolist() == [0, 1, 2, 3, 4, 5] and local.tolist() == [2, 4]
    # source 0: expert 1 first is impossible (sorted), but source 1 may send
    # expert 0 rows after source 0's expert 1 rows: they move ahead of them
    order, local = oracle.ep_recv_order(np.array([[1, 2], [2, 1]], np.int32))
    assert order.tolist() == [0, 3, 4, 1, 2, 5] and local.tolist() == [3, 3]


def test_all_to_all_emulation():
    blocks = [[np.array([1]), np.array([2, 3])], [np.array([4, 5]), np.array([], int)]]
    got = oracle.all_to_all(blocks)
    assert got[0].tolist() == [1, 4, 5] and got[1].tolist() == [2, 3]


def test_ep_dest_hand_case():
    """Two ranks, four experts (rank 0 owns 0-1, rank 1 owns 2-3), two tokens
    of two slots each.  Rank 0's slots carry experts 0, 2, 3, 0 and rank 1's
    1, 2, 0, 3.  Owner 0 receives expert 0 from rank 0 (slots 0, 3) and rank 1
    (slot 2), then expert 1 from rank 1 (slot 0); owner 1 receives expert 2
    from rank 0 (slot 1) and rank 1 (slot 1), then expert 3 from rank 0
    (slot 2) and rank 1 (slot 3)."""
    dest, local = oracle.ep_dest([np.array([[0, 2], [3, 0]]), np.array([[1, 2], [0, 3]])], 4)
    assert dest[0].tolist() == [0, 0, 2, 1]
    assert dest[1].tolist() == [3, 1, 2, 3]
    assert local[0].tolist() == [3, 1] and local[1].tolist() == [2, 2]


@pytest.mark.parametrize("ep,N_r,k", [(1, 16, 4), (2, 16, 3), (4, 64, 8), (8, 256, 8),
                                      (3, 12, 2)])
def test_ep_dest_is_the_sorted_rank_of_expert_source_slot(ep, N_r, k):
    """The destination against its plain definition: owner r's buffer lists
    the slots routed to r's experts sorted by (expert, source rank, slot), so
    a slot's row is its rank in that sort, computed here by numpy's lexsort
    over all ranks' slots (ragged batch sizes, one rank with none).  With one
    rank it is the inverse of the expert-sorted permutation."""
    rng = np.random.default_rng(ep * 31 + N_r)
    E_loc = N_r // ep
    Ts = [int(rng.integers(0, 40)) for _ in range(ep)]
    Ts[-1] = 0
    idx_all = [np.stack([rng.choice(N_r, k, replace=False) for _ in range(T)]).astype(np.int32)
               if T else np.zeros((0, k), np.int32) for T in Ts]
    dest, local = oracle.ep_dest(idx_all, N_r)
    g = np.concatenate([i.reshape(-1) for i in idx_all])
    src = np.concatenate([np.full(i.size, s) for s, i in enumerate(idx_all)])
    slot = np.concatenate([np.arange(i.size) for i in idx_all])
    got = np.concatenate(dest)
    for r in range(ep):
        mine = np.nonzero(g // E_loc == r)[0]
        order = mine[np.lexsort((slot[mine], src[mine], g[mine]))]
        want = np.empty(mine.size, np.int64)
        want[np.searchsorted(mine, order)] = np.arange(mine.size)
        assert np.array_equal(got[mine], want)
        assert np.array_equal(local[r], np.bincount(g[mine] - r * E_loc, minlength=E_loc))
    if ep == 1:
        assert np.array_equal(dest[0], oracle.dispatch(idx_all[0], N_r)[3])


# --------------------------------------------------------------------------
# One expert layer over the expert-sorted rows (the grouped GEMM the gather
# feeds), against numpy's matmul on fancy-indexed rows, per expert segment.

@pytest.mark.parametrize("skew", [False, True])
def test_expert_gemm_matches_numpy_per_segment(skew):
    rng = np.random.default_rng(11 + skew)
    T, d, N_r, k, n_out = 37, 48, 8, 3, 20
    if skew:
        idx = np.where(rng.random((T, k)) < 0.8, 2, rng.integers(0, N_r, (T, k)))
    else:
        idx = np.stack([rng.permutation(N_r)[:k] for _ in range(T)])
    counts, offsets, perm, inv = oracle.dispatch(idx.astype(np.int32), N_r)
    x = wl.to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    W = wl.to_bf16_bits(rng.standard_normal((N_r, n_out, d)).astype(np.float32))
    got = oracle.expert_gemm(x, k, perm, offsets, W)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    Wf = wl.bf16_bits_to_f32(W).astype(np.float64)
    for e in range(N_r):
        seg = slice(offsets[e], offsets[e + 1])
        want = xf[perm[seg] // k] @ Wf[e].T
        assert np.allclose(got[seg], want, rtol=1e-12, atol=1e-12), e
    rows = np.array([0, offsets[3], T * k - 1], np.int32)
    assert np.array_equal(oracle.expert_gemm(x, k, perm, offsets, W, rows=rows), got[rows])


def test_expert_gemm_hand_case():
    """Two tokens, two experts, k = 1: token 0 -> expert 1, token 1 -> expert 0.
    Sorted rows: (token 1, expert 0), (token 0, expert 1)."""
    x = wl.to_bf16_bits(np.array([[1.0, 2.0], [3.0, -1.0]], np.float32))
    W = wl.to_bf16_bits(np.array([[[1.0, 0.0]], [[0.5, 0.25]]], np.float32))  # [2,1,2]
    counts, offsets, perm, inv = oracle.dispatch(np.array([[1], [0]], np.int32), 2)
    got = oracle.expert_gemm(x, 1, perm, offsets, W)
    assert got.tolist() == [[3.0], [1.0]]  # 3*1 + -1*0 ; 1*0.5 + 2*0.25
