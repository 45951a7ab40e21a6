"""CPU oracle for the MoE routing hot path (router, dispatch, gather, combine).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product package
(``token_dispatch_fp32_b200``) never imports this module, and this module
never imports the product package; the two share only the seeded input
generators in ``workloads.py``.

The arithmetic lives in ``moe_oracle.c`` (plain C, binary64, sort-based top-k,
one token at a time); this file only builds it with gcc and marshals numpy
arrays.  Each function's docstring names the page passage it follows.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute force, closed forms, library routines, invariants, hand-derived golden
cases); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

NEAR_TIE_EPS = 1e-5


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc, -O2, OpenMP, portable ISA)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        # MO_ORACLE_LIB: test hook used by the mutation test to load a
        # deliberately broken copy of the oracle; never set otherwise.
        path = os.environ.get("MO_ORACLE_LIB") or build()
        lib = C.CDLL(path)
        p = C.c_void_p
        lib.mo_router.argtypes = [p, p, p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                  C.c_int, C.c_double, C.c_int, p, p, p, p, C.c_int]
        lib.mo_router2.argtypes = [p, p, p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                   C.c_int, C.c_double, C.c_int, C.c_int, C.c_int, C.c_int,
                                   p, p, p, p, C.c_int]
        lib.mo_dispatch.argtypes = [p, C.c_int, C.c_int, C.c_int, p, p, p, p]
        lib.mo_expert_gemm.argtypes = [p, C.c_int, C.c_int, C.c_int, p, p, C.c_int, p,
                                       C.c_int, p, C.c_long, p, C.c_int]
        lib.mo_ep_splits.argtypes = [p, C.c_int, C.c_int, C.c_int, p, p, p]
        lib.mo_ep_recv_order.argtypes = [p, C.c_int, C.c_int, p, p]
        lib.mo_gather.argtypes = [p, C.c_long, C.c_int, C.c_int, p, p, C.c_long, p]
        lib.mo_round_bf16.argtypes = [C.c_double]
        lib.mo_round_bf16.restype = C.c_double
        lib.mo_round_bf16_array.argtypes = [p, C.c_long, p]
        lib.mo_combine.argtypes = [p, C.c_int, p, p, p, C.c_int, C.c_int, C.c_int, p,
                                   C.c_long, p, p, C.c_int]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def num_threads() -> int:
    return int(_load().mo_num_threads())


def router(x, W, b, n_group, topk_group, k, route_scale, mask_mode,
           want_logits=False, threads=0, score="sigmoid", group_score="top2",
           eps=True) -> dict:
    """Gate forward for every row of x (Kimi K2 "Normalize weights" page,
    MoEGate.forward; DeepSeek-V3.2-Exp "Normalize weights" page,
    Gate.forward; DeepSeek-V3 "MoE Router" note, "How it works").

    x [T,d] fp32 values, W [N_r,d] fp32, b [N_r] fp32 or None.
    Variants (DeepSeek-V3.2-Exp Gate.forward): score="softmax" (softmax over
    all experts; the weights are the scaled scores, not renormalised),
    group_score="max" (a group's largest biased score instead of its top-2
    sum), eps=False (renormalise by the plain sum).
    Returns idx [T,k] int32 in canonical order (masked biased score
    descending, index ascending), w [T,k] float64, margins [T,3] float64
    (selection, group, slot-order margins) and optionally logits [T,N_r].
    """
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    W = np.ascontiguousarray(W, dtype=np.float32)
    b = None if b is None else np.ascontiguousarray(b, dtype=np.float32)
    T, d = x.shape
    N_r = W.shape[0]
    assert W.shape[1] == d
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    margins = np.empty((T, 3), np.float64)
    logits = np.empty((T, N_r), np.float64) if want_logits else None
    assert score in ("sigmoid", "softmax") and group_score in ("top2", "max")
    rc = lib.mo_router2(_ptr(x), _ptr(W), _ptr(b), T, d, N_r, n_group, topk_group, k,
                        float(route_scale), mask_mode, int(score == "softmax"),
                        int(group_score == "max"), int(bool(eps)), _ptr(idx), _ptr(w),
                        _ptr(logits), _ptr(margins), threads)
    if rc != 0:
        raise ValueError(f"oracle router rejected the arguments (rc={rc})")
    return {"idx": idx, "w": w, "margins": margins, "logits": logits}


def near_tie(margins, eps=NEAR_TIE_EPS):
    """Tokens whose selection (k-th vs k+1-th) or group margin is <= eps."""
    return np.minimum(margins[:, 0], margins[:, 1]) <= eps


def order_tie(margins, eps=NEAR_TIE_EPS):
    """Tokens whose slot order within the top-k is decided by a gap <= eps."""
    return near_tie(margins, eps) | (margins[:, 2] <= eps)


def dispatch(idx, N_r):
    """moe_infer dispatch (Kimi K2 "Add shared output" page, moe_infer:
    tokens_per_expert, idxs = argsort(topk_ids.view(-1)) as a stable sort,
    and the inverse of idxs used by new_x[idxs] = outs).

    Returns counts [N_r], offsets [N_r+1], perm [T*k], inv [T*k] (int32).
    """
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.empty(N_r, np.int32)
    offsets = np.empty(N_r + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    rc = lib.mo_dispatch(_ptr(idx), T, k, N_r, _ptr(counts), _ptr(offsets), _ptr(perm),
                         _ptr(inv))
    if rc != 0:
        raise ValueError(f"oracle dispatch rejected the input (rc={rc})")
    return counts, offsets, perm, inv


def ep_splits(counts_all, r):
    """Expert-parallel bookkeeping of rank r (Kimi K2 "Add shared output"
    page, moe_infer, ep_size > 1: tokens_per_ep_rank, the all_to_all_single
    of tokens_per_expert, output_splits).  counts_all [ep, N_r]: every rank's
    tokens_per_expert; rank r owns experts [r*E_loc, (r+1)*E_loc).
    Returns send_splits [ep], recv_counts [ep, E_loc], recv_splits [ep]."""
    counts_all = np.ascontiguousarray(counts_all, dtype=np.int32)
    ep, N_r = counts_all.shape
    E_loc = N_r // ep
    send = np.empty(ep, np.int32)
    recv_counts = np.empty((ep, E_loc), np.int32)
    recv = np.empty(ep, np.int32)
    if _load().mo_ep_splits(_ptr(counts_all), ep, N_r, r, _ptr(send), _ptr(recv_counts),
                            _ptr(recv)) != 0:
        raise ValueError("oracle ep_splits rejected the arguments")
    return send, recv_counts, recv


def ep_recv_order(recv_counts):
    """Order of the received rows by local expert (the page's gatherd_idxs
    labels and their argsort, taken stable).  recv_counts [ep, E_loc].
    Returns order [R] (sorted_tokens = gathered_tokens[order]) and
    local_counts [E_loc] (tokens_per_expert_post_gather)."""
    recv_counts = np.ascontiguousarray(recv_counts, dtype=np.int32)
    ep, E_loc = recv_counts.shape
    order = np.empty(int(recv_counts.sum()), np.int32)
    local = np.empty(E_loc, np.int32)
    if _load().mo_ep_recv_order(_ptr(recv_counts), ep, E_loc, _ptr(order), _ptr(local)) != 0:
        raise ValueError("oracle ep_recv_order rejected the arguments")
    return order, local


def all_to_all(send_blocks):
    """The all-to-all exchange itself, for ranks emulated in one process:
    send_blocks[s][r] is what rank s sends rank r; rank r receives the
    concatenation over s, in source order (dist.all_to_all)."""
    ep = len(send_blocks)
    return [np.concatenate([send_blocks[s][r] for s in range(ep)], axis=0) for r in range(ep)]


def ep_dest(idx_all, N_r):
    """Where each routed row of each rank lands in its owner's receive buffer
    once the page's exchange has run (Kimi K2 "Add shared output" page,
    moe_infer, ep_size > 1): every rank sorts its slots by expert (stable),
    sends owner r the block of r's experts, the owner concatenates what it
    receives in source order and sorts it by local expert (the stable argsort
    of the received labels).  Here the exchange carries slot labels (source,
    slot) instead of rows, so the position of a label in the owner's final
    order is the row the slot's data takes there.

    idx_all: list of ep [T_s, k] expert-id arrays (ids in [0, N_r)).
    Returns (dest, local): dest[s] [T_s*k] int32 (row in the owner's buffer),
    local[r] [E_loc] int32 (rows per local expert of owner r).
    """
    ep = len(idx_all)
    if N_r % ep:
        raise ValueError(f"{N_r} experts do not split over {ep} ranks")
    per = [dispatch(np.asarray(i, np.int32), N_r) for i in idx_all]
    counts_all = np.stack([c for c, _, _, _ in per])
    send_blocks = []
    for s, (_, offsets, perm, _) in enumerate(per):
        labels = np.stack([np.full(int(offsets[-1]), s, np.int64),
                           perm[:int(offsets[-1])].astype(np.int64)], axis=1)
        send, _, _ = ep_splits(counts_all, s)
        bounds = np.concatenate([[0], np.cumsum(send)])
        send_blocks.append([labels[bounds[r]:bounds[r + 1]] for r in range(ep)])
    received = all_to_all(send_blocks)
    dest = [np.full(np.asarray(i).size, -1, np.int32) for i in idx_all]
    local = []
    for r in range(ep):
        _, recv_counts, _ = ep_splits(counts_all, r)
        order, local_r = ep_recv_order(recv_counts)
        final = received[r][order]
        for pos, (s, slot) in enumerate(final):
            dest[s][slot] = pos
        local.append(local_r)
    return dest, local


def expert_gemm(x_bits, k, perm, offsets, W_bits, rows=None, threads=0):
    """One expert layer over the expert-sorted rows (Kimi K2 "Add shared
    output" page, moe_infer: expert(sorted_tokens[start_idx:end_idx]) for
    each expert), the expert a linear map with synthetic weights:
    out[j] = x[perm[j] // k] . W[e(j)]^T in binary64, e(j) the expert whose
    segment [offsets[e], offsets[e+1]) holds sorted row j.  x_bits [T,d] and
    W_bits [N_r, n_out, d] are bf16 bit patterns (uint16); rows selects
    sorted rows (all when None).  Returns float64 [n_rows, n_out]."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    T, d = x_bits.shape
    N_r, n_out, dw = W_bits.shape
    assert dw == d and offsets.shape == (N_r + 1,)
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n = int(offsets[-1]) if rows is None else rows_a.shape[0]
    out = np.empty((n, n_out), np.float64)
    rc = _load().mo_expert_gemm(_ptr(x_bits), T, d, k, _ptr(perm), _ptr(offsets), N_r,
                                _ptr(W_bits), n_out, _ptr(rows_a), n, _ptr(out), threads)
    if rc != 0:
        raise ValueError(f"oracle expert_gemm: index out of range (rc={rc})")
    return out


def gather(x, k, perm, rows=None):
    """sorted_tokens = x[idxs // k] (Kimi K2 "Add shared output" page,
    moe_infer).  x is [T,d] of any element type, copied byte for byte;
    rows selects a subset of output rows (all rows when None)."""
    lib = _load()
    x = np.ascontiguousarray(x)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    T = x.shape[0]
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n = perm.shape[0] if rows is None else rows_a.shape[0]
    out = np.empty((n,) + x.shape[1:], x.dtype)
    row_bytes = x.dtype.itemsize * int(np.prod(x.shape[1:]))  # numpy gives an empty array stride 0
    rc = lib.mo_gather(_ptr(x), row_bytes, T, k, _ptr(perm), _ptr(rows_a), n, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle gather: index out of range (rc={rc})")
    return out


def round_bf16(a):
    """binary64 -> nearest-even bf16 value (returned as binary64)."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty_like(a)
    _load().mo_round_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


def combine(E, w, inv, shared, k, tokens=None, threads=0):
    """Weighted combine and shared add (Kimi K2 "Add shared output" page:
    moe_infer scatter-back and weighted sum, DeepseekV3MoE.forward shared
    add, formula Delta_ffn = y_routed + y_shared).

    E [T*k,d] expert outputs in expert-sorted order, fp32 or bf16 bits
    (uint16); w [T,k] fp32; inv [T*k] int32; shared [T,d] same dtype as E,
    or None.  Returns (y, routed) as float64 [n_tok,d], already rounded to
    the row dtype for bf16.
    """
    lib = _load()
    E = np.ascontiguousarray(E)
    dtype = 1 if E.dtype == np.uint16 else 0
    assert E.dtype in (np.uint16, np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    inv = np.ascontiguousarray(inv, dtype=np.int32)
    T, kk = w.shape
    assert kk == k
    d = E.shape[1]
    if shared is not None:
        shared = np.ascontiguousarray(shared)
        assert shared.dtype == E.dtype and shared.shape == (T, d)
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = T if tokens is None else tok.shape[0]
    y = np.empty((n, d), np.float64)
    routed = np.empty((n, d), np.float64)
    rc = lib.mo_combine(_ptr(E), dtype, _ptr(w), _ptr(inv), _ptr(shared), T, d, k,
                        _ptr(tok), n, _ptr(y), _ptr(routed), threads)
    if rc != 0:
        raise ValueError(f"oracle combine rejected the input (rc={rc})")
    return y, routed
