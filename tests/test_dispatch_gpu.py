"""Dispatch parity on the GPU: counts, offsets, perm and inv_perm bit-exact
against the oracle (stable argsort reading of idxs = argsort(topk_ids)), for
the one-launch cooperative kernel and, beyond what fits at once, the
three-kernel counting sort."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr

pytestmark = pytest.mark.gpu


def _gpu(idx, N_r, want_inv=True):
    counts, offsets, perm, inv = mr.mr_dispatch(torch.from_numpy(idx).cuda(), N_r,
                                                want_inv=want_inv)
    st = mr.mr_get_error()
    out = [t.cpu().numpy() if t is not None else None for t in (counts, offsets, perm, inv)]
    return out, st


def _idx(kind, T, k, N_r, seed):
    rng = np.random.default_rng(seed)
    if kind == "uniform_distinct":
        return np.stack([rng.permutation(N_r)[:k] for _ in range(T)]).astype(np.int32)
    if kind == "uniform":
        return rng.integers(0, N_r, (T, k)).astype(np.int32)
    if kind == "skewed":  # 90% of picks land on 32 hot experts
        return np.where(rng.random((T, k)) < 0.9, rng.integers(0, 32, (T, k)),
                        rng.integers(0, N_r, (T, k))).astype(np.int32)
    if kind == "one_expert":
        return np.full((T, k), N_r - 1, np.int32)
    raise ValueError(kind)


CASES = [
    ("uniform_distinct", 16384, 8, 256),   # the full-size shape
    ("skewed", 16384, 8, 256),
    ("uniform", 8192, 8, 384),
    ("uniform", 1, 8, 256),
    ("uniform", 513, 3, 17),                # ragged chunk tail, odd sizes
    ("uniform", 5000, 32, 1024),            # largest k and N_r
    ("one_expert", 3000, 4, 64),            # every entry in one segment
    ("uniform", 64, 1, 1),
    ("skewed", 200000, 8, 256),             # more chunks than fit at once: three kernels
]


@pytest.mark.parametrize("kind,T,k,N_r", CASES)
def test_dispatch_bit_exact(kind, T, k, N_r):
    idx = _idx(kind, T, k, N_r, seed=T + k + N_r)
    (counts, offsets, perm, inv), st = _gpu(idx, N_r)
    assert st == mr.MR_OK
    rc, ro, rp, ri = oracle.dispatch(idx, N_r)
    assert (counts == rc).all()
    assert (offsets == ro).all()
    assert (perm == rp).all()
    assert (inv == ri).all()


def test_dispatch_without_inverse():
    idx = _idx("skewed", 2000, 8, 256, 3)
    (counts, offsets, perm, inv), st = _gpu(idx, 256, want_inv=False)
    assert st == mr.MR_OK and inv is None
    assert (perm == oracle.dispatch(idx, 256)[2]).all()


def test_dispatch_empty():
    counts, offsets, perm, inv = mr.mr_dispatch(torch.zeros((0, 8), dtype=torch.int32,
                                                            device="cuda"), 16)
    assert counts.cpu().numpy().sum() == 0 and (offsets.cpu().numpy() == 0).all()


def test_dispatch_bad_ids_raise_device_flag_and_are_dropped():
    """Out-of-range ids are injected from the host; the kernel skips them,
    raises the device flag and keeps the valid entries' dispatch exact."""
    idx = _idx("uniform", 1000, 8, 64, 9)
    idx[3, 2] = 64
    idx[500, 0] = -5
    (counts, offsets, perm, inv), st = _gpu(idx, 64)
    assert st == mr.MR_ERR_DEVICE
    assert mr.mr_get_error() == mr.MR_OK  # flag was cleared
    flat = idx.reshape(-1)
    valid = (flat >= 0) & (flat < 64)
    assert (counts == np.bincount(flat[valid], minlength=64)).all()
    n_valid = valid.sum()
    slots = np.nonzero(valid)[0]
    assert (perm[:n_valid] == slots[np.argsort(flat[valid], kind="stable")]).all()
    assert (perm[n_valid:] == -1).all()
    assert (inv[~valid] == -1).all()
    assert (inv[perm[:n_valid]] == np.arange(n_valid)).all()
