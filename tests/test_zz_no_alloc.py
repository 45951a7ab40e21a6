"""mr_dispatch_noalloc: the dispatch entry point for callers that cannot
allocate device memory at dispatch time (e.g. a serving loop with a memory
plan fixed before requests start, or a plug-in inside another framework's
runtime that is handed only tensors and a stream).  It must give exactly what
mr_dispatch gives with a caller-provided workspace, call after call, even
though every call reuses the same scratch array inside the library.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr


def _ids(T, k, N_r, seed, skew=False):
    rng = np.random.default_rng(seed)
    if skew:
        a = np.where(rng.random((T, k)) < 0.9, rng.integers(0, 32, (T, k)),
                     rng.integers(0, N_r, (T, k)))
    else:
        a = np.stack([rng.permutation(N_r)[:k] for _ in range(T)])
    return torch.from_numpy(a.astype(np.int32)).cuda()


def _outs(T, k, N_r):
    z = lambda n: torch.full((n,), -7, dtype=torch.int32, device="cuda")  # noqa: E731
    return z(N_r), z(N_r + 1), z(T * k), z(T * k)


@pytest.mark.gpu
def test_noalloc_dispatch_matches_workspace_dispatch_twice_in_a_row():
    cases = [(16384, 8, 256, 1, True), (3000, 6, 384, 2, False)]
    for T, k, N_r, seed, skew in cases:
        idx = _ids(T, k, N_r, seed, skew)
        ref = mr.mr_dispatch(idx, N_r)  # existing entry point, caller workspace
        # and the oracle's stable counting sort of the same ids
        orc = oracle.dispatch(idx.cpu().numpy(), N_r)
        for _ in range(2):              # two calls in a row share the scratch
            got = mr.mr_dispatch_noalloc(idx, N_r, *_outs(T, k, N_r))
            assert mr.mr_get_error() == mr.MR_OK
            for g, r, o in zip(got, ref, orc):
                assert torch.equal(g, r)
                assert np.array_equal(g.cpu().numpy(), o)


@pytest.mark.gpu
def test_noalloc_dispatch_drops_out_of_range_ids_like_mr_dispatch():
    """Ids outside [0, N_r) are dropped by both entry points alike: the valid
    entries are sorted, the dropped slots' inverse entries and the tail of
    perm read -1, and the device flag reports it."""
    T, k, N_r = 500, 4, 64
    a = _ids(T, k, N_r, 3).cpu().numpy()
    a[7, 2], a[123, 0], a[499, 3] = -1, N_r, N_r + 5
    idx = torch.from_numpy(a).cuda()
    ref = mr.mr_dispatch(idx, N_r)
    assert mr.mr_get_error() == mr.MR_ERR_DEVICE
    for _ in range(2):
        got = mr.mr_dispatch_noalloc(idx, N_r, *_outs(T, k, N_r))
        assert mr.mr_get_error() == mr.MR_ERR_DEVICE
        for g, r in zip(got, ref):
            assert torch.equal(g, r)
    counts, offsets, perm, inv = (t.cpu().numpy() for t in got)
    assert counts.sum() == T * k - 3 and offsets[-1] == T * k - 3
    assert (perm[T * k - 3:] == -1).all()
    assert inv[7 * k + 2] == -1 and inv[123 * k] == -1 and inv[499 * k + 3] == -1


@pytest.mark.gpu
def test_noalloc_dispatch_rejects_sizes_beyond_its_scratch():
    cap = mr.mr_dispatch_noalloc_max_workspace()
    assert cap == 1 << 20
    T, k, N_r = 300000, 8, 256  # needs ceil(2.4M / 1024) * 256 * 4 bytes > 1 MiB
    assert mr.mr_dispatch_workspace_size(T, k, N_r) > cap
    p = C.c_void_p(16)  # rejected before any launch: never dereferenced
    st = mr.lib().mr_dispatch_noalloc(p, T, k, N_r, p, p, p, p, None)
    assert st == mr.MR_ERR_UNSUPPORTED
