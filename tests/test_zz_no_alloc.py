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
        for _ in range(2):              # two calls in a row share the scratch
            got = mr.mr_dispatch_noalloc(idx, N_r, *_outs(T, k, N_r))
            assert mr.mr_get_error() == mr.MR_OK
            for g, r in zip(got, ref):
                assert torch.equal(g, r)


@pytest.mark.gpu
def test_noalloc_dispatch_rejects_sizes_beyond_its_scratch():
    cap = mr.mr_dispatch_noalloc_max_workspace()
    assert cap == 1 << 20
    T, k, N_r = 300000, 8, 256  # needs ceil(2.4M / 1024) * 256 * 4 bytes > 1 MiB
    assert mr.mr_dispatch_workspace_size(T, k, N_r) > cap
    p = C.c_void_p(16)  # rejected before any launch: never dereferenced
    st = mr.lib().mr_dispatch_noalloc(p, T, k, N_r, p, p, p, p, None)
    assert st == mr.MR_ERR_UNSUPPORTED
