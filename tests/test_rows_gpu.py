"""Gather (bit-exact) and combine (tolerance) parity on the GPU."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_fp32_b200 as mr
from parity import compare_combine, widen

pytestmark = pytest.mark.gpu


def _problem(T, d, k, N_r, dtype, seed, with_shared=True):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(N_r)[:k] for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.05, 1.0, (T, k)).astype(np.float32)
    w = (w / w.sum(1, keepdims=True) * np.float32(2.5)).astype(np.float32)
    z = rng.standard_normal((T * k, d)).astype(np.float32)
    sh = rng.standard_normal((T, d)).astype(np.float32) if with_shared else None
    x = rng.standard_normal((T, d)).astype(np.float32)
    if dtype == "bf16":
        to = lambda a: None if a is None else (a.view(np.uint32) >> 16).astype(np.uint16)  # noqa
        z, sh, x = to(z), to(sh), to(x)
    return idx, w, z, sh, x


def _dev(a):
    t = torch.from_numpy(a)
    return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).cuda()


def _host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


ROW_CASES = [  # T, d, k, N_r, dtype
    (300, 7168, 8, 256, "bf16"),
    (257, 512, 4, 64, "f32"),
    (100, 1001, 3, 40, "bf16"),   # odd row: element path
    (64, 37, 2, 8, "f32"),        # ragged fp32 row
    (1, 8, 1, 1, "bf16"),
    (128, 64, 32, 64, "bf16"),    # k = 32
    (2000, 7168, 8, 256, "bf16"),  # several tokens per CTA: the row ring wraps
    (1500, 4096, 6, 64, "f32"),
]


@pytest.mark.parametrize("T,d,k,N_r,dtype", ROW_CASES)
@pytest.mark.parametrize("use_inv", [True, False], ids=["inv", "perm"])
def test_gather_bit_exact(T, d, k, N_r, dtype, use_inv):
    idx, _, _, _, x = _problem(T, d, k, N_r, dtype, seed=T * 7 + d)
    _, _, perm, inv = oracle.dispatch(idx, N_r)
    xs = mr.mr_gather_rows(_dev(x), k, perm=torch.from_numpy(perm).cuda(),
                           inv_perm=torch.from_numpy(inv).cuda() if use_inv else None)
    assert mr.mr_get_error() == mr.MR_OK
    assert np.array_equal(_host(xs), oracle.gather(x, k, perm))


@pytest.mark.parametrize("T,d,k,N_r,dtype", ROW_CASES)
@pytest.mark.parametrize("with_shared", [True, False], ids=["shared", "noshared"])
def test_combine_matches_oracle(T, d, k, N_r, dtype, with_shared):
    idx, w, E, sh, _ = _problem(T, d, k, N_r, dtype, seed=T * 11 + d, with_shared=with_shared)
    _, _, perm, inv = oracle.dispatch(idx, N_r)
    y = mr.mr_combine(_dev(E), torch.from_numpy(w).cuda(), torch.from_numpy(inv).cuda(),
                      None if sh is None else _dev(sh))
    assert mr.mr_get_error() == mr.MR_OK
    ry, rr = oracle.combine(E, w, inv, sh, k)
    stats = compare_combine(widen(_host(y)), ry, rr, None if sh is None else widen(sh),
                            bf16=dtype == "bf16")
    print(T, d, k, dtype, with_shared, stats)


@pytest.mark.parametrize("d,dtype", [(7168, "bf16"), (512, "f32"), (1001, "bf16")])
def test_gather_skips_dropped_slots(d, dtype):
    """Slots whose inverse entry is -1 (assignments dispatch dropped) write
    nothing: their sorted rows keep what was there, every other row is the
    token's row."""
    T, k, N_r = 700, 4, 32
    idx, _, _, _, x = _problem(T, d, k, N_r, dtype, seed=11)
    _, _, perm, inv = oracle.dispatch(idx, N_r)
    rng = np.random.default_rng(5)
    drop = rng.random(T * k) < 0.1
    inv_d = np.where(drop, -1, inv).astype(np.int32)
    poison = np.full((T * k, d), 0x7FC1 if dtype == "bf16" else np.nan,
                     dtype=np.uint16 if dtype == "bf16" else np.float32)
    xs = _dev(poison.copy())
    mr.mr_gather_rows(_dev(x), k, perm=torch.from_numpy(perm).cuda(),
                      inv_perm=torch.from_numpy(inv_d).cuda(), xs=xs)
    assert mr.mr_get_error() == mr.MR_OK
    got = _host(xs)
    want = oracle.gather(x, k, perm)
    kept_rows = np.sort(inv[~drop])
    dropped_rows = np.sort(inv[drop])
    assert np.array_equal(got[kept_rows], want[kept_rows])
    assert np.array_equal(got[dropped_rows].view(np.uint8), poison[dropped_rows].view(np.uint8))
