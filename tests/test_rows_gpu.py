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
    (50, 1000, 4, 16, "bf16"),    # 2000-byte rows: 16-byte vectors, not 32
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


def _offset_view(a, off_bytes):
    """A device copy of `a` whose first element sits `off_bytes` past a
    32-byte boundary (torch's allocations start on 512-byte boundaries)."""
    t = _dev(a)
    n = t.numel()
    esz = t.element_size()
    buf = torch.empty(n + 64 // esz, dtype=t.dtype, device="cuda")
    v = buf[off_bytes // esz: off_bytes // esz + n].view(t.shape)
    v.copy_(t)
    assert v.data_ptr() % 32 == off_bytes % 32
    return v


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rows_on_16_byte_offsets(dtype):
    """Buffers that start 16 bytes past a 32-byte boundary take the 16-byte
    vector kernels; gather stays bit-exact and combine matches the oracle and,
    bit for bit, the same data on 32-byte aligned buffers (both widths add the
    slots in the same order)."""
    T, d, k, N_r = 333, 7168, 8, 256
    idx, w, E, sh, x = _problem(T, d, k, N_r, dtype, seed=21)
    _, _, perm, inv = oracle.dispatch(idx, N_r)
    inv_d, perm_d = torch.from_numpy(inv).cuda(), torch.from_numpy(perm).cuda()
    w_d = torch.from_numpy(w).cuda()
    ys = []
    for off in (0, 16):
        xs = _offset_view(np.zeros((T * k, d), x.dtype), off)
        mr.mr_gather_rows(_offset_view(x, off), k, perm=perm_d, inv_perm=inv_d, xs=xs)
        assert mr.mr_get_error() == mr.MR_OK
        assert np.array_equal(_host(xs), oracle.gather(x, k, perm))
        y = _offset_view(np.zeros((T, d), E.dtype), off)
        mr.mr_combine(_offset_view(E, off), w_d, inv_d, _offset_view(sh, off), y=y)
        assert mr.mr_get_error() == mr.MR_OK
        ys.append(_host(y))
    assert np.array_equal(ys[0].view(np.uint8), ys[1].view(np.uint8))
    ry, rr = oracle.combine(E, w, inv, sh, k)
    compare_combine(widen(ys[1]), ry, rr, widen(sh), bf16=dtype == "bf16")


@pytest.mark.parametrize("d,dtype,k", [(7168, "bf16", 8), (512, "f32", 4), (1001, "bf16", 3),
                                       (64, "bf16", 20)])
def test_combine_skips_dropped_slots(d, dtype, k):
    """A slot whose inverse entry is -1 (an assignment dispatch dropped)
    contributes nothing: the result is the oracle's with that slot's weight
    set to zero (fma(0, e, acc) = acc for finite e)."""
    T, N_r = 600, 32
    idx, w, E, sh, _ = _problem(T, d, k, N_r, dtype, seed=13)
    _, _, perm, inv = oracle.dispatch(idx, N_r)
    rng = np.random.default_rng(6)
    drop = rng.random(T * k) < 0.15
    drop[:k] = True  # one token with every slot dropped
    inv_d = np.where(drop, -1, inv).astype(np.int32)
    y = mr.mr_combine(_dev(E), torch.from_numpy(w).cuda(), torch.from_numpy(inv_d).cuda(),
                      _dev(sh))
    assert mr.mr_get_error() == mr.MR_OK
    w0 = np.where(drop.reshape(T, k), np.float32(0), w).astype(np.float32)
    ry, rr = oracle.combine(E, w0, inv, sh, k)
    compare_combine(widen(_host(y)), ry, rr, widen(sh), bf16=dtype == "bf16")
    # the token with no slot left is its shared row (bf16: bf16(0 + s) = s)
    assert np.array_equal(_host(y)[0].view(np.uint8), sh[0].view(np.uint8))
