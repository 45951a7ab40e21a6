"""libmr.so loads, exports every entry point include/mr.h declares, and its
host-side argument validation rejects bad calls before touching the GPU
(these run without a GPU: validation returns before any CUDA call)."""
import ctypes as C
import os
import re
import shutil
import subprocess

import pytest

import token_dispatch_fp32_b200 as mr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mr.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mr_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for fn in ("mr_router_forward", "mr_dispatch", "mr_gather_rows", "mr_combine"):
        assert fn in names


def test_library_exports_every_declared_symbol():
    lib = mr.lib()
    for fn in declared_functions():
        assert hasattr(lib, fn), fn


def test_library_has_no_oracle_dependency():
    """The product library neither links the oracle nor carries its entry
    points (ELF dynamic section and exported symbols)."""
    lib = mr.lib()
    for sym in ("mo_router", "mo_router2", "mo_dispatch", "mo_gather", "mo_combine"):
        assert not hasattr(lib, sym), sym
    readelf = shutil.which("readelf")
    if readelf is None:
        pytest.skip("readelf not available")
    dyn = subprocess.run([readelf, "-d", mr._binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    needed = re.findall(r"\(NEEDED\)\s+Shared library: \[([^\]]+)\]", dyn)
    assert needed and not any("oracle" in n for n in needed), needed


def header_parameter_counts():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for name, args in re.findall(r"\b(mr_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
        args = " ".join(args.split())
        out[name] = 0 if args in ("", "void") else len(args.split(","))
    return out


def test_binding_marshals_the_declared_arguments():
    """Each ctypes prototype of the binding has as many arguments as the
    header's declaration (an ABI drift would pass garbage, not fail)."""
    lib = mr.lib()
    counts = header_parameter_counts()
    assert set(counts) == set(declared_functions())
    for name, n in counts.items():
        argtypes = getattr(lib, name).argtypes
        if argtypes is None:
            assert n == 0, f"{name}: {n} parameters declared, no prototype in the binding"
        else:
            assert len(argtypes) == n, f"{name}: header {n}, binding {len(argtypes)}"


def test_version_and_status_strings():
    assert mr.version() >= 100
    assert mr.status_string(mr.MR_OK) == "ok"
    assert "invalid" in mr.status_string(mr.MR_ERR_INVALID_ARG)


NULL = None


def router(T=8, d=64, N_r=64, G=8, Gk=4, k=8, scale=2.5, mask=0, x=1, W=1, idx=1, w=1):
    p = lambda v: C.c_void_p(16) if v else None  # noqa: E731  (never dereferenced)
    return mr.lib().mr_router_forward(p(x), p(W), None, T, d, N_r, G, Gk, k, scale, mask,
                                      p(idx), p(w), None)


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), mr.MR_ERR_INVALID_ARG),
    (dict(d=0), mr.MR_ERR_INVALID_ARG),
    (dict(G=7), mr.MR_ERR_INVALID_ARG),           # N_r % n_group != 0
    (dict(Gk=9), mr.MR_ERR_INVALID_ARG),          # topk_group > n_group
    (dict(Gk=0), mr.MR_ERR_INVALID_ARG),
    (dict(k=0), mr.MR_ERR_INVALID_ARG),
    (dict(G=32, Gk=1, k=3), mr.MR_ERR_INVALID_ARG),  # -inf mask: k > kept experts
    (dict(N_r=64, G=64, Gk=2, k=2), mr.MR_ERR_INVALID_ARG),  # group of one expert
    (dict(mask=2), mr.MR_ERR_INVALID_ARG),
    (dict(scale=float("nan")), mr.MR_ERR_INVALID_ARG),
    (dict(x=0), mr.MR_ERR_INVALID_ARG),
    (dict(idx=0), mr.MR_ERR_INVALID_ARG),
    (dict(k=9, G=1, Gk=1), mr.MR_ERR_UNSUPPORTED),  # k > 8
    (dict(N_r=1024, G=1, Gk=1), mr.MR_ERR_UNSUPPORTED),
    (dict(T=0, x=0, W=0, idx=0, w=0), mr.MR_OK),  # empty batch: nothing to do
])
def test_router_validation(kw, status):
    assert router(**kw) == status


def test_router_ex_validation():
    L = mr.lib()
    p = C.c_void_p(16)
    # bad dtype / precision codes
    assert L.mr_router_forward_ex(p, 7, p, None, 4, 64, 64, 8, 4, 8, 2.5, 0, 0, p, p, None,
                                  None, 0, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_router_forward_ex(p, 0, p, None, 4, 64, 64, 8, 4, 8, 2.5, 0, 9, p, p, None,
                                  None, 0, None) == mr.MR_ERR_INVALID_ARG


def test_router_ex2_rejects_unknown_flags():
    L = mr.lib()
    p = C.c_void_p(16)
    for flags in (8, 16, -1):
        assert L.mr_router_forward_ex2(p, 0, p, None, 4, 64, 64, 8, 4, 8, 2.5, 0, 0, flags, p, p,
                                       None, None, 0, None) == mr.MR_ERR_INVALID_ARG
    # the known flags pass flag validation and then fail on the bad dtype
    assert L.mr_router_forward_ex2(p, 7, p, None, 4, 64, 64, 8, 4, 8, 2.5, 0, 0, 7, p, p,
                                   None, None, 0, None) == mr.MR_ERR_INVALID_ARG


def test_dispatch_validation():
    L = mr.lib()
    p = C.c_void_p(16)
    ws = L.mr_dispatch_workspace_size(100, 8, 256)
    assert ws == 16 + 4 * 256 + 4 * 256  # barrier word, one chunk of 1024 entries, totals
    assert L.mr_dispatch(p, 100, 0, 256, p, p, p, p, p, ws, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_dispatch(p, 100, 8, 0, p, p, p, p, p, ws, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_dispatch(p, 100, 8, 256, p, p, p, p, p, ws - 1, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_dispatch(p, 100, 8, 256, p, p, p, p, None, ws, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_dispatch(p, 100, 33, 256, p, p, p, p, p, 1 << 20, None) == mr.MR_ERR_UNSUPPORTED
    assert L.mr_dispatch(p, 100, 8, 2048, p, p, p, p, p, 1 << 20, None) == mr.MR_ERR_UNSUPPORTED
    assert L.mr_dispatch(p, 1 << 28, 8, 256, p, p, p, p, p, 1 << 40, None) == mr.MR_ERR_INVALID_ARG


def test_rows_validation():
    L = mr.lib()
    p = C.c_void_p(16)
    assert L.mr_gather_rows(p, 5, 10, 64, 8, p, p, p, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_gather_rows(p, 1, 10, 64, 8, None, None, p, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_gather_rows(p, 1, 10, 64, 40, p, p, p, None) == mr.MR_ERR_UNSUPPORTED
    assert L.mr_gather_rows(None, 1, 0, 64, 8, None, None, None, None) == mr.MR_OK
    assert L.mr_combine(p, 1, None, p, None, p, 10, 64, 8, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_combine(p, 1, p, p, None, p, 10, 0, 8, None) == mr.MR_ERR_INVALID_ARG
    assert L.mr_combine(None, 1, None, None, None, None, 0, 64, 8, None) == mr.MR_OK


def test_expert_layer_validation():
    """Argument checks of the expert-layer entry points that return before
    any device call (so they hold on a machine without a GPU)."""
    L = mr.lib()
    p = C.c_void_p(64)
    # mr_expert_gemm_gather(x, perm, offsets, W, T, d, k, N_r, n_out, out)
    assert L.mr_expert_gemm_gather(p, p, p, p, -1, 64, 8, 16, 32, p, None) == \
        mr.MR_ERR_INVALID_ARG
    assert L.mr_expert_gemm_gather(None, p, p, p, 10, 64, 8, 16, 32, p, None) == \
        mr.MR_ERR_INVALID_ARG
    assert L.mr_expert_gemm_gather(p, p, p, p, 0, 64, 8, 16, 32, p, None) == mr.MR_OK
    # mr_expert_gemm_gather_combine(x, perm, offsets, W, w_packed, w, shared,
    #                               T, d, k, N_r, n_out, acc, y)
    comb = L.mr_expert_gemm_gather_combine
    assert comb(p, p, p, p, 0, p, None, -1, 64, 8, 16, 32, p, p, None) == mr.MR_ERR_INVALID_ARG
    assert comb(p, p, p, p, 2, p, None, 10, 64, 8, 16, 32, p, p, None) == mr.MR_ERR_INVALID_ARG
    assert comb(p, None, p, p, 0, p, None, 10, 64, 8, 16, 32, p, p, None) == \
        mr.MR_ERR_INVALID_ARG  # perm is required: it gives each row's slot
    assert comb(p, p, p, p, 0, None, None, 10, 64, 8, 16, 32, p, p, None) == \
        mr.MR_ERR_INVALID_ARG  # no router weights
    assert comb(p, p, p, p, 0, p, None, 10, 64, 8, 16, 32, None, p, None) == \
        mr.MR_ERR_INVALID_ARG  # no accumulator
    assert comb(p, p, p, p, 0, p, None, 10, 64, 8, 16, 24, p, p, None) == \
        mr.MR_ERR_UNSUPPORTED  # n_out % 16 != 0
    assert comb(p, p, p, p, 0, p, C.c_void_p(72), 10, 64, 8, 16, 32, p, p, None) == \
        mr.MR_ERR_UNSUPPORTED  # shared not 16-byte aligned
    assert comb(None, None, None, None, 0, None, None, 0, 64, 8, 16, 32, None, None, None) == \
        mr.MR_OK


def test_selftest_rejects_unknown_case():
    assert mr.lib().mr_selftest_bounded_wait(7, None) == mr.MR_ERR_INVALID_ARG
