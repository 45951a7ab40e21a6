"""ctypes binding of libmr.so (include/mr.h): argument marshalling only.

Every function here takes torch CUDA tensors, checks dtype/shape/contiguity,
allocates missing outputs with torch (device memory is PyTorch's job), and
calls the C entry point of the same name on the current torch stream.  No
step of the routing path is computed in Python; there is no CPU fallback:
if libmr.so is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmr.so")

MR_OK = 0
MR_ERR_INVALID_ARG = -1
MR_ERR_UNSUPPORTED = -2
MR_ERR_CUDA = -3
MR_ERR_DEVICE = -4
MR_ERR_TIMEOUT = -5
MR_ERR_OVERFLOW = -6

MR_F32 = 0
MR_BF16 = 1
MR_MASK_NEG_INF = 0
MR_MASK_ZERO = 1
MR_PREC_3XTF32 = 0
MR_PREC_TF32 = 1
MR_PREC_FFMA = 2
MR_PREC_BF16X3 = 3
MR_SCORE_SOFTMAX = 1
MR_GROUP_MAX = 2
MR_NORM_NO_EPS = 4

_lib = None


class MRError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")


class _IpcHandle(C.Structure):
    """mr_ipc_handle_t: the CUDA IPC handle of an allocation, the buffer's
    offset in it and its size."""
    _fields_ = [("handle", C.c_ubyte * 64), ("offset", C.c_uint64), ("bytes", C.c_uint64)]


def lib():
    """The loaded libmr.so (raises ImportError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run "
                              "`python -m token_dispatch_fp32_b200.build`")
        L = C.CDLL(LIB_PATH)
        p, i, f, sz = C.c_void_p, C.c_int, C.c_float, C.c_size_t
        L.mr_version.restype = i
        L.mr_status_string.argtypes = [i]
        L.mr_status_string.restype = C.c_char_p
        L.mr_router_forward.argtypes = [p, p, p, i, i, i, i, i, i, f, i, p, p, p]
        L.mr_router_forward_ex.argtypes = [p, i, p, p, i, i, i, i, i, i, f, i, i, p, p, p, p,
                                           sz, p]
        L.mr_router_forward_ex2.argtypes = [p, i, p, p, i, i, i, i, i, i, f, i, i, i, p, p, p,
                                            p, sz, p]
        L.mr_router_forward_bf16w.argtypes = [p, i, p, p, i, i, i, i, i, i, f, i, i, p, p, p,
                                              p, sz, p]
        L.mr_router_workspace_size.argtypes = [i, i, i]
        L.mr_router_workspace_size.restype = sz
        L.mr_dispatch_workspace_size.argtypes = [i, i, i]
        L.mr_dispatch_workspace_size.restype = sz
        L.mr_dispatch.argtypes = [p, i, i, i, p, p, p, p, p, sz, p]
        L.mr_dispatch_noalloc.argtypes = [p, i, i, i, p, p, p, p, p]
        L.mr_dispatch_noalloc_max_workspace.restype = sz
        L.mr_router_forward_max_scratch.restype = sz
        L.mr_gather_rows.argtypes = [p, i, i, i, i, p, p, p, p]
        L.mr_ep_recv_order.argtypes = [p, i, i, i, p, p, p, p, p]
        L.mr_expert_gemm_gather.argtypes = [p, p, p, p, i, i, i, i, i, p, p]
        L.mr_expert_gemm_gather_packed.argtypes = [p, p, p, p, i, i, i, i, i, p, p]
        L.mr_expert_gemm_gather_combine.argtypes = [p, p, p, p, i, p, p, i, i, i, i, i, p, p, p]
        L.mr_expert_packed_bytes.argtypes = [i, i, i]
        L.mr_expert_packed_bytes.restype = sz
        L.mr_expert_pack_weights.argtypes = [p, i, i, i, p, sz, p]
        L.mr_combine.argtypes = [p, i, p, p, p, p, i, i, i, p]
        L.mr_ep_dispatch_p2p.argtypes = [p, i, i, i, i, p, p, p, p, i, i, i, p, i, p, p, p, p]
        L.mr_ep_combine_p2p.argtypes = [p, i, i, p, p, p, i, i, i, p, p, i, i, p]
        L.mr_ipc_export.argtypes = [p, sz, C.POINTER(_IpcHandle)]
        L.mr_ipc_import.argtypes = [C.POINTER(_IpcHandle), C.POINTER(p), C.POINTER(p)]
        L.mr_ipc_close.argtypes = [p]
        L.mr_get_error.argtypes = [p]
        L.mr_selftest_bounded_wait.argtypes = [i, p]
        L.mr_launch_count.restype = C.c_uint64
        for fn in ("mr_router_forward", "mr_router_forward_ex", "mr_dispatch", "mr_dispatch_noalloc",
                   "mr_gather_rows", "mr_combine", "mr_get_error"):
            getattr(L, fn).restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().mr_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != MR_OK:
        raise MRError(fn, status)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _call(fn: str, dev, stream, *args) -> None:
    """Calls C entry point `fn` with `dev` as the current CUDA device and the
    stream handle as the last argument: the library launches on the current
    device, so the tensors' device is made current for the call.  `stream`
    (default: that device's current stream) must belong to the same device."""
    with torch.cuda.device(dev):
        if stream is None:
            stream = torch.cuda.current_stream(dev)
        elif stream.device != dev:
            raise ValueError(f"stream is on {stream.device}, tensors on {dev}")
        _check(fn, getattr(lib(), fn)(*args, C.c_void_p(stream.cuda_stream)))


def _device_of(*tensors):
    """The one CUDA device of the given tensors (None entries ignored)."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"tensors must be on one CUDA device, got {sorted(map(str, devs))}")
    return devs.pop()


def _need(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _row_dtype(t):
    if t.dtype == torch.bfloat16:
        return MR_BF16
    if t.dtype == torch.float32:
        return MR_F32
    raise TypeError("row tensors must be bfloat16 or float32")


def version() -> int:
    return int(lib().mr_version())


def mr_router_forward(x, W, bias, n_group, topk_group, k, route_scale, mask_mode,
                      idx_out=None, w_out=None, stream=None):
    """Gate forward (include/mr.h).  x [T,d] fp32, W [N_r,d] fp32, bias [N_r]
    fp32 or None.  Returns (idx [T,k] int32, w [T,k] fp32)."""
    _need(x, "x", torch.float32)
    T, d = x.shape
    _need(W, "W", torch.float32)
    N_r = W.shape[0]
    _need(W, "W", torch.float32, (N_r, d))
    if bias is not None:
        _need(bias, "bias", torch.float32, (N_r,))
    idx_out = torch.empty((T, k), dtype=torch.int32, device=x.device) if idx_out is None else \
        _need(idx_out, "idx_out", torch.int32, (T, k))
    w_out = torch.empty((T, k), dtype=torch.float32, device=x.device) if w_out is None else \
        _need(w_out, "w_out", torch.float32, (T, k))
    dev = _device_of(x, W, bias, idx_out, w_out)
    _call("mr_router_forward", dev, stream, _ptr(x), _ptr(W), _ptr(bias), T, d, N_r, n_group,
          topk_group, k, float(route_scale), mask_mode, _ptr(idx_out), _ptr(w_out))
    return idx_out, w_out


def mr_router_forward_max_scratch() -> int:
    """Bytes of the fixed array holding mr_router_forward's split-K partials."""
    return int(lib().mr_router_forward_max_scratch())


def mr_router_workspace_size(T, d, N_r) -> int:
    return int(lib().mr_router_workspace_size(T, d, N_r))


def mr_router_forward_ex(x, W, bias, n_group, topk_group, k, route_scale, mask_mode,
                         precision=MR_PREC_3XTF32, idx_out=None, w_out=None, logits_out=None,
                         workspace=None, stream=None, flags=0):
    """mr_router_forward with x dtype (fp32 or bf16), precision, optional
    logits output and workspace; flags != 0 (MR_SCORE_SOFTMAX, MR_GROUP_MAX,
    MR_NORM_NO_EPS) calls mr_router_forward_ex2.  Returns (idx, w)."""
    _need(x, "x")
    x_dtype = _row_dtype(x)
    T, d = x.shape
    N_r = W.shape[0]
    _need(W, "W", torch.float32, (N_r, d))
    if bias is not None:
        _need(bias, "bias", torch.float32, (N_r,))
    idx_out = torch.empty((T, k), dtype=torch.int32, device=x.device) if idx_out is None else \
        _need(idx_out, "idx_out", torch.int32, (T, k))
    w_out = torch.empty((T, k), dtype=torch.float32, device=x.device) if w_out is None else \
        _need(w_out, "w_out", torch.float32, (T, k))
    if logits_out is not None:
        _need(logits_out, "logits_out", torch.float32, (T, N_r))
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    dev = _device_of(x, W, bias, idx_out, w_out, logits_out, workspace)
    if flags:
        _call("mr_router_forward_ex2", dev, stream, _ptr(x), x_dtype, _ptr(W), _ptr(bias), T, d,
              N_r, n_group, topk_group, k, float(route_scale), mask_mode, precision,
              int(flags), _ptr(idx_out), _ptr(w_out), _ptr(logits_out), _ptr(workspace),
              ws_bytes)
    else:
        _call("mr_router_forward_ex", dev, stream, _ptr(x), x_dtype, _ptr(W), _ptr(bias), T, d,
              N_r, n_group, topk_group, k, float(route_scale), mask_mode, precision,
              _ptr(idx_out), _ptr(w_out), _ptr(logits_out), _ptr(workspace), ws_bytes)
    return idx_out, w_out


def mr_router_forward_bf16w(x, W_bf16, bias, n_group, topk_group, k, route_scale, mask_mode,
                            idx_out=None, w_out=None, logits_out=None, workspace=None,
                            stream=None, flags=0):
    """The gate with a bf16-stored weight W_bf16 [N_r,d] (torch.bfloat16):
    x [T,d] bf16 (tensor cores) or fp32 (CUDA cores).  Returns (idx, w)."""
    _need(x, "x")
    x_dtype = _row_dtype(x)
    T, d = x.shape
    N_r = W_bf16.shape[0]
    _need(W_bf16, "W_bf16", torch.bfloat16, (N_r, d))
    if bias is not None:
        _need(bias, "bias", torch.float32, (N_r,))
    idx_out = torch.empty((T, k), dtype=torch.int32, device=x.device) if idx_out is None else \
        _need(idx_out, "idx_out", torch.int32, (T, k))
    w_out = torch.empty((T, k), dtype=torch.float32, device=x.device) if w_out is None else \
        _need(w_out, "w_out", torch.float32, (T, k))
    if logits_out is not None:
        _need(logits_out, "logits_out", torch.float32, (T, N_r))
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    _call("mr_router_forward_bf16w", _device_of(x, W_bf16, bias, idx_out, w_out, logits_out,
                                                 workspace), stream,
          _ptr(x), x_dtype, _ptr(W_bf16), _ptr(bias), T, d, N_r, n_group, topk_group, k,
          float(route_scale), mask_mode, int(flags), _ptr(idx_out), _ptr(w_out),
          _ptr(logits_out), _ptr(workspace), ws_bytes)
    return idx_out, w_out


def mr_dispatch_workspace_size(T, k, N_r) -> int:
    return int(lib().mr_dispatch_workspace_size(T, k, N_r))


def mr_dispatch(idx, N_r, counts=None, offsets=None, perm=None, inv_perm=None, workspace=None,
                want_inv=True, stream=None):
    """Dispatch bookkeeping.  idx [T,k] int32.  Returns (counts, offsets,
    perm, inv_perm) as int32 tensors (inv_perm None when want_inv is False)."""
    _need(idx, "idx", torch.int32)
    T, k = idx.shape
    dev = idx.device
    counts = torch.empty(N_r, dtype=torch.int32, device=dev) if counts is None else \
        _need(counts, "counts", torch.int32, (N_r,))
    offsets = torch.empty(N_r + 1, dtype=torch.int32, device=dev) if offsets is None else \
        _need(offsets, "offsets", torch.int32, (N_r + 1,))
    perm = torch.empty(T * k, dtype=torch.int32, device=dev) if perm is None else \
        _need(perm, "perm", torch.int32, (T * k,))
    if inv_perm is None and want_inv:
        inv_perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    elif inv_perm is not None:
        _need(inv_perm, "inv_perm", torch.int32, (T * k,))
    need = mr_dispatch_workspace_size(T, k, N_r)
    if workspace is None:
        workspace = torch.empty(max(need, 4), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace")
    _call("mr_dispatch", _device_of(idx, counts, offsets, perm, inv_perm, workspace), stream,
          _ptr(idx), T, k, N_r, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv_perm),
          _ptr(workspace), workspace.numel() * workspace.element_size())
    return counts, offsets, perm, inv_perm


def mr_dispatch_noalloc(idx, N_r, counts, offsets, perm, inv_perm=None, stream=None):
    """Dispatch into caller-provided outputs with no workspace argument: the C
    entry point uses a fixed scratch array inside libmr.so and allocates
    nothing (for callers that may not allocate device memory at dispatch
    time).  Outputs must be preallocated int32 CUDA tensors."""
    _need(idx, "idx", torch.int32)
    T, k = idx.shape
    _need(counts, "counts", torch.int32, (N_r,))
    _need(offsets, "offsets", torch.int32, (N_r + 1,))
    _need(perm, "perm", torch.int32, (T * k,))
    if inv_perm is not None:
        _need(inv_perm, "inv_perm", torch.int32, (T * k,))
    # the device made current here is the one whose scratch array the call uses
    _call("mr_dispatch_noalloc", _device_of(idx, counts, offsets, perm, inv_perm), stream,
          _ptr(idx), T, k, N_r, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv_perm))
    return counts, offsets, perm, inv_perm


def mr_dispatch_noalloc_max_workspace() -> int:
    return int(lib().mr_dispatch_noalloc_max_workspace())


def mr_ep_recv_order(recv_counts, R, order=None, inv_order=None, local_counts=None,
                     local_offsets=None, stream=None):
    """Receive-side order of the expert-parallel exchange: recv_counts
    [ep, E_loc] int32 (device), R = its sum (rows received).  Returns
    (order [R], inv_order [R], local_counts [E_loc], local_offsets [E_loc+1])."""
    _need(recv_counts, "recv_counts", torch.int32)
    ep, E_loc = recv_counts.shape
    dev = recv_counts.device
    order = torch.empty(R, dtype=torch.int32, device=dev) if order is None else \
        _need(order, "order", torch.int32, (R,))
    inv_order = torch.empty(R, dtype=torch.int32, device=dev) if inv_order is None else \
        _need(inv_order, "inv_order", torch.int32, (R,))
    local_counts = torch.empty(E_loc, dtype=torch.int32, device=dev) if local_counts is None \
        else _need(local_counts, "local_counts", torch.int32, (E_loc,))
    local_offsets = torch.empty(E_loc + 1, dtype=torch.int32, device=dev) \
        if local_offsets is None else _need(local_offsets, "local_offsets", torch.int32,
                                            (E_loc + 1,))
    _call("mr_ep_recv_order", _device_of(recv_counts, order, inv_order, local_counts,
                                          local_offsets), stream,
          _ptr(recv_counts), ep, E_loc, int(R), _ptr(order), _ptr(inv_order),
          _ptr(local_counts), _ptr(local_offsets))
    return order, inv_order, local_counts, local_offsets


def mr_expert_gemm_gather(x, k, perm, offsets, W_exp, out=None, stream=None):
    """One linear expert layer over the expert-sorted rows with the row
    gather fused in: out [T*k, n_out] bf16, row j = x[perm[j] // k] .
    W_exp[e(j)]^T.  x [T,d] bf16, perm [T*k], offsets [N_r+1] int32 (from
    mr_dispatch), W_exp [N_r, n_out, d] bf16."""
    _need(x, "x", torch.bfloat16)
    T, d = x.shape
    if perm is None:  # x already holds the T*k expert-sorted rows
        if T % k:
            raise ValueError("without perm, x must have T*k rows")
        T //= k
    else:
        _need(perm, "perm", torch.int32, (T * k,))
    _need(W_exp, "W_exp", torch.bfloat16)
    N_r, n_out, dw = W_exp.shape
    if dw != d:
        raise ValueError(f"W_exp is [N_r, n_out, {dw}], x rows have {d} columns")
    _need(offsets, "offsets", torch.int32, (N_r + 1,))
    out = torch.empty((T * k, n_out), dtype=torch.bfloat16, device=x.device) if out is None \
        else _need(out, "out", torch.bfloat16, (T * k, n_out))
    _call("mr_expert_gemm_gather", _device_of(x, perm, offsets, W_exp, out), stream,
          _ptr(x), _ptr(perm), _ptr(offsets), _ptr(W_exp), T, d, k, N_r, n_out, _ptr(out))
    return out


def mr_expert_pack_weights(W_exp, stream=None):
    """W_exp [N_r, n_out, d] bf16 -> the packed tile layout (a flat bf16
    tensor) that mr_expert_gemm_gather_packed reads."""
    _need(W_exp, "W_exp", torch.bfloat16)
    N_r, n_out, d = W_exp.shape
    n = int(lib().mr_expert_packed_bytes(N_r, n_out, d))
    Wp = torch.empty(n // 2, dtype=torch.bfloat16, device=W_exp.device)
    _call("mr_expert_pack_weights", _device_of(W_exp, Wp), stream, _ptr(W_exp), N_r, n_out, d,
          _ptr(Wp), n)
    return Wp


def mr_expert_gemm_gather_packed(x, k, perm, offsets, W_packed, N_r, n_out, out=None,
                                 stream=None):
    """mr_expert_gemm_gather with packed weights (mr_expert_pack_weights)."""
    _need(x, "x", torch.bfloat16)
    T, d = x.shape
    if perm is None:  # x already holds the T*k expert-sorted rows
        if T % k:
            raise ValueError("without perm, x must have T*k rows")
        T //= k
    else:
        _need(perm, "perm", torch.int32, (T * k,))
    _need(offsets, "offsets", torch.int32, (N_r + 1,))
    _need(W_packed, "W_packed", torch.bfloat16)
    if W_packed.numel() * 2 < int(lib().mr_expert_packed_bytes(N_r, n_out, d)):
        raise ValueError("W_packed is smaller than mr_expert_packed_bytes")
    out = torch.empty((T * k, n_out), dtype=torch.bfloat16, device=x.device) if out is None \
        else _need(out, "out", torch.bfloat16, (T * k, n_out))
    _call("mr_expert_gemm_gather_packed", _device_of(x, perm, offsets, W_packed, out), stream,
          _ptr(x), _ptr(perm), _ptr(offsets), _ptr(W_packed), T, d, k, N_r, n_out, _ptr(out))
    return out


def mr_expert_gemm_gather_combine(x, k, perm, offsets, W, w, shared=None, N_r=None,
                                  n_out=None, packed=False, acc=None, y=None, stream=None):
    """The expert layer with the gather and the weighted combine fused in:
    y [T, n_out] bf16 = bf16(bf16(sum_j w[t,j] * bf16(x[t] . W[e_j]^T)) +
    shared[t]).  x [T,d] bf16; perm [T*k], offsets [N_r+1] int32 (from
    mr_dispatch); W [N_r, n_out, d] bf16, or the packed layout
    (mr_expert_pack_weights; packed=True, N_r and n_out given); w [T,k] fp32;
    shared [T, n_out] bf16 or None.  acc: [T, n_out] fp32 scratch (allocated
    when None; holds the fp32 routed sums afterwards).  Returns y."""
    _need(x, "x", torch.bfloat16)
    T, d = x.shape
    _need(perm, "perm", torch.int32, (T * k,))
    _need(W, "W", torch.bfloat16)
    if packed:
        if N_r is None or n_out is None:
            raise ValueError("packed weights need N_r and n_out")
        if W.numel() * 2 < int(lib().mr_expert_packed_bytes(N_r, n_out, d)):
            raise ValueError("W is smaller than mr_expert_packed_bytes")
    else:
        N_r, n_out, dw = W.shape
        if dw != d:
            raise ValueError(f"W is [N_r, n_out, {dw}], x rows have {d} columns")
    _need(offsets, "offsets", torch.int32, (N_r + 1,))
    _need(w, "w", torch.float32, (T, k))
    if shared is not None:
        _need(shared, "shared", torch.bfloat16, (T, n_out))
    acc = torch.empty((T, n_out), dtype=torch.float32, device=x.device) if acc is None \
        else _need(acc, "acc", torch.float32, (T, n_out))
    y = torch.empty((T, n_out), dtype=torch.bfloat16, device=x.device) if y is None \
        else _need(y, "y", torch.bfloat16, (T, n_out))
    _call("mr_expert_gemm_gather_combine", _device_of(x, perm, offsets, W, w, shared, acc, y),
          stream, _ptr(x), _ptr(perm), _ptr(offsets), _ptr(W), 1 if packed else 0, _ptr(w),
          _ptr(shared), T, d, k, N_r, n_out, _ptr(acc), _ptr(y))
    return y


def mr_gather_rows(x, k, perm=None, inv_perm=None, xs=None, stream=None):
    """sorted rows xs [T*k, d] = x[perm // k] (x bf16 or fp32)."""
    _need(x, "x")
    T, d = x.shape
    dt = _row_dtype(x)
    if perm is not None:
        _need(perm, "perm", torch.int32, (T * k,))
    if inv_perm is not None:
        _need(inv_perm, "inv_perm", torch.int32, (T * k,))
    xs = torch.empty((T * k, d), dtype=x.dtype, device=x.device) if xs is None else \
        _need(xs, "xs", x.dtype, (T * k, d))
    _call("mr_gather_rows", _device_of(x, perm, inv_perm, xs), stream, _ptr(x), dt, T, d, k,
          _ptr(perm), _ptr(inv_perm), _ptr(xs))
    return xs


def mr_combine(expert_out, w, inv_perm, shared=None, y=None, stream=None):
    """y [T,d] = combine of expert_out [T*k,d] with w [T,k] (+ shared [T,d])."""
    _need(w, "w", torch.float32)
    T, k = w.shape
    _need(expert_out, "expert_out")
    d = expert_out.shape[1]
    _need(expert_out, "expert_out", None, (T * k, d))
    dt = _row_dtype(expert_out)
    _need(inv_perm, "inv_perm", torch.int32, (T * k,))
    if shared is not None:
        _need(shared, "shared", expert_out.dtype, (T, d))
    y = torch.empty((T, d), dtype=expert_out.dtype, device=expert_out.device) if y is None else \
        _need(y, "y", expert_out.dtype, (T, d))
    _call("mr_combine", _device_of(expert_out, w, inv_perm, shared, y), stream,
          _ptr(expert_out), dt, _ptr(w), _ptr(inv_perm), _ptr(shared), _ptr(y), T, d, k)
    return y


def _addresses(bufs, name, dev):
    """HOST array of device addresses: each entry an int address or a CUDA
    tensor on `dev`."""
    out = []
    for j, b in enumerate(bufs):
        if isinstance(b, torch.Tensor):
            if not b.is_cuda or b.device != dev:
                raise ValueError(f"{name}[{j}] must be on {dev}")
            out.append(b.data_ptr())
        else:
            out.append(int(b))
    return (C.c_void_p * len(out))(*out)


def mr_ep_dispatch_p2p(x, idx, inv_perm, offsets, counts_all, rank, recv_bufs, capacity,
                       dest=None, local_counts=None, local_offsets=None, stream=None):
    """This rank's rows to their owners' receive buffers (peer memory).
    x [T,d] bf16/fp32, idx [T,k] int32, inv_perm/offsets from mr_dispatch,
    counts_all [ep, N_r] int32 (every rank's counts), recv_bufs: ep device
    addresses (int, e.g. from mr_ipc_import) or tensors, each a buffer of
    capacity rows of d elements of x's dtype.  Returns (dest [T*k],
    local_counts [E_loc], local_offsets [E_loc+1])."""
    _need(x, "x")
    T, d = x.shape
    dt = _row_dtype(x)
    _need(idx, "idx", torch.int32)
    k = idx.shape[1]
    _need(idx, "idx", torch.int32, (T, k))
    _need(counts_all, "counts_all", torch.int32)
    ep, N_r = counts_all.shape
    _need(inv_perm, "inv_perm", torch.int32, (T * k,))
    _need(offsets, "offsets", torch.int32, (N_r + 1,))
    if len(recv_bufs) != ep:
        raise ValueError(f"{len(recv_bufs)} receive buffers for {ep} ranks")
    if N_r % ep:
        raise ValueError(f"{N_r} experts do not split over {ep} ranks")
    E_loc = N_r // ep
    dev = _device_of(x, idx, inv_perm, offsets, counts_all)
    dest = torch.empty(T * k, dtype=torch.int32, device=dev) if dest is None else \
        _need(dest, "dest", torch.int32, (T * k,))
    local_counts = torch.empty(E_loc, dtype=torch.int32, device=dev) if local_counts is None \
        else _need(local_counts, "local_counts", torch.int32, (E_loc,))
    local_offsets = torch.empty(E_loc + 1, dtype=torch.int32, device=dev) \
        if local_offsets is None else _need(local_offsets, "local_offsets", torch.int32,
                                            (E_loc + 1,))
    _call("mr_ep_dispatch_p2p", _device_of(x, dest, local_counts, local_offsets), stream,
          _ptr(x), dt, T, d, k, _ptr(idx), _ptr(inv_perm), _ptr(offsets), _ptr(counts_all), ep,
          int(rank), N_r, _addresses(recv_bufs, "recv_bufs", dev), int(capacity), _ptr(dest),
          _ptr(local_counts), _ptr(local_offsets))
    return dest, local_counts, local_offsets


def mr_ep_combine_p2p(out_bufs, w, idx, dest, N_r, capacity, d, dtype, shared=None, y=None,
                      stream=None):
    """y [T,d] = the weighted combine (+ shared [T,d]) of the expert outputs
    in the owners' output buffers out_bufs (ep device addresses or tensors,
    capacity rows of d elements of `dtype` each), slot t*k+j at row dest[t*k+j]
    of idx[t,j]'s owner."""
    _need(w, "w", torch.float32)
    T, k = w.shape
    _need(idx, "idx", torch.int32, (T, k))
    _need(dest, "dest", torch.int32, (T * k,))
    dev = _device_of(w, idx, dest)
    dt = MR_BF16 if dtype == torch.bfloat16 else MR_F32 if dtype == torch.float32 else None
    if dt is None:
        raise TypeError("rows must be bfloat16 or float32")
    if shared is not None:
        _need(shared, "shared", dtype, (T, d))
    y = torch.empty((T, d), dtype=dtype, device=dev) if y is None else \
        _need(y, "y", dtype, (T, d))
    ep = len(out_bufs)
    _call("mr_ep_combine_p2p", _device_of(w, idx, dest, shared, y), stream,
          _addresses(out_bufs, "out_bufs", dev), dt, int(d), _ptr(w), _ptr(idx), _ptr(dest), ep,
          int(N_r), int(capacity), _ptr(shared), _ptr(y), T, k)
    return y


def mr_ipc_export(t) -> bytes:
    """The IPC handle (bytes) of CUDA tensor t's memory, for another process."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("t must be a CUDA tensor")
    h = _IpcHandle()
    with torch.cuda.device(t.device):
        _check("mr_ipc_export", lib().mr_ipc_export(C.c_void_p(t.data_ptr()),
                                                    t.numel() * t.element_size(), C.byref(h)))
    return bytes(C.string_at(C.addressof(h), C.sizeof(h)))


def mr_ipc_import(handle: bytes, device):
    """Opens another process's handle on `device`: returns (base, address,
    bytes); pass base to mr_ipc_close."""
    if len(handle) != C.sizeof(_IpcHandle):
        raise ValueError(f"an IPC handle has {C.sizeof(_IpcHandle)} bytes, got {len(handle)}")
    h = _IpcHandle.from_buffer_copy(handle)
    base, ptr = C.c_void_p(), C.c_void_p()
    with torch.cuda.device(device):
        _check("mr_ipc_import", lib().mr_ipc_import(C.byref(h), C.byref(base), C.byref(ptr)))
    return base.value, ptr.value, int(h.bytes)


def mr_ipc_close(base, device) -> None:
    """Unmaps a buffer opened by mr_ipc_import."""
    with torch.cuda.device(device):
        _check("mr_ipc_close", lib().mr_ipc_close(C.c_void_p(base)))


def mr_launch_count() -> int:
    """Kernels launched by libmr.so in this process so far."""
    return int(lib().mr_launch_count())


def mr_get_error(stream=None) -> int:
    """Synchronise the stream and read/clear the error flag of the stream's
    device (default: the current stream of the current device); returns the
    status."""
    if stream is None:
        return int(lib().mr_get_error(_stream(None)))
    with torch.cuda.device(stream.device):
        return int(lib().mr_get_error(C.c_void_p(stream.cuda_stream)))
