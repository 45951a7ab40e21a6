"""Seeded synthetic workloads for the MoE routing hot path.

This module is shared by the CUDA-side tests/bench and by the CPU oracle's
tests.  It holds *only* workload shapes, value distributions and the random
draws; none of the routing arithmetic (no logits, scores, top-k, dispatch or
combine) lives here.

Shapes and hyper-parameters follow the pages:

* DeepSeek-V3 / V3.2 router: 256 routed experts, 8 groups of which 4 are
  kept, top-8, route_scale 2.5 (DeepSeek-V3.2-Exp "Normalize weights" page,
  model.py excerpt; DeepSeek-V3 "MoE Router" study note, "Official code").
* Kimi K2 router: 384 experts, one group, top-8, route_scale 2.827 (Kimi K2
  "Normalize weights" page, formula and explanation).
* Hidden size d = 7168 (Kimi K2 "Add shared output" page, shapes; Kimi K3
  "MoE update" decode shape).

Random recipe (stated once, used everywhere):

* numpy ``Generator(PCG64)``; one child ``SeedSequence`` per tensor, spawned
  from ``SeedSequence(seed)`` in the order x, W, b, E, shared.  Large tensors
  are drawn in row blocks of ``_BLOCK`` elements, each block from its own
  grandchild sequence, so the values do not depend on thread count.
* x: N(0,1).  For bf16 workloads x is quantised to bf16 (round to nearest
  even) and the fp32 copy holds the widened bf16 values exactly.
* W: N(0,1)/sqrt(d) in fp32 (logits ~ N(0,1)); the bf16-stored gate weight
  is that W rounded to bf16 (nearest even).
* b: U(lo, hi) fp32; the skewed workload adds +1.0 to experts [0, 32).
* E (synthetic expert outputs, expert-sorted rows [T*k, d]) and shared
  ([T, d]): N(0,1), bf16 for bf16 workloads, fp32 otherwise.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import math
import os

import numpy as np

F32 = "f32"
BF16 = "bf16"

MASK_NEG_INF = 0
MASK_ZERO = 1

_BLOCK = 1 << 24  # elements per independently-seeded block


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic routing problem: sizes, router hyper-parameters, recipe."""

    name: str
    T: int
    d: int
    N_r: int
    n_group: int
    topk_group: int
    k: int
    route_scale: float
    mask_mode: int
    seed: int
    io_dtype: str = BF16          # dtype of x rows moved by gather, E, shared, y
    bias_lo: float = -0.1
    bias_hi: float = 0.1
    hot_experts: int = 0          # experts [0, hot_experts) get hot_bias added
    hot_bias: float = 0.0
    with_bias: bool = True

    @property
    def S(self) -> int:
        return self.N_r // self.n_group

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five configurations the routing path is specified on.
TINY = Workload("tiny_T64_d512_E64", T=64, d=512, N_r=64, n_group=4, topk_group=2,
                k=4, route_scale=2.5, mask_mode=MASK_NEG_INF, seed=0,
                io_dtype=F32, bias_lo=-0.05, bias_hi=0.05)
V3_PREFILL = Workload("deepseek_v3_prefill_T4096", T=4096, d=7168, N_r=256,
                      n_group=8, topk_group=4, k=8, route_scale=2.5,
                      mask_mode=MASK_NEG_INF, seed=1)
K2_PREFILL = Workload("kimi_k2_prefill_T8192", T=8192, d=7168, N_r=384,
                      n_group=1, topk_group=1, k=8, route_scale=2.827,
                      mask_mode=MASK_ZERO, seed=2)
V3_DECODE = Workload("deepseek_v3_decode_T64", T=64, d=7168, N_r=256, n_group=8,
                     topk_group=4, k=8, route_scale=2.5, mask_mode=MASK_NEG_INF,
                     seed=3)
V3_FULL = Workload("deepseek_v3_full_route_dispatch_combine_T16384", T=16384,
                   d=7168, N_r=256, n_group=8, topk_group=4, k=8,
                   route_scale=2.5, mask_mode=MASK_NEG_INF, seed=4,
                   hot_experts=32, hot_bias=1.0)

ALL = [TINY, V3_PREFILL, K2_PREFILL, V3_DECODE, V3_FULL]
BY_NAME = {w.name: w for w in ALL}

_TENSORS = ("x", "W", "b", "E", "shared", "expert_W")


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Quantise finite fp32 values to bf16 bit patterns, round-to-nearest-even.

    Used only to *make* bf16 inputs; the values drawn here are finite.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + (np.uint32(0x7FFF) + lsb)) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _child(seed: int, tensor: str) -> np.random.SeedSequence:
    return np.random.SeedSequence(seed).spawn(len(_TENSORS))[_TENSORS.index(tensor)]


def _normal_blocks(ss: np.random.SeedSequence, n: int, out_dtype: str,
                   threads: int | None = None) -> np.ndarray:
    """n draws of N(0,1) as fp32 (or bf16 bits), block-seeded, thread-parallel."""
    nblk = max(1, math.ceil(n / _BLOCK))
    kids = ss.spawn(nblk)
    out = np.empty(n, dtype=np.uint16 if out_dtype == BF16 else np.float32)

    def fill(i: int) -> None:
        lo, hi = i * _BLOCK, min(n, (i + 1) * _BLOCK)
        z = np.random.Generator(np.random.PCG64(kids[i])).standard_normal(
            hi - lo, dtype=np.float32)
        out[lo:hi] = to_bf16_bits(z) if out_dtype == BF16 else z

    if nblk == 1:
        fill(0)
    else:
        nt = threads or min(16, len(os.sched_getaffinity(0)))
        with _cf.ThreadPoolExecutor(nt) as ex:
            list(ex.map(fill, range(nblk)))
    return out


def gen_x(w: Workload) -> dict:
    """Token rows.  Returns {'x_f32': [T,d] fp32, 'x_bf16': [T,d] uint16 | None}."""
    n = w.T * w.d
    if w.io_dtype == BF16:
        bits = _normal_blocks(_child(w.seed, "x"), n, BF16).reshape(w.T, w.d)
        return {"x_f32": bf16_bits_to_f32(bits), "x_bf16": bits}
    x = _normal_blocks(_child(w.seed, "x"), n, F32).reshape(w.T, w.d)
    return {"x_f32": x, "x_bf16": None}


def gen_W(w: Workload) -> np.ndarray:
    """Gate weight [N_r, d] fp32, N(0, 1/d)."""
    z = _normal_blocks(_child(w.seed, "W"), w.N_r * w.d, F32).reshape(w.N_r, w.d)
    return (z / np.float32(math.sqrt(w.d))).astype(np.float32)


def gen_W_bf16(w: Workload) -> dict:
    """The gate weight stored in bf16: gen_W rounded to bf16 (nearest even).
    Returns the bf16 bit patterns [N_r, d] (uint16) and their exact fp32
    values."""
    bits = to_bf16_bits(gen_W(w))
    return {"W_bf16": bits, "W_f32": bf16_bits_to_f32(bits)}


def gen_expert_W(w: Workload, n_out: int) -> np.ndarray:
    """Synthetic expert weights [N_r, n_out, d] as bf16 bit patterns:
    N(0, 1/d) rounded to bf16 (a linear expert layer; no trained weights)."""
    z = _normal_blocks(_child(w.seed, "expert_W"), w.N_r * n_out * w.d, F32)
    return to_bf16_bits((z / np.float32(math.sqrt(w.d))).astype(np.float32)).reshape(
        w.N_r, n_out, w.d)


def gen_b(w: Workload) -> np.ndarray | None:
    """Selection bias [N_r] fp32, or None for a bias-free workload."""
    if not w.with_bias:
        return None
    g = np.random.Generator(np.random.PCG64(_child(w.seed, "b")))
    b = g.uniform(w.bias_lo, w.bias_hi, size=w.N_r).astype(np.float32)
    if w.hot_experts:
        b[: w.hot_experts] += np.float32(w.hot_bias)
    return b


def gen_E(w: Workload) -> np.ndarray:
    """Synthetic expert outputs in expert-sorted order, [T*k, d] (bf16 bits or fp32)."""
    return _normal_blocks(_child(w.seed, "E"), w.T * w.k * w.d, w.io_dtype).reshape(
        w.T * w.k, w.d)


def gen_shared(w: Workload) -> np.ndarray:
    """Shared-expert output [T, d] (bf16 bits or fp32)."""
    return _normal_blocks(_child(w.seed, "shared"), w.T * w.d, w.io_dtype).reshape(
        w.T, w.d)


def gen_router_inputs(w: Workload) -> dict:
    d = gen_x(w)
    d["W"] = gen_W(w)
    d["b"] = gen_b(w)
    return d


def describe() -> str:
    lines = []
    for w in ALL:
        lines.append(f"{w.name}: T={w.T} d={w.d} N_r={w.N_r} G={w.n_group} "
                     f"Gk={w.topk_group} k={w.k} scale={w.route_scale} "
                     f"mask={'-inf' if w.mask_mode == MASK_NEG_INF else 'zero'} "
                     f"seed={w.seed} io={w.io_dtype}")
    return "\n".join(lines)
