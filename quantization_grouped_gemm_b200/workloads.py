"""Seeded synthetic MoE workloads for the FP8 quantisation + grouped-GEMM path.

This module holds no quantisation or GEMM arithmetic: it only draws random
numbers, rounds them to bf16 (torch's round-to-nearest-even cast) and builds
routing offsets.  Both the CUDA path and the CPU oracle are fed from here.

RNG: numpy PCG64, one stream per tensor via ``SeedSequence(seed, spawn_key=(tensor_id,))``.
Seed of the named workloads = 1000 + workload number.  Shapes follow the
model shapes the pages quote (Llama3-8B FFN, DeepSeek-MoE-16B, DeepSeek-V3
with 32 local experts, Llama-4-style 16 experts); no model weights or data.
"""
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

# tensor ids of the per-tensor random streams
_T_X, _T_W, _T_G, _T_ROUTE, _T_OUTL, _T_ZERO = 1, 2, 3, 4, 5, 6


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(tensor_id,))))


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32 numpy -> bf16 torch (CPU), round to nearest even."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a CPU bf16 tensor as numpy uint16 (no copy)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def normal_bf16(seed: int, tensor_id: int, shape, std: float) -> torch.Tensor:
    g = rng(seed, tensor_id)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return to_bf16(a)


def offsets_from_sizes(sizes) -> np.ndarray:
    return np.cumsum(np.asarray(sizes, dtype=np.int64)).astype(np.int32)


def zipf_weights(n: int, exponent: float) -> np.ndarray:
    w = 1.0 / np.arange(1, n + 1, dtype=np.float64) ** exponent
    return w / w.sum()


@dataclass
class Workload:
    """One named workload.  Tensors are CPU bf16; offsets are int32 cumulative ends."""
    name: str
    x: torch.Tensor                      # [M_total, K] routed activations
    offsets: np.ndarray                  # [E]
    w: Optional[torch.Tensor] = None     # [E, N, K] expert weights
    grad_out: Optional[torch.Tensor] = None  # [M_total, N] (backward workloads)
    fmts: List[int] = field(default_factory=lambda: [0])
    meta: Dict = field(default_factory=dict)

    @property
    def num_groups(self) -> int:
        return int(self.offsets.shape[0])

    @property
    def group_sizes(self) -> np.ndarray:
        return np.diff(np.concatenate([[0], self.offsets.astype(np.int64)]))


def tiny_moe(seed: int = 1001) -> Workload:
    """4 experts, K=256, N=128, 512 routed rows ~N(0,1), one seeded expert empty,
    the other three sizes multinomial(512, uniform); weights ~N(0, 0.02)."""
    g = rng(seed, _T_ROUTE)
    e_total, m_total, k, n = 4, 512, 256, 128
    empty = int(g.integers(0, e_total))
    live = [e for e in range(e_total) if e != empty]
    counts = g.multinomial(m_total, [1.0 / 3] * 3)
    sizes = np.zeros(e_total, np.int64)
    sizes[live] = counts
    x = normal_bf16(seed, _T_X, (m_total, k), 1.0)
    w = normal_bf16(seed, _T_W, (e_total, n, k), 0.02)
    return Workload("tiny_moe_e4_k256_n128_m512", x, offsets_from_sizes(sizes), w=w,
                    meta=dict(E=e_total, K=k, N=n, M=m_total, empty=[empty]))


def llama3_8b_up_proj(seed: int = 1002) -> Workload:
    """Dense Llama3-8B FFN up-projection: one group, X [8192, 4096] ~N(0,1) with a
    seeded 0.1% of entries scaled x100, W [14336, 4096] ~N(0, 0.02)."""
    m, k, n = 8192, 4096, 14336
    g = rng(seed, _T_X)
    xa = g.standard_normal(size=(m, k), dtype=np.float32)
    go = rng(seed, _T_OUTL)
    idx = go.integers(0, m * k, size=(m * k) // 1000)
    flat = xa.reshape(-1)
    flat[idx] *= np.float32(100.0)
    x = to_bf16(xa)
    w = normal_bf16(seed, _T_W, (1, n, k), 0.02)
    return Workload("llama3_8b_ffn_up_m8192_k4096_n14336", x, np.array([m], np.int32), w=w,
                    meta=dict(E=1, K=k, N=n, M=m))


def route_top_k_gumbel(seed: int, tokens: int, experts: int, top_k: int, exponent: float):
    """Per token, top_k DISTINCT experts by Gumbel-top-k over Zipf rank weights;
    ranks are assigned to experts by a seeded permutation.  Returns loads [E]."""
    g = rng(seed, _T_ROUTE)
    perm = g.permutation(experts)
    logw = np.log(zipf_weights(experts, exponent))[np.argsort(perm)]  # weight of expert e
    loads = np.zeros(experts, np.int64)
    chunk = 4096
    for t0 in range(0, tokens, chunk):
        t1 = min(tokens, t0 + chunk)
        gumbel = -np.log(-np.log(g.random((t1 - t0, experts))))
        top = np.argpartition(-(logw[None, :] + gumbel), top_k - 1, axis=1)[:, :top_k]
        loads += np.bincount(top.ravel(), minlength=experts)
    return loads


def deepseek_moe_16b_backward(seed: int = 1003, with_x: bool = True) -> Workload:
    """DeepSeek-MoE-16B-shaped backward: 64 experts, hidden 2048, expert inter 1408,
    16384 tokens top-6 (Gumbel-top-6 on Zipf(1.1)) -> 98304 routed rows.
    grad_out [98304, 1408] ~N(0, 1e-3); X [98304, 2048] ~N(0, 1)."""
    loads = route_top_k_gumbel(seed, 16384, 64, 6, 1.1)
    m = int(loads.sum())
    go = normal_bf16(seed, _T_G, (m, 1408), 1e-3)
    x = normal_bf16(seed, _T_X, (m, 2048), 1.0) if with_x else None
    return Workload("deepseek_moe16b_bwd_e64_h2048_i1408_m98304", x, offsets_from_sizes(loads),
                    grad_out=go, meta=dict(E=64, K=2048, N=1408, M=m))


def zipf_loads(seed: int, m_total: int, experts: int, exponent: float, n_empty: int):
    g = rng(seed, _T_ROUTE)
    empty = sorted(g.choice(experts, size=n_empty, replace=False).tolist()) if n_empty else []
    live = [e for e in range(experts) if e not in empty]
    perm = g.permutation(len(live))
    p = zipf_weights(len(live), exponent)[perm]
    counts = g.multinomial(m_total, p)
    sizes = np.zeros(experts, np.int64)
    sizes[live] = counts
    return sizes, empty


def deepseek_v3_local_experts(seed: int = 1004, with_w: bool = True) -> Workload:
    """DeepSeek-V3-shaped forward on 32 local experts: hidden 7168, expert inter
    2048, 65536 routed rows ~N(0,1); Zipf(1.2) loads with two seeded empty experts
    and some sizes not multiples of 16; W [32, 2048, 7168] ~N(0, 0.02)."""
    sizes, empty = zipf_loads(seed, 65536, 32, 1.2, 2)
    assert any(s % 16 for s in sizes), "workload must hold ragged group sizes"
    x = normal_bf16(seed, _T_X, (65536, 7168), 1.0)
    w = normal_bf16(seed, _T_W, (32, 2048, 7168), 0.02) if with_w else None
    return Workload("deepseek_v3_fwd_e32_k7168_n2048_m65536", x, offsets_from_sizes(sizes), w=w,
                    meta=dict(E=32, K=7168, N=2048, M=65536, empty=empty))


def _outliers_and_zeros(a: np.ndarray, seed: int, tensor_id: int):
    """1e-3 of entries set to +-1e4; 0.5% of rows and of columns set to zero."""
    g = rng(seed, tensor_id * 16 + _T_OUTL)
    flat = a.reshape(-1)
    idx = g.integers(0, flat.size, size=max(1, flat.size // 1000))
    flat[idx] = np.where(g.random(idx.size) < 0.5, -1e4, 1e4).astype(np.float32)
    rows, cols = a.shape[-2], a.shape[-1]
    a2 = a.reshape(-1, cols)
    zr = g.choice(a2.shape[0], size=max(1, a2.shape[0] // 200), replace=False)
    zc = g.choice(cols, size=max(1, cols // 200), replace=False)
    a2[zr, :] = 0.0
    a2[:, zc] = 0.0
    return a


def llama4_sweep(m_total: int, loads: str = "uniform", seed: int = 1005,
                 with_w: bool = True) -> Workload:
    """Llama-4-style MoE: 16 experts, hidden 5120, expert inter 8192; routed rows
    m_total in {4096 ... 131072}; uniform (m/16 each) or Zipf(1.2) loads; inputs
    ~N(0,1) (weights ~N(0,0.02)) with 1e-3 of entries +-1e4 and 0.5% of rows and
    columns all zero.  Quantisation runs under e4m3fn and e4m3fnuz."""
    e, k, n = 16, 5120, 8192
    s = seed + m_total  # distinct stream per sweep point
    if loads == "uniform":
        sizes = np.full(e, m_total // e, np.int64)
    else:
        sizes, _ = zipf_loads(s, m_total, e, 1.2, 0)
    xa = rng(s, _T_X).standard_normal(size=(m_total, k), dtype=np.float32)
    x = to_bf16(_outliers_and_zeros(xa, s, _T_X))
    w = None
    if with_w:
        wa = rng(s, _T_W).standard_normal(size=(e * n, k), dtype=np.float32)
        wa *= np.float32(0.02)
        w = to_bf16(_outliers_and_zeros(wa, s, _T_W)).reshape(e, n, k)
    return Workload(f"llama4_moe_e16_k5120_n8192_m{m_total}_{loads}", x,
                    offsets_from_sizes(sizes), w=w, fmts=[0, 1],
                    meta=dict(E=e, K=k, N=n, M=m_total, loads=loads))


def random_jagged(seed: int, sizes, cols: int, std: float = 1.0, outlier_frac: float = 0.0,
                  zero_cols: int = 0) -> Workload:
    """Small jagged case for parity tests: given group sizes, X [sum, cols]."""
    sizes = np.asarray(sizes, np.int64)
    m = int(sizes.sum())
    g = rng(seed, _T_X)
    a = g.standard_normal(size=(m, cols), dtype=np.float32) * np.float32(std)
    if outlier_frac > 0 and a.size:
        idx = g.integers(0, a.size, size=max(1, int(a.size * outlier_frac)))
        a.reshape(-1)[idx] *= np.float32(100.0)
    if zero_cols and cols:
        a[:, g.choice(cols, size=min(zero_cols, cols), replace=False)] = 0.0
    return Workload(f"random_jagged_{seed}", to_bf16(a), offsets_from_sizes(sizes),
                    meta=dict(M=m, K=cols))
