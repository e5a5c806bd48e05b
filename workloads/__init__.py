"""Seeded synthetic inputs for MoE token dispatch / combine.

This module only draws inputs: hidden states, routing (``topk_idx``) and gate
weights (``topk_weights``).  It holds none of the dispatch / combine arithmetic,
so both the CPU oracle and the CUDA path can take their inputs from here
without sharing any code with one another.

Workloads follow the settings the DeepEP pages describe:

* "DeepSeek 开源周第二弹：DeepEP" (m.youleyou.com), section "DeepEP 的常规内核和低延迟内核":
  normal kernels tested with 4096 tokens per batch, hidden 7168, top-4 groups,
  top-8 experts, FP8 dispatch and BF16 combine; low-latency kernels with 128
  tokens per batch, hidden 7168, top-8, FP8 dispatch and BF16 combine.
* "DeepEP 项目开源" (deepseek.csdn.net), section "推理解码阶段的应用": the
  low-latency buffer holds ``num_max_tokens * hidden * num_experts`` elements,
  i.e. a capacity of ``num_max_tokens`` rows per expert.
* "deepseek-ai/DeepEP" (agentlenshq.com), section "主要特性": redundant
  experts (replicas of hot experts).

The five named workloads:

======== ====== ====== == ============ =================================== =====
name     T      H      K  E / P        routing                             quant
======== ====== ====== == ============ =================================== =====
ll       128    7168   8  256 / 8      8 distinct experts, uniform          fp8
normal   4096   7168   8  256 / 8      group-limited (top-4 of 8 groups)    fp8
skew     4096   7168   8  256 / 8      Zipf(1.2) without replacement, 5%    fp8
                                        of slots masked (-1)
bf16     8192   4096   6  64 / 16      6 distinct experts, uniform, 1% of  none
                                        rows scaled x100 (outliers)
stress   32768  7168   8  288 / 8      group-limited on 256 experts + 32    fp8
                                        replica slots of the 32 hottest
======== ====== ====== == ============ =================================== =====

Hidden states are BF16 draws of N(0, 1) (the float32 draw is rounded to BF16
by torch's own cast).  Gate weights are float32.  ``topk_idx`` is int64, the
dtype ``torch.topk`` returns.

Every array is produced on the host from ``numpy.random.default_rng(seed)``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "make_workload",
    "make_custom",
    "random_bf16",
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
]


@dataclass
class Workload:
    """One batch of dispatch / combine inputs (host numpy arrays)."""

    name: str
    num_tokens: int
    hidden: int
    num_topk: int
    num_experts: int
    num_partitions: int
    quant: str  # "fp8" (e4m3, 1x128 scales) or "none" (BF16 copy)
    x: np.ndarray  # uint16 [T, H], BF16 bit patterns
    topk_idx: np.ndarray  # int64 [T, K], -1 = masked
    topk_weights: np.ndarray  # float32 [T, K]
    num_max_tokens: int = 0  # low-latency capacity per expert (0: not a low-latency workload)
    seed: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def experts_per_partition(self) -> int:
        return self.num_experts // self.num_partitions


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round float32 to BF16 with torch's cast; return the uint16 bit patterns."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def random_bf16(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    """BF16 draws of N(0, scale^2) as uint16 bit patterns."""
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return bf16_bits_from_f32(a)


def _softmax_weights(rng: np.random.Generator, T: int, K: int) -> np.ndarray:
    logits = rng.standard_normal(size=(T, K), dtype=np.float32).astype(np.float64)
    logits -= logits.max(axis=1, keepdims=True)
    e = np.exp(logits)
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def _uniform_distinct(rng: np.random.Generator, T: int, K: int, E: int) -> np.ndarray:
    """K distinct experts per token, uniformly at random (random order)."""
    keys = rng.random(size=(T, E))
    return np.argsort(keys, axis=1, kind="stable")[:, :K].astype(np.int64)


def _group_limited(rng: np.random.Generator, T: int, E: int = 256, groups: int = 8,
                   topk_groups: int = 4, K: int = 8):
    """Group-limited routing: sigmoid affinities, top-4 of 8 groups, then top-8 experts.

    Group score = sum of the two largest affinities in the group.  Ties go to
    the lower index (stable sorts).  Weights are the chosen affinities
    normalised to sum to one.
    """
    logits = rng.standard_normal(size=(T, E), dtype=np.float32)
    s = (1.0 / (1.0 + np.exp(-logits.astype(np.float64)))).astype(np.float32)
    per = E // groups
    sg = s.reshape(T, groups, per)
    top2 = -np.sort(-sg, axis=2, kind="stable")[:, :, :2].sum(axis=2)
    keep = np.argsort(-top2, axis=1, kind="stable")[:, :topk_groups]
    mask = np.zeros((T, groups), dtype=bool)
    np.put_along_axis(mask, keep, True, axis=1)
    masked = np.where(np.repeat(mask, per, axis=1), s, -np.inf)
    idx = np.argsort(-masked, axis=1, kind="stable")[:, :K]
    sel = np.take_along_axis(s, idx, axis=1).astype(np.float64)
    w = (sel / sel.sum(axis=1, keepdims=True)).astype(np.float32)
    return idx.astype(np.int64), w


def _zipf_routing(rng: np.random.Generator, T: int, K: int, E: int, s: float):
    ranks = np.arange(1, E + 1, dtype=np.float64)
    p = ranks ** (-s)
    p /= p.sum()
    rank_to_expert = rng.permutation(E)
    idx = np.empty((T, K), dtype=np.int64)
    for t in range(T):
        idx[t] = rank_to_expert[rng.choice(E, K, replace=False, p=p)]
    return idx


def _build(name, seed, T, H, K, E, P, quant, x, idx, w, cap=0, **meta) -> Workload:
    return Workload(name=name, num_tokens=T, hidden=H, num_topk=K, num_experts=E,
                    num_partitions=P, quant=quant, x=x, topk_idx=np.ascontiguousarray(idx),
                    topk_weights=np.ascontiguousarray(w, dtype=np.float32),
                    num_max_tokens=cap, seed=seed, meta=meta)


def _ll(seed: int, T: Optional[int], H: Optional[int]) -> Workload:
    rng = np.random.default_rng(seed)
    T = 128 if T is None else T
    H = 7168 if H is None else H
    K, E, P = 8, 256, 8
    x = random_bf16(rng, (T, H))
    idx = _uniform_distinct(rng, T, K, E)
    w = _softmax_weights(rng, T, K)
    return _build("ll", seed, T, H, K, E, P, "fp8", x, idx, w, cap=max(T, 128))


def _normal(seed: int, T: Optional[int], H: Optional[int]) -> Workload:
    rng = np.random.default_rng(seed)
    T = 4096 if T is None else T
    H = 7168 if H is None else H
    x = random_bf16(rng, (T, H))
    idx, w = _group_limited(rng, T)
    return _build("normal", seed, T, H, 8, 256, 8, "fp8", x, idx, w)


def _skew(seed: int, T: Optional[int], H: Optional[int]) -> Workload:
    rng = np.random.default_rng(seed)
    T = 4096 if T is None else T
    H = 7168 if H is None else H
    K, E, P = 8, 256, 8
    x = random_bf16(rng, (T, H))
    idx = _zipf_routing(rng, T, K, E, 1.2)
    w = _softmax_weights(rng, T, K)
    n_mask = int(round(0.05 * T * K))
    flat = rng.choice(T * K, n_mask, replace=False)
    idx.reshape(-1)[flat] = -1
    return _build("skew", seed, T, H, K, E, P, "fp8", x, idx, w, num_masked=n_mask)


def _bf16(seed: int, T: Optional[int], H: Optional[int]) -> Workload:
    rng = np.random.default_rng(seed)
    T = 8192 if T is None else T
    H = 4096 if H is None else H
    K, E, P = 6, 64, 16
    a = rng.standard_normal(size=(T, H), dtype=np.float32)
    n_out = max(1, int(round(0.01 * T)))
    rows = rng.choice(T, n_out, replace=False)
    a[rows] *= np.float32(100.0)
    x = bf16_bits_from_f32(a)
    idx = _uniform_distinct(rng, T, K, E)
    w = _softmax_weights(rng, T, K)
    return _build("bf16", seed, T, H, K, E, P, "none", x, idx, w, outlier_rows=np.sort(rows))


def _stress(seed: int, T: Optional[int], H: Optional[int]) -> Workload:
    rng = np.random.default_rng(seed)
    T = 32768 if T is None else T
    H = 7168 if H is None else H
    K, P = 8, 8
    x = random_bf16(rng, (T, H))
    logical, w = _group_limited(rng, T)
    # 256 logical experts -> 288 slots: 8 partitions x (32 primaries + 4 replicas).
    counts = np.bincount(logical.reshape(-1), minlength=256)
    hottest = np.argsort(-counts, kind="stable")[:32]
    slot = (np.arange(256) // 32) * 36 + np.arange(256) % 32
    replica = np.full(256, -1, dtype=np.int64)
    for i, e in enumerate(hottest):
        replica[e] = (i % 8) * 36 + 32 + i // 8
    idx = slot[logical]
    use_replica = (replica[logical] >= 0) & ((np.arange(T) % 2)[:, None] == 1)
    idx = np.where(use_replica, replica[logical], idx).astype(np.int64)
    # slot -> the slot holding its expert's primary copy (primaries name themselves)
    primary_of = np.empty(288, dtype=np.int32)
    primary_of[slot] = slot
    primary_of[replica[hottest]] = slot[hottest]
    return _build("stress", seed, T, H, K, 288, P, "fp8", x, idx, w, hottest=hottest,
                  logical_idx=logical, primary_of=primary_of)


WORKLOADS = {
    "ll": _ll,
    "normal": _normal,
    "skew": _skew,
    "bf16": _bf16,
    "stress": _stress,
}


def make_workload(name: str, seed: int = 0, num_tokens: Optional[int] = None,
                  hidden: Optional[int] = None) -> Workload:
    """Draw one named workload.  ``num_tokens`` / ``hidden`` shrink it for tests."""
    if name not in WORKLOADS:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}")
    return WORKLOADS[name](seed, num_tokens, hidden)


def make_custom(num_tokens: int, hidden: int, num_topk: int, num_experts: int,
                num_partitions: int, seed: int = 0, quant: str = "fp8",
                mask_frac: float = 0.0, duplicates: bool = False,
                hot_expert: Optional[int] = None, x_scale: float = 1.0,
                num_max_tokens: int = 0) -> Workload:
    """A free-form workload for edge cases (ragged sizes, masks, duplicates, empties).

    ``duplicates`` draws experts with replacement (one token may name an expert
    twice).  ``hot_expert`` sends every token's first choice to that expert.
    """
    rng = np.random.default_rng(seed)
    T, H, K, E = num_tokens, hidden, num_topk, num_experts
    x = random_bf16(rng, (T, H), scale=x_scale)
    if duplicates or K > E:
        idx = rng.integers(0, E, size=(T, K), dtype=np.int64)
    else:
        idx = _uniform_distinct(rng, T, K, E) if T > 0 else np.zeros((0, K), np.int64)
    if hot_expert is not None and T > 0:
        # keep the row distinct unless duplicates were asked for
        for t in range(T):
            if not duplicates and hot_expert in idx[t]:
                j = int(np.nonzero(idx[t] == hot_expert)[0][0])
                idx[t, j] = idx[t, 0]
            idx[t, 0] = hot_expert
    w = _softmax_weights(rng, T, K) if T > 0 else np.zeros((0, K), np.float32)
    if mask_frac > 0 and T > 0:
        n = int(round(mask_frac * T * K))
        flat = rng.choice(T * K, n, replace=False)
        idx.reshape(-1)[flat] = -1
    return _build("custom", seed, T, H, K, E, num_partitions, quant, x, idx, w,
                  cap=num_max_tokens)
