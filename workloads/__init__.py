"""Seeded synthetic MoE routing workloads: inputs only.

This module draws the inputs of the dispatch/combine path -- hidden states
``x``, top-k expert ids ``idx`` and gate weights ``w`` -- with the shapes and
distributions of the DeepEP workloads (DeepSeek-V3-shaped: hidden 7168,
256 routed experts, top-8; plus a small case, a 128-token decode batch, a
Zipf-skewed batch and a large 32K-token batch).  It also holds the stand-in
"experts" that turn dispatched rows into expert outputs ``y`` for combine.

It contains none of the dispatch/combine arithmetic (no layout, no
permutation, no FP8 cast, no weighted reduction); both the CPU oracle and the
CUDA path consume what it produces.  Every draw comes from one
``numpy.random.default_rng(seed)`` stream in a fixed order, so a
(config, seed, size override) triple always gives the same bytes.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np
import torch

__all__ = ["Config", "Batch", "CONFIGS", "make_batch", "expert_outputs",
           "row_experts"]


@dataclasses.dataclass(frozen=True)
class Config:
    """One workload shape.

    T tokens of hidden size H, E experts split into R logical ranks of
    G = E // R consecutive experts, top-k routing.
    """
    name: str
    T: int
    H: int
    E: int
    R: int
    k: int
    routing: str            # "uniform" | "group_limited" | "zipf"
    dispatch: Tuple[str, ...]  # subset of ("bf16", "fp8")
    expert: str             # stand-in expert: "identity" | "scale"
    topk_groups: int = 0    # group-limited routing: groups kept per token
    zipf_s: float = 0.0     # Zipf exponent of the skewed popularity


CONFIGS = {
    # 128 tokens, hidden 256, 16 experts in 4 ranks, top-4: the small case.
    "tiny": Config("tiny", 128, 256, 16, 4, 4, "uniform", ("bf16",), "identity"),
    # 128-token decode batch, DeepSeek-V3 shape, FP8 dispatch.
    "decode": Config("decode", 128, 7168, 256, 8, 8, "uniform", ("fp8",),
                     "identity"),
    # 4096-token prefill batch with group-limited gating (8 groups of 32,
    # top-4 groups), bf16 and FP8 dispatch.
    "prefill": Config("prefill", 4096, 7168, 256, 8, 8, "group_limited",
                      ("bf16", "fp8"), "identity", topk_groups=4),
    # 8192 tokens with Zipf(1.2) expert popularity, FP8 dispatch.
    "skewed": Config("skewed", 8192, 7168, 256, 8, 8, "zipf", ("fp8",),
                     "identity", zipf_s=1.2),
    # 32768 tokens, hidden 4096, 128 experts in 16 ranks; experts scale
    # their input by (1 + 0.01 * expert id) so combine's weighting shows.
    "large": Config("large", 32768, 4096, 128, 16, 8, "uniform", ("bf16",),
                    "scale"),
}


@dataclasses.dataclass
class Batch:
    """Host (CPU) tensors of one routed batch."""
    cfg: Config
    seed: int
    x: torch.Tensor     # [T, H] bfloat16
    idx: torch.Tensor   # [T, k] int64, expert ids (-1 = dropped slot)
    w: torch.Tensor     # [T, k] float32 gate weights

    @property
    def T(self) -> int:
        return self.x.shape[0]

    @property
    def H(self) -> int:
        return self.x.shape[1]


def _softmax_rows(logits: np.ndarray) -> np.ndarray:
    z = logits.astype(np.float64)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def _uniform_distinct(rng, T, E, k):
    # k distinct ids per token, uniformly: the first k of a random ordering.
    keys = rng.random((T, E))
    return np.argsort(keys, axis=1, kind="stable")[:, :k]


def _group_limited(rng, T, E, R, k, topk_groups):
    # DeepSeek-V3 style: sigmoid scores, groups ranked by their best expert,
    # the top groups kept, then the top-k experts among the kept groups.
    # Ties go to the lower index (stable sorts).  Weights = s / sum(s).
    G = E // R
    s = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, E))))
    s = s.astype(np.float32)
    gscore = s.reshape(T, R, G).max(axis=2)
    groups = np.argsort(-gscore, axis=1, kind="stable")[:, :topk_groups]
    keep = np.zeros((T, R), dtype=bool)
    np.put_along_axis(keep, groups, True, axis=1)
    masked = np.where(np.repeat(keep, G, axis=1), s, -np.inf)
    idx = np.argsort(-masked, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(s, idx, axis=1).astype(np.float64)
    w = (sel / sel.sum(axis=1, keepdims=True)).astype(np.float32)
    return idx, w


def _zipf(rng, T, E, k, s_exp):
    # Popularity p[perm[i]] ~ (1 + i)^-s over a seeded permutation of the
    # experts; k ids per token without replacement via Gumbel-top-k.
    perm = rng.permutation(E)
    p = np.empty(E)
    p[perm] = (1.0 + np.arange(E)) ** (-s_exp)
    p /= p.sum()
    keys = np.log(p)[None, :] + rng.gumbel(size=(T, E))
    return np.argsort(-keys, axis=1, kind="stable")[:, :k]


def make_batch(cfg: Config | str, seed: int = 0, T: Optional[int] = None,
               H: Optional[int] = None, drop_frac: float = 0.0,
               dup_frac: float = 0.0) -> Batch:
    """Draw one batch of ``cfg`` (optionally with T or H overridden).

    drop_frac: fraction of slots set to -1 (dropped, e.g. by a capacity cap).
    dup_frac:  fraction of tokens whose slot 1 repeats slot 0's expert.
    Both default to 0, which gives the workloads as specified.
    """
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    T = cfg.T if T is None else int(T)
    H = cfg.H if H is None else int(H)
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H), dtype=np.float32)
    if cfg.routing == "uniform":
        idx = _uniform_distinct(rng, T, cfg.E, cfg.k)
        w = _softmax_rows(rng.standard_normal((T, cfg.k), dtype=np.float32))
    elif cfg.routing == "group_limited":
        idx, w = _group_limited(rng, T, cfg.E, cfg.R, cfg.k, cfg.topk_groups)
    elif cfg.routing == "zipf":
        idx = _zipf(rng, T, cfg.E, cfg.k, cfg.zipf_s)
        w = _softmax_rows(rng.standard_normal((T, cfg.k), dtype=np.float32))
    else:
        raise ValueError(f"unknown routing {cfg.routing!r}")
    idx = idx.astype(np.int64)
    if dup_frac > 0 and cfg.k > 1 and T > 0:
        dup = rng.random(T) < dup_frac
        idx[dup, 1] = idx[dup, 0]
    if drop_frac > 0 and T > 0:
        idx[rng.random(idx.shape) < drop_frac] = -1
    return Batch(cfg=cfg, seed=seed,
                 x=torch.from_numpy(x).to(torch.bfloat16),
                 idx=torch.from_numpy(np.ascontiguousarray(idx)),
                 w=torch.from_numpy(np.ascontiguousarray(w)))


def row_experts(off_e: torch.Tensor, n_rows: int) -> torch.Tensor:
    """Expert that owns each receive row, given expert offsets off_e[E+1]
    (rows past off_e[E] get -1)."""
    off = off_e.to(torch.int64)
    rows = torch.arange(n_rows, dtype=torch.int64, device=off.device)
    e = torch.searchsorted(off[1:], rows, right=True)
    return torch.where(rows < off[-1], e, torch.full_like(e, -1))


def expert_outputs(x: torch.Tensor, recv_src: torch.Tensor,
                   off_e: torch.Tensor, kind: str) -> torch.Tensor:
    """Stand-in expert outputs y [N, H] bf16 for combine.

    Row r holds expert e = row_experts(off_e)[r] applied to its source token
    x[recv_src[r]]:  "identity" -> x[src];  "scale" -> bf16(x[src] * (1 +
    0.01 e)) with the factor formed in fp32.  Rows without a source are 0.
    Works on whichever device the tensors live on.
    """
    src = recv_src.to(torch.int64)
    n = src.numel()
    y = torch.zeros((n, x.shape[1]), dtype=torch.bfloat16, device=x.device)
    if kind not in ("identity", "scale"):
        raise ValueError(f"unknown expert kind {kind!r}")
    e_all = row_experts(off_e.to(x.device), n) if kind == "scale" else None
    step = 1 << 16  # rows per chunk: bounds the fp32 temporaries
    for r0 in range(0, n, step):
        s = src[r0:r0 + step]
        valid = s >= 0
        if not bool(valid.any()):
            continue
        rows = x[s[valid]]
        if kind == "identity":
            y[r0:r0 + step][valid] = rows
        else:
            f = 1.0 + 0.01 * e_all[r0:r0 + step][valid].to(torch.float32)
            y[r0:r0 + step][valid] = (rows.to(torch.float32) * f[:, None]).to(torch.bfloat16)
    return y
