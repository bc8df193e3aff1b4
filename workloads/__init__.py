"""Seeded synthetic inputs for the expert-parallel MoE dispatch / combine path.

This module only draws inputs. It holds none of the dispatch, layout, quantisation,
combine or exchange arithmetic, so both the CUDA library's tests and the CPU oracle
can take their inputs from here without sharing any of the method's code.

Notation (as on the pages): ``W`` expert-parallel ranks, ``T`` tokens per rank,
``G = W*T`` global tokens (token ``g = r*T + t`` lives on source rank ``r``),
``H`` hidden size, ``E`` experts (``ne = E/W`` per rank), ``K`` experts per token.

All random draws use ``numpy.random.Generator(PCG64(seed))``. bf16 values are held
as their raw 16-bit patterns (``numpy.uint16``); the fp32 -> bf16 cast is torch's
round-to-nearest-even conversion on the CPU.

Workloads (sizes and distributions follow the benchmark configurations):

* ``tiny``   W=4,  T=16,   H=128,  E=8,   K=2, uniform distinct experts, no quant.
* ``cfg2``   W=8,  T=256,  H=4096, E=64,  K=8, uniform distinct experts, no quant.
* ``cfg3``   W=8,  T=4096, H=7168, E=256, K=8, Zipf(1.2) over a seeded expert
             permutation with 8 experts forced to probability 0 (so some experts
             receive no token), 1 % of rows scaled by 100 (outliers), int8 quant.
* ``cfg4``   W=16, T=2048, H=2048, E=128, K=8, uniform distinct, 25 % of tokens
             inactive (Bernoulli(0.75) active mask), fp8-e4m3 quant.
* ``a2a64``  raw uneven all-to-all-v, W=64, splits ~ randint[0, 512) with a seeded
             10 % of entries forced to 0, rows of 4096 bf16 where row k of rank i
             holds 10*i + k.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

QUANT_NONE = 0
QUANT_INT8 = 2
QUANT_FP8_E4M3 = 3


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even) raw bits, via torch's CPU cast."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 raw bits -> fp32 (exact: bf16 is the top half of an fp32)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class MoEWorkload:
    name: str
    W: int
    T: int
    H: int
    E: int
    K: int
    quant_mode: int
    x_bits: np.ndarray              # uint16 [G, H]  (bf16 bits)
    expert_ids: np.ndarray          # int32  [G, K]
    weights: np.ndarray             # fp32   [G, K]  gate weights (expert scales)
    active: Optional[np.ndarray]    # uint8  [G] (tokens) or [G, K] (slots); None = all active
    recipe: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.W * self.T

    @property
    def ne(self) -> int:
        return self.E // self.W

    def n_active_slots(self) -> int:
        if self.active is None:
            return self.G * self.K
        n = int(self.active.astype(np.int64).sum())
        return n * self.K if self.active.ndim == 1 else n

    def token_active(self) -> np.ndarray:
        """uint8 [G]: tokens with at least one active slot."""
        if self.active is None:
            return np.ones(self.G, np.uint8)
        return (self.active if self.active.ndim == 1 else self.active.max(axis=1, initial=0)).astype(np.uint8)

    def rows_cap(self) -> int:
        """Receive capacity for all ranks together: every (token, k) slot may land."""
        return self.G * self.K


def _uniform_distinct(rng: np.random.Generator, G: int, E: int, K: int) -> np.ndarray:
    # K distinct experts per token, uniformly: the K smallest of E iid uniform keys.
    keys = rng.random((G, E))
    return np.argsort(keys, axis=1, kind="stable")[:, :K].astype(np.int32)


def _zipf_distinct(rng: np.random.Generator, G: int, E: int, K: int, s: float,
                   n_zero: int) -> tuple[np.ndarray, np.ndarray]:
    # Zipf(s) popularity over a seeded permutation of the experts; n_zero experts are
    # forced to probability 0. K distinct experts are drawn one after another without
    # replacement (renormalising each time); the Gumbel-top-K draw below samples
    # exactly that sequential process.
    perm = rng.permutation(E)
    p = np.empty(E, dtype=np.float64)
    p[perm] = 1.0 / np.arange(1, E + 1, dtype=np.float64) ** s
    zero = rng.choice(E, size=n_zero, replace=False)
    p[zero] = 0.0
    p /= p.sum()
    with np.errstate(divide="ignore"):
        logp = np.log(p)
    gumbel = -np.log(-np.log(rng.random((G, E))))
    keys = logp[None, :] + gumbel
    ids = np.argsort(-keys, axis=1, kind="stable")[:, :K].astype(np.int32)
    return ids, np.sort(zero)


def _softmax_f32(rng: np.random.Generator, G: int, K: int) -> np.ndarray:
    logits = rng.standard_normal((G, K)).astype(np.float32)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m, dtype=np.float32)
    return (e / e.sum(axis=1, keepdims=True, dtype=np.float32)).astype(np.float32)


MOE_CONFIGS = {
    "tiny": dict(W=4, T=16, H=128, E=8, K=2, quant_mode=QUANT_NONE, routing="uniform"),
    "cfg2": dict(W=8, T=256, H=4096, E=64, K=8, quant_mode=QUANT_NONE, routing="uniform"),
    "cfg3": dict(W=8, T=4096, H=7168, E=256, K=8, quant_mode=QUANT_INT8, routing="zipf",
                 outlier_frac=0.01, outlier_scale=100.0, zipf_s=1.2, zipf_zero=8),
    "cfg4": dict(W=16, T=2048, H=2048, E=128, K=8, quant_mode=QUANT_FP8_E4M3,
                 routing="uniform", active_p=0.75),
}


def moe_workload(name: str = "cfg2", seed: int = 0, **over) -> MoEWorkload:
    """Draw one MoE dispatch/combine workload.

    ``name`` picks a configuration from ``MOE_CONFIGS``; keyword overrides change any
    of its fields (used for small parity cases that span several tiles with a ragged
    tail). Extra override keys: ``routing`` ("uniform" | "zipf" | "dup" — "dup" draws
    experts with replacement, so a token can pick one expert twice), ``active_p``
    (per-token Bernoulli mask [G]), ``slot_active_p`` (per-slot Bernoulli mask [G, K], plus
    5% of tokens with no active slot), ``outlier_frac``, ``outlier_scale``, ``zero_rows``
    (fraction of all-zero rows).
    """
    cfg = dict(MOE_CONFIGS[name])
    cfg.update(over)
    W, T, H, E, K = (int(cfg[k]) for k in ("W", "T", "H", "E", "K"))
    G = W * T
    rng = _rng(seed)
    recipe = dict(cfg)
    recipe["seed"] = seed

    x = rng.standard_normal((G, H), dtype=np.float32)
    of = float(cfg.get("outlier_frac", 0.0))
    if of > 0 and G > 0:
        n_out = max(1, int(round(of * G)))
        rows = rng.choice(G, size=n_out, replace=False)
        x[rows] *= np.float32(cfg.get("outlier_scale", 100.0))
        recipe["outlier_rows"] = int(n_out)
    zr = float(cfg.get("zero_rows", 0.0))
    if zr > 0 and G > 0:
        n_zero = max(1, int(round(zr * G)))
        x[rng.choice(G, size=n_zero, replace=False)] = 0.0
    x_bits = f32_to_bf16_bits(x)

    routing = cfg.get("routing", "uniform")
    if routing == "uniform":
        ids = _uniform_distinct(rng, G, E, K)
    elif routing == "zipf":
        ids, zero = _zipf_distinct(rng, G, E, K, float(cfg.get("zipf_s", 1.2)),
                                   int(cfg.get("zipf_zero", 8)))
        recipe["forced_zero_experts"] = zero.tolist()
    elif routing == "dup":
        ids = rng.integers(0, E, size=(G, K), dtype=np.int64).astype(np.int32)
    else:
        raise ValueError(f"unknown routing {routing!r}")

    w = _softmax_f32(rng, G, K)

    active = None
    ap = cfg.get("active_p")
    if ap is not None:
        active = (rng.random(G) < float(ap)).astype(np.uint8)
    sp = cfg.get("slot_active_p")
    if sp is not None:
        # per-slot mask [G, K]; a seeded 5% of tokens get all K flags false
        active = (rng.random((G, K)) < float(sp)).astype(np.uint8)
        if G > 0:
            active[rng.choice(G, size=max(1, G // 20), replace=False)] = 0

    return MoEWorkload(name=name, W=W, T=T, H=H, E=E, K=K,
                       quant_mode=int(cfg["quant_mode"]), x_bits=x_bits,
                       expert_ids=np.ascontiguousarray(ids, dtype=np.int32),
                       weights=np.ascontiguousarray(w, dtype=np.float32),
                       active=active, recipe=recipe)


def expert_rows(R: int, H: int, seed: int = 1) -> np.ndarray:
    """Synthetic expert outputs for combine: bf16 bits [R, H], N(0,1)."""
    rng = _rng(seed)
    return f32_to_bf16_bits(rng.standard_normal((R, H), dtype=np.float32))


def smooth_scales(E: int, H: int, seed: int = 9) -> np.ndarray:
    """Per-expert smoothing factors for quantisation, fp32 [E, H], log-uniform in
    [1/4, 4)."""
    rng = _rng(seed)
    return np.exp2(rng.uniform(-2.0, 2.0, size=(E, H))).astype(np.float32)


def rmsnorm_inputs(G: int, H: int, seed: int = 7):
    """Inputs of the fused combine + residual + RMSNorm tail: the residual stream as bf16
    bits [G, H], N(0,1), and the RMSNorm weight gamma, fp32 [H], uniform in [0.5, 1.5)."""
    rng = _rng(seed)
    residual = f32_to_bf16_bits(rng.standard_normal((G, H), dtype=np.float32))
    gamma = (0.5 + rng.random(H, dtype=np.float32)).astype(np.float32)
    return residual, gamma


# --------------------------------------------------------------------------------------
# raw uneven all-to-all-v


@dataclass
class A2AWorkload:
    W: int
    row_elems: int                  # bf16 elements per row
    in_splits: np.ndarray           # int64 [W, W]; S[i][j] = rows rank i sends to rank j
    recipe: dict = field(default_factory=dict)

    @property
    def row_bytes(self) -> int:
        return 2 * self.row_elems

    @property
    def cap_in(self) -> int:
        """Rows per sender (every rank padded to the largest send total)."""
        return int(max(1, self.in_splits.sum(axis=1).max())) if self.W else 1

    @property
    def cap_out(self) -> int:
        """Receive capacity per rank (largest receive total)."""
        return int(max(1, self.in_splits.sum(axis=0).max())) if self.W else 1

    def moved_rows(self) -> int:
        return int(self.in_splits.sum())


def a2a_workload(seed: int = 0, W: int = 64, max_split: int = 512, zero_frac: float = 0.10,
                 row_elems: int = 4096) -> A2AWorkload:
    rng = _rng(seed)
    S = rng.integers(0, max_split, size=(W, W), dtype=np.int64)
    if zero_frac > 0:
        S[rng.random((W, W)) < zero_frac] = 0
    return A2AWorkload(W=W, row_elems=row_elems, in_splits=S,
                       recipe=dict(seed=seed, W=W, max_split=max_split,
                                   zero_frac=zero_frac, row_elems=row_elems))


def a2a_label_rows(W: int, cap_in: int, row_elems: int, with_provenance: bool = False) -> np.ndarray:
    """Send buffers [W, cap_in, row_elems] (bf16 bits): row k of rank i holds bf16(10*i+k).

    bf16 holds integers exactly only up to 256, so labels of large (i, k) collide. With
    ``with_provenance`` the first two 16-bit lanes of each row carry the raw i and k
    instead (the exchange copies bytes, so any payload works) so that each received row's
    origin can be read back.
    """
    i = np.arange(W, dtype=np.float32)[:, None]
    k = np.arange(cap_in, dtype=np.float32)[None, :]
    lab = f32_to_bf16_bits(10.0 * i + k)                      # [W, cap_in]
    rows = np.broadcast_to(lab[:, :, None], (W, cap_in, row_elems)).copy()
    if with_provenance and row_elems >= 2:
        rows[:, :, 0] = np.arange(W, dtype=np.uint16)[:, None]
        rows[:, :, 1] = (np.arange(cap_in, dtype=np.int64) & 0xFFFF).astype(np.uint16)[None, :]
    return rows
