"""Seeded synthetic inputs for the KDA chunked forward.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
bench. It holds no arithmetic of the method itself (no recurrence, no chunking,
no decay products): it only draws random tensors with the distributions of the
workloads and stores them in the formats the library consumes.

Formats
-------
* ``q``, ``k``, ``v``: bf16 stored as ``uint16`` bit patterns, shape ``[T, H, d]``.
* ``g``: float32 natural-log decay per key channel, shape ``[T, H, dk]``.
* ``beta``: float32, shape ``[T, H]``.
* ``cu_seqlens``: int32, shape ``[num_seqs + 1]`` (FlashAttention convention).
* ``initial_state``: float32 ``[num_seqs, H, dk, dv]`` or ``None`` (zero state).

Distributions (the workloads of the KDA prefill benchmarks)
----------------------------------------------------------
* q, k ~ N(0, 1) in float32, L2-normalised over the head dimension per
  (token, head) in float32, then rounded to bf16 (round to nearest even).
* v ~ N(0, 1), rounded to bf16.
* g = clamp(logsigmoid(x), -5, 0) with x ~ N(gate_mean, gate_std^2); the clamp
  is the gate lower bound of -5 that FlashKDA uses (page "Kimi K3 开源满月…",
  section "KDA 内核到底难在哪"). logsigmoid is evaluated stably in float64, then
  rounded to float32.
* beta = sigmoid(N(0, 1)) in float32.
* initial states ~ N(0, 0.1^2) float32 when requested.

Every tensor draws from its own Philox-4x64 counter-based stream keyed by
``(seed, tensor id)``, so a tensor never depends on the order in which the
others were generated.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

# Philox stream ids, one per tensor.
_STREAM = {"q": 1, "k": 2, "v": 3, "g": 4, "beta": 5, "init": 6, "perm": 7}

GATE_LOWER_BOUND = -5.0


def _rng(seed: int, name: str) -> np.random.Generator:
    key = np.array([seed & 0xFFFFFFFFFFFFFFFF, _STREAM[name]], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bit patterns.

    NaN inputs are kept NaN (quiet); the generator never produces them.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding_bias = ((u >> 16) & 1) + 0x7FFF
    r = ((u + rounding_bias) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class KDAInputs:
    q: np.ndarray            # uint16 [T, H, dk] (bf16 bits)
    k: np.ndarray            # uint16 [T, H, dk]
    v: np.ndarray            # uint16 [T, H, dv]
    g: np.ndarray            # float32 [T, H, dk]
    beta: np.ndarray         # float32 [T, H]
    cu_seqlens: np.ndarray   # int32 [N + 1]
    initial_state: Optional[np.ndarray]  # float32 [N, H, dk, dv] or None
    scale: float
    seed: int
    # The raw draws behind q, k, g and beta (make_inputs(..., raw=True)), for
    # the fused-preprocessing entry point: q, k before normalisation (bf16
    # bits), the gate logits x and the beta logits (float32).
    q_raw: Optional[np.ndarray] = None
    k_raw: Optional[np.ndarray] = None
    g_logit: Optional[np.ndarray] = None
    beta_logit: Optional[np.ndarray] = None

    @property
    def total_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def num_heads(self) -> int:
        return int(self.q.shape[1])

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def seqlens(self) -> list:
        return [int(x) for x in np.diff(self.cu_seqlens)]


def _normal(seed: int, name: str, shape, dtype=np.float32) -> np.ndarray:
    return _rng(seed, name).standard_normal(size=shape, dtype=dtype)


def _l2_normalise_f32(x: np.ndarray) -> np.ndarray:
    # float32 throughout, normalised over the last axis (the head dimension).
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32))
    return (x / np.maximum(n, np.float32(1e-6))).astype(np.float32)


def _logsigmoid_f64(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    # log(sigmoid(x)) = -log1p(exp(-x)) for x >= 0, x - log1p(exp(x)) for x < 0.
    return np.where(x >= 0, -np.log1p(np.exp(-np.abs(x))), x - np.log1p(np.exp(-np.abs(x))))


def make_inputs(seqlens: Sequence[int], num_heads: int, seed: int, *, dk: int = 128,
                dv: int = 128, gate_mean: float = 3.0, gate_std: float = 1.5,
                random_initial_state: bool = False, init_std: float = 0.1,
                scale: Optional[float] = None, row_block: int = 1 << 20, raw: bool = False) -> KDAInputs:
    """Draw one packed (varlen) batch.

    ``row_block`` bounds the float32 temporaries (tokens drawn per step); the
    values do not depend on it because each tensor's Philox stream is consumed
    in row order. ``raw`` also keeps the draws before normalisation and
    activation (``q_raw``, ``k_raw`` rounded to bf16; ``g_logit`` and
    ``beta_logit`` in float32); the other tensors are the same either way.
    """
    seqlens = [int(s) for s in seqlens]
    if any(s < 0 for s in seqlens):
        raise ValueError("sequence lengths must be >= 0")
    T = int(sum(seqlens))
    H = int(num_heads)
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(seqlens, dtype=np.int64))
    if scale is None:
        scale = 1.0 / float(np.sqrt(dk))

    q = np.empty((T, H, dk), dtype=np.uint16)
    k = np.empty((T, H, dk), dtype=np.uint16)
    v = np.empty((T, H, dv), dtype=np.uint16)
    g = np.empty((T, H, dk), dtype=np.float32)
    rq, rk, rv, rg = (_rng(seed, n) for n in ("q", "k", "v", "g"))
    if raw:
        q_raw = np.empty((T, H, dk), dtype=np.uint16)
        k_raw = np.empty((T, H, dk), dtype=np.uint16)
        g_logit = np.empty((T, H, dk), dtype=np.float32)
    for t0 in range(0, T, row_block):
        t1 = min(T, t0 + row_block)
        n = t1 - t0
        dq = rq.standard_normal((n, H, dk), dtype=np.float32)
        dkk = rk.standard_normal((n, H, dk), dtype=np.float32)
        q[t0:t1] = f32_to_bf16_bits(_l2_normalise_f32(dq))
        k[t0:t1] = f32_to_bf16_bits(_l2_normalise_f32(dkk))
        v[t0:t1] = f32_to_bf16_bits(rv.standard_normal((n, H, dv), dtype=np.float32))
        x = rg.standard_normal((n, H, dk), dtype=np.float32).astype(np.float64) * gate_std + gate_mean
        g[t0:t1] = np.clip(_logsigmoid_f64(x), GATE_LOWER_BOUND, 0.0).astype(np.float32)
        if raw:
            q_raw[t0:t1] = f32_to_bf16_bits(dq)
            k_raw[t0:t1] = f32_to_bf16_bits(dkk)
            g_logit[t0:t1] = x.astype(np.float32)
    xb = _normal(seed, "beta", (T, H)).astype(np.float64)
    beta = (1.0 / (1.0 + np.exp(-xb))).astype(np.float32)
    init = None
    if random_initial_state:
        init = (_normal(seed, "init", (len(seqlens), H, dk, dv)) * np.float32(init_std)).astype(np.float32)
    out = KDAInputs(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu, initial_state=init,
                    scale=float(scale), seed=int(seed))
    if raw:
        out.q_raw, out.k_raw, out.g_logit = q_raw, k_raw, g_logit
        out.beta_logit = xb.astype(np.float32)
    return out


# ---------------------------------------------------------------------------
# The five benchmark workloads (d = dk = dv = 128).
# ---------------------------------------------------------------------------
MIXED_LENGTHS = (37, 130, 250, 511, 2048, 3000, 4096, 8192)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seqlens: tuple
    num_heads: int
    random_initial_state: bool
    gate_mean: float = 3.0
    gate_std: float = 1.5
    seed: int = 0
    description: str = ""

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    def make(self, seed: Optional[int] = None, **kw) -> KDAInputs:
        return make_inputs(self.seqlens, self.num_heads, self.seed if seed is None else seed,
                           gate_mean=self.gate_mean, gate_std=self.gate_std,
                           random_initial_state=self.random_initial_state, **kw)


def _mixed_order(seed: int) -> tuple:
    perm = _rng(seed, "perm").permutation(len(MIXED_LENGTHS))
    return tuple(int(MIXED_LENGTHS[i]) for i in perm)


WORKLOADS = {
    1: Workload("tiny_fixed_T256_H2", (256,), 2, False, seed=1001,
                description="B=1, T=256, H=2, zero initial state"),
    2: Workload("kimi_linear_fixed_T8192_H32", (8192,), 32, False, seed=1002,
                description="B=1, T=8192, H=32, zero initial state"),
    3: Workload("uniform_varlen_8x1024_H32", (1024,) * 8, 32, True, seed=1003,
                description="8 x 1024 packed via cu_seqlens, H=32, random initial states"),
    4: Workload("mixed_varlen_T18264_H32", _mixed_order(1004), 32, True, seed=1004,
                description="lengths {37,130,250,511,2048,3000,4096,8192} in seeded order, H=32"),
    5: Workload("long_context_T131072_H8", (131072,), 8, True, gate_mean=4.0, gate_std=1.0,
                seed=1005, description="B=1, T=131072, H=8, x~N(4,1) gate, random initial state"),
}


# One decode step of a serving batch: 256 requests with one token each against
# resident per-request states (random, like the prefill workloads' initial
# states), H=32 (the Kimi-Linear-shaped head count of the prefill workloads).
DECODE = Workload("decode_B256_H32", (1,) * 256, 32, True, seed=1006,
                  description="decode step: 256 requests x 1 token, H=32, resident random states")


def workload(n: int) -> Workload:
    return WORKLOADS[int(n)]
