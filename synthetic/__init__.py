"""Seeded synthetic inputs for sink-structured FP8 attention.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Both the CPU oracle (in the tests) and the CUDA path
read the E4M3 bytes it returns.

Construction (the attention-sink model of "P-Cast Precision in FP8 Attention:
Sink-Induced Collapse and the Optimality of S=2^8", technical summary,
section 1 and section 2's definitions of Delta and delta_k): the first
``n_sink`` keys have a logit gap Delta over standard-normal non-sink logits.
  * q[..., 0] = sqrt(d); k[..., j, 0] = Delta for j < n_sink, 0 otherwise;
  * every other q and k component i.i.d. N(0, 1);
  * v i.i.d. N(0, 1) (or, with v_mode="mass", v = 1 for non-sink keys and 0
    for sink keys, so each output column reads out the retained non-sink
    probability mass);
  * everything clamped to +-448 and cast to E4M3 by PyTorch's float8_e4m3fn
    conversion (round to nearest even).
Then s_ij = q_i . k_j / sqrt(d) = Delta_eff * [j < n_sink] + N(0, (d-1)/d),
where Delta_eff = e4m3(sqrt(d)) * e4m3(Delta) / sqrt(d) (for d = 128,
e4m3(sqrt(128)) = 11, so Delta_eff = 0.9723 * e4m3(Delta)).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    """One attention problem: shape, sink strength, and the (S, order) cells run on it."""

    name: str
    B: int
    H: int
    Hkv: int
    N: int
    d: int
    causal: bool
    delta: object  # float, or "uniform0-10" for a per-(b, kv-head) draw
    scales: tuple = (256.0,)
    orders: tuple = (1,)  # 0 = forward, 1 = reverse
    n_sink: int = 4
    block_n: int = 128
    sampled_rows: int = 0  # >0: the oracle evaluates this many evenly spaced rows per head
    extra: dict = field(default_factory=dict)

    def flops(self) -> float:
        """Algorithmic FLOPs of one forward pass: 4 * d per visible (query, key) pair."""
        pairs = self.N * (self.N + 1) // 2 if self.causal else self.N * self.N
        return 4.0 * self.d * pairs * self.B * self.H


#: The five workloads: a tiny case with 64-key blocks, the Delta/S sweep shape,
#: the 32K causal prefill, a grouped-query batch and a 128K causal prefill.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 256, 64, False, 7.0, scales=(1.0, 256.0, 448.0),
                     orders=(0, 1), block_n=64),
    "sweep": Workload("sweep", 1, 8, 8, 4096, 128, False, 7.0,
                      scales=tuple([2.0 ** e for e in range(10)] + [448.0]), orders=(0, 1),
                      extra={"deltas": tuple(float(x) for x in range(11))}),
    "prefill32k": Workload("prefill32k", 1, 32, 32, 32768, 128, True, 7.0,
                           scales=(256.0,), orders=(1,), sampled_rows=256),
    "gqa8k": Workload("gqa8k", 4, 32, 8, 8192, 128, True, "uniform0-10",
                      scales=(256.0,), orders=(0, 1), sampled_rows=256),
    "prefill128k": Workload("prefill128k", 1, 32, 8, 131072, 128, True, 8.0,
                            scales=(1.0, 256.0), orders=(0, 1), sampled_rows=256),
}


def sampled_rows(N: int, count: int = 256) -> np.ndarray:
    """Evenly spaced query positions floor((2r + 1) N / (2 count)), r = 0..count-1."""
    r = np.arange(count, dtype=np.int64)
    return ((2 * r + 1) * N // (2 * count)).astype(np.int32)


def _to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    import torch

    t = torch.from_numpy(np.clip(x, -448.0, 448.0))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def sink_deltas(B: int, Hkv: int, delta, rng: np.random.Generator) -> np.ndarray:
    """Per-(b, kv-head) sink strength: a constant, or U[0, 10] draws."""
    if isinstance(delta, str):
        if delta != "uniform0-10":
            raise ValueError(f"unknown delta spec {delta!r}")
        return rng.uniform(0.0, 10.0, size=(B, Hkv)).astype(np.float32)
    return np.full((B, Hkv), float(delta), dtype=np.float32)


def make_inputs(B: int, H: int, Hkv: int, N: int, d: int, delta, seed: int,
                n_sink: int = 4, v_mode: str = "normal"):
    """E4M3 bytes q [B,H,N,d], k [B,Hkv,N,d], v [B,Hkv,N,d] and the per-(b, kv-head) Delta.

    Draw order (fixed, so a seed always gives the same bytes): Delta (if
    random), then q, k, v, each one standard-normal array in C order.
    """
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    rng = np.random.Generator(np.random.PCG64(seed))
    deltas = sink_deltas(B, Hkv, delta, rng)
    q = rng.standard_normal((B, H, N, d), dtype=np.float32)
    q[..., 0] = math.sqrt(d)
    qb = _to_e4m3_bytes(q)
    del q
    k = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    k[..., 0] = 0.0
    k[:, :, :n_sink, 0] = deltas[:, :, None]
    kb = _to_e4m3_bytes(k)
    del k
    if v_mode == "normal":
        v = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    elif v_mode == "mass":
        v = np.ones((B, Hkv, N, d), dtype=np.float32)
        v[:, :, :n_sink, :] = 0.0
    else:
        raise ValueError(f"unknown v_mode {v_mode!r}")
    vb = _to_e4m3_bytes(v)
    del v
    return qb, kb, vb, deltas


def workload_inputs(w: Workload, seed: int, delta=None, v_mode: str = "normal"):
    """Inputs for a workload (``delta`` overrides the workload's sink strength)."""
    return make_inputs(w.B, w.H, w.Hkv, w.N, w.d, w.delta if delta is None else delta,
                       seed, n_sink=w.n_sink, v_mode=v_mode)


def _to_bf16_values(x: np.ndarray) -> np.ndarray:
    """float32 values rounded to bfloat16 (PyTorch's conversion, round to nearest even)."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def make_wide_inputs(B: int, H: int, Hkv: int, N: int, d: int, delta, seed: int,
                     n_sink: int = 4, outliers: int = 0, outlier_gain: float = 16.0):
    """Unquantised inputs for the quantisation path: float32 arrays holding bfloat16 values.

    Same sink construction as ``make_inputs`` (q[..., 0] = sqrt(d), sink keys
    k[..., 0] = Delta), without the E4M3 cast.  ``outliers`` > 0 multiplies
    that many fixed channels (1 .. outliers) of q and k by ``outlier_gain``,
    the kind of outlier channel that makes a direct per-block cast lose
    precision on every other channel.  Draw order: Delta, q, k, v.
    """
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    rng = np.random.Generator(np.random.PCG64(seed))
    deltas = sink_deltas(B, Hkv, delta, rng)
    q = rng.standard_normal((B, H, N, d), dtype=np.float32)
    q[..., 0] = math.sqrt(d)
    k = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    k[..., 0] = 0.0
    k[:, :, :n_sink, 0] = deltas[:, :, None]
    if outliers:
        q[..., 1:1 + outliers] *= outlier_gain
        k[..., 1:1 + outliers] *= outlier_gain
    v = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    return _to_bf16_values(q), _to_bf16_values(k), _to_bf16_values(v), deltas


def make_output_grad(shape, seed: int) -> np.ndarray:
    """A seeded output gradient dO: standard-normal float32 values rounded to bfloat16."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return _to_bf16_values(rng.standard_normal(shape, dtype=np.float32))


def hadamard_signs(d: int, seed: int) -> np.ndarray:
    """The random +-1 column signs of the rotation (float32 [d]), from a seeded generator."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.where(rng.random(d) < 0.5, -1.0, 1.0).astype(np.float32)
