"""Seeded synthetic inputs for the DiT-MoE sparse expert layer.

This module is the single source of inputs for both sides of every parity
check: the CUDA path and the fp64 oracle.  It holds no arithmetic of the
method itself (no routing, no softmax, no expert MLP); it only draws
numbers and lays them out.

Recipe (the same for every workload):

* ``numpy.random.Generator(PCG64(seed))``; every array is drawn as fp64
  standard normals, scaled by its standard deviation, cast to fp32, and for
  bf16 (fp16) workloads rounded to the nearest bf16 (fp16) value, ties to even.  The
  returned arrays are fp32 whose values are exactly representable in the
  workload's storage type, so both sides read identical numbers.
* Draw order: x, Wg, W1 (E,H,D), W2 (E,D,H), shared W1 (n_s,H,D), shared
  W2 (n_s,D,H), router bias (only for the ``normal`` bias recipe), then the
  optional expert biases b1, b2, shared b1, shared b2.
* x ~ N(0, 1); Wg, W1 ~ N(0, 1/D); W2 ~ N(0, 1/H) (fan-in scaling); expert
  biases are zero unless ``bias_std`` is given (tests use it to exercise the
  bias terms of nn.Linear-style experts).
* Router bias (not on the pages; a synthetic device to skew expert load):
  ``zipf`` gives b_i = ln(z_i) with z_i proportional to i^-1.2 (i = 1..E),
  normalised; ``normal`` gives b_i ~ N(0, variance 0.5).

Workload shapes follow the DiT-MoE model table (hub page, model list: S/B/XL
with 8 or 16 experts, 2 active) and the DiT size table (DiT page, "model
scale": D = 384 / 768 / 1152, mlp ratio 4, 256 tokens per image at 256x256
and 1024 at 512x512 with p = 2).  They stand in for ImageNet latents, which
are not available here.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens in one call (batch x tokens per image)
    D: int            # model width
    H: int            # expert MLP hidden width
    E: int            # routed experts
    K: int            # experts per token (race: average, S = K*T)
    n_shared: int     # shared experts every token visits
    dtype: str        # "f32", "bf16" or "f16" (storage type of activations and weights)
    routing: str      # "topk" or "race"
    alpha: float      # balance-loss factor
    seed: int
    router_bias: str  # "none", "zipf", "normal"
    batch: int
    tokens_per_image: int

    def with_tokens(self, T: int) -> "Workload":
        return replace(self, T=T)


# The five layer workloads.  Seeds 0 and 4 are the ones the workload list
# fixes; seeds 1..3 were chosen here.
WORKLOADS = {
    "s2_8e2a_f32": Workload("DiT-MoE-S/2-8E2A layer, fp32", 512, 384, 1536, 8, 2, 2,
                            "f32", "topk", 0.01, 0, "none", 2, 256),
    "s2_16e2a_zipf": Workload("DiT-MoE-S/2-16E2A layer, bf16, Zipf(1.2) router bias",
                              16384, 384, 1536, 16, 2, 2, "bf16", "topk", 0.01, 1,
                              "zipf", 64, 256),
    "b2_8e2a": Workload("DiT-MoE-B/2-8E2A layer, bf16", 32768, 768, 3072, 8, 2, 2,
                        "bf16", "topk", 0.01, 2, "none", 128, 256),
    "xl2_8e2a_512": Workload("DiT-MoE-XL/2-8E2A layer at 512x512, bf16", 32768, 1152,
                             4608, 8, 2, 2, "bf16", "topk", 0.01, 3, "normal", 32, 1024),
    "xl_race_16e": Workload("Expert-Race routing at XL width, bf16, E=16, S=K*T",
                            32768, 1152, 4608, 16, 2, 1, "bf16", "race", 0.01, 4,
                            "none", 32, 1024),
}

WORKLOAD_ORDER = ["s2_8e2a_f32", "s2_16e2a_zipf", "b2_8e2a", "xl2_8e2a_512", "xl_race_16e"]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 value (ties to even); returns fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of fp32 values that are exactly bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def round_to_f16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest fp16 value (IEEE round to nearest even); returns fp32."""
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).astype(np.float32)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    if dtype == "bf16":
        return round_to_bf16(a)
    if dtype == "f16":
        return round_to_f16(a)
    return a


def make_inputs(w: Workload, bias_std: float = 0.0, x_only_tokens: Optional[int] = None) -> dict:
    """Draw every input array of workload ``w``.

    Returns a dict with (shapes; all fp32 arrays holding storage-type values):
      x [T,D], wg [E,D], router_bias [E] or None,
      w1 [E,H,D], b1 [E,H] or None, w2 [E,D,H], b2 [E,D] or None,
      ws1 [n_s,H,D], bs1 [n_s,H] or None, ws2 [n_s,D,H], bs2 [n_s,D] or None.
    Expert weights follow nn.Linear (out x in).
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    T, D, H, E, ns = w.T, w.D, w.H, w.E, w.n_shared
    out = {}
    out["x"] = _store(rng.standard_normal((T, D)), w.dtype)
    out["wg"] = _store(rng.standard_normal((E, D)) * np.sqrt(1.0 / D), w.dtype)
    out["w1"] = _store(rng.standard_normal((E, H, D)) * np.sqrt(1.0 / D), w.dtype)
    out["w2"] = _store(rng.standard_normal((E, D, H)) * np.sqrt(1.0 / H), w.dtype)
    out["ws1"] = _store(rng.standard_normal((ns, H, D)) * np.sqrt(1.0 / D), w.dtype)
    out["ws2"] = _store(rng.standard_normal((ns, D, H)) * np.sqrt(1.0 / H), w.dtype)
    if w.router_bias == "zipf":
        z = np.arange(1, E + 1, dtype=np.float64) ** -1.2
        out["router_bias"] = np.log(z / z.sum()).astype(np.float32)
    elif w.router_bias == "normal":
        out["router_bias"] = (rng.standard_normal(E) * np.sqrt(0.5)).astype(np.float32)
    else:
        out["router_bias"] = None
    if bias_std > 0.0:
        out["b1"] = _store(rng.standard_normal((E, H)) * bias_std, w.dtype)
        out["b2"] = _store(rng.standard_normal((E, D)) * bias_std, w.dtype)
        out["bs1"] = _store(rng.standard_normal((ns, H)) * bias_std, w.dtype)
        out["bs2"] = _store(rng.standard_normal((ns, D)) * bias_std, w.dtype)
    else:
        out["b1"] = out["b2"] = out["bs1"] = out["bs2"] = None
    return out


def small_workload(T: int, D: int, H: int, E: int, K: int, n_shared: int, dtype: str = "bf16",
                   routing: str = "topk", seed: int = 100, router_bias: str = "none",
                   alpha: float = 0.01) -> Workload:
    """A test-sized workload with the same recipe as the named ones."""
    return Workload(f"test T={T} D={D} H={H} E={E} K={K} ns={n_shared} {dtype} {routing}",
                    T, D, H, E, K, n_shared, dtype, routing, alpha, seed, router_bias, 1, T)
