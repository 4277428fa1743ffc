"""Seeded generators for the SERQ linear workloads.

Shapes and value distributions follow the LLaMA-2-7B / LLaMA-3-8B linear
layers the SERQ pages evaluate on (reading notes "GPU 性能分析" table: LLaMA-3
8B at 2K context; results tables: LLaMA-2 7B).  The pages use trained weights
and real calibration text, which are not available here; these seeded tensors
stand in for them with the same shapes:

* activations X ~ N(0, 1), with a seeded set of outlier channels multiplied
  by a constant (x30 or x50) or by a lognormal magnitude 50*exp(0.5*z);
* weights W ~ N(0, 0.02^2), laid out K x N (input channels x output
  channels), the math layout of Y = X W.

Every draw comes from ``numpy.random.default_rng([seed, stream])`` (PCG64),
so the same tensors are produced on any machine.  Values are rounded to
bfloat16 (round to nearest even) and returned as float32 arrays that are
exactly bf16-representable.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

# stream ids: keep X, W and calibration draws independent of each other
_STREAM_X = 1
_STREAM_OUTLIER_IDX = 2
_STREAM_OUTLIER_MAG = 3
_STREAM_W = 4
_STREAM_GAMMA = 5


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of bf16-representable float32 values (no rounding)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("values are not bf16-representable")
    return (u >> 16).astype(np.uint16)


def activations(seed: int, M: int, K: int, n_outliers: int,
                magnitude: str = "const", factor: float = 50.0) -> np.ndarray:
    """Token activations X (M x K) with ``n_outliers`` outlier channels.

    magnitude="const": outlier channels are scaled by ``factor``.
    magnitude="lognormal": channel c is scaled by factor*exp(0.5*z_c), z_c ~ N(0,1).
    """
    x = np.random.default_rng([seed, _STREAM_X]).standard_normal((M, K), dtype=np.float32)
    if n_outliers > 0:
        idx = np.random.default_rng([seed, _STREAM_OUTLIER_IDX]).choice(K, n_outliers, replace=False)
        if magnitude == "const":
            mag = np.full(n_outliers, factor, dtype=np.float32)
        elif magnitude == "lognormal":
            z = np.random.default_rng([seed, _STREAM_OUTLIER_MAG]).standard_normal(n_outliers)
            mag = (factor * np.exp(0.5 * z)).astype(np.float32)
        else:
            raise ValueError(magnitude)
        x[:, idx] *= mag[None, :]
    return round_to_bf16(x)


def weights(seed: int, K: int, N: int, std: float = 0.02) -> np.ndarray:
    """Weight W (K x N, input channel major) drawn N(0, std^2)."""
    w = np.random.default_rng([seed, _STREAM_W]).standard_normal((K, N), dtype=np.float32)
    return round_to_bf16(w * np.float32(std))


def norm_weight(seed: int, K: int, spread: float = 0.2) -> np.ndarray:
    """RMSNorm weight gamma (K,) drawn 1 + spread * N(0, 1) (a trained norm
    weight's typical range), rounded to bf16."""
    g = np.random.default_rng([seed, _STREAM_GAMMA]).standard_normal(K, dtype=np.float32)
    return round_to_bf16(np.float32(1.0) + np.float32(spread) * g)


@dataclasses.dataclass
class Linear:
    """One SERQ linear of a workload: shapes, rank, format and its draw recipe."""
    name: str
    K: int
    N: int
    r: int
    fmt: str                      # "int4" | "mxfp4"
    w_seeds: Tuple[int, ...]      # one seed per fused weight (gate/up share an input)
    x_seed: int
    n_outliers: int
    magnitude: str
    factor: float
    calib_seed: Optional[int] = None  # None: calibrate on the layer's own X
    calib_tokens: int = 2048

    def W(self) -> np.ndarray:
        n_each = self.N // len(self.w_seeds)
        return np.concatenate([weights(s, self.K, n_each) for s in self.w_seeds], axis=1)

    def X(self, M: int) -> np.ndarray:
        return activations(self.x_seed, M, self.K, self.n_outliers, self.magnitude, self.factor)

    def X_calib(self, M: int) -> np.ndarray:
        """Calibration activations for the SAF absmax (same distribution)."""
        if self.calib_seed is None:
            return self.X(M)
        return activations(self.calib_seed, self.calib_tokens, self.K, self.n_outliers,
                           self.magnitude, self.factor)


@dataclasses.dataclass
class Workload:
    name: str
    M: int
    linears: List[Linear]
    description: str


def _pct(K: int) -> int:
    return int(round(0.01 * K))


def workload(name: str, r: Optional[int] = None, M: Optional[int] = None) -> Workload:
    """The named synthetic workloads (shapes of the pages' LLaMA layers)."""
    if name == "tiny_int4":
        rr = 16 if r is None else r
        lin = Linear("tiny", 256, 256, rr, "int4", (0,), 0, 4, "const", 30.0)
        return Workload(name, M or 64, [lin],
                        "INT4, M=64, K=N=256, r=16; X N(0,1) with 4 channels x30; W N(0,0.02^2); seed 0")
    if name == "qproj_int4":
        rr = 128 if r is None else r
        lin = Linear("q_proj", 4096, 4096, rr, "int4", (0,), 0, _pct(4096), "const", 50.0)
        return Workload(name, M or 2048, [lin],
                        "LLaMA-2-7B q_proj shape, INT4, M=2048, K=N=4096, r=128; 1% channels x50")
    if name == "mlp_mxfp4":
        rr = 128 if r is None else r
        # gate and up read the same input, so they share one SAF scale vector and
        # one saliency permutation: they are prepared as one linear with N = 2*14336.
        gu = Linear("gate_up", 4096, 2 * 14336, rr, "mxfp4", (1, 2), 1, _pct(4096), "lognormal", 50.0)
        dn = Linear("down", 14336, 4096, rr, "mxfp4", (3,), 3, _pct(14336), "lognormal", 50.0)
        return Workload(name, M or 2048, [gu, dn],
                        "LLaMA-3-8B MLP, MXFP4, M=2048: gate/up 4096->2x14336 (shared input), "
                        "down 14336->4096, r=128; 1% outlier channels x 50*exp(0.5 z)")
    if name.startswith("decode_mxfp4"):
        rr = 128 if r is None else r
        shapes = [("q", 4096, 4096), ("kv", 4096, 1024), ("gate_up", 4096, 14336), ("down", 14336, 4096)]
        lins = [Linear(nm, K, N, rr, "mxfp4", (10 + i,), 10 + i, _pct(K), "const", 50.0,
                       calib_seed=100 + i) for i, (nm, K, N) in enumerate(shapes)]
        return Workload(name, M or 16, lins,
                        "LLaMA-3-8B linears at decode, MXFP4, M in {1,4,16}, r=128; "
                        "SAF calibrated on a separate 2048-token draw")
    if name == "stack_mxfp4":
        rr = 128 if r is None else r
        lins = []
        for blk in range(32):
            base = 7 * blk
            for idx, (nm, K, N) in enumerate([("qkv", 4096, 4096 + 2 * 1024), ("o", 4096, 4096),
                                              ("gate_up", 4096, 2 * 14336), ("down", 14336, 4096)]):
                lins.append(Linear(f"b{blk}.{nm}", K, N, rr, "mxfp4", (base + idx,), base + idx,
                                   _pct(K), "lognormal", 50.0))
        return Workload(name, M or 2048, lins,
                        "random-init LLaMA-3-8B stack, 32 blocks, MXFP4, M=2048")
    raise KeyError(name)


WORKLOADS: Dict[str, str] = {
    "tiny_int4": "configs: tiny INT4 layer",
    "qproj_int4": "configs: LLaMA-2-7B q_proj INT4",
    "mlp_mxfp4": "configs: LLaMA-3-8B MLP MXFP4 prefill",
    "decode_mxfp4": "configs: LLaMA-3-8B linears MXFP4 decode",
    "stack_mxfp4": "configs: LLaMA-3-8B 32-block stack MXFP4",
}
