"""Seeded synthetic workloads for the MoE FFN layer.

This module only *draws inputs*: shapes, value distributions and seeds of the
layers the pages describe.  It contains none of the layer's arithmetic (no
routing, no capacity rule, no expert math), so both the CUDA path and the CPU
oracle can be fed from it without sharing any of the method.

Storage convention (fixed for the whole library, ``nn.Linear`` style, out-major
and K-contiguous):

* ``W_g``    router weight ``[E][d]``; the pages write ``z = x . W_g`` with
  ``W_g`` of shape ``d x E``, so ``W_g_store[e][i] = W_g_math[i][e]``.
* ``W_gu``   ``[E + S][2F][d]``: rows ``[0, F)`` hold ``W_gate``, rows
  ``[F, 2F)`` hold ``W_up`` (a ReLU expert stores only ``W1`` as ``[E+S][F][d]``).
* ``W_down`` ``[E + S][d][F]``.
* the shared expert (``S = 1``) is stored last, at index ``E``.

Workloads (shapes and distributions follow the pages and the layer sizes they
quote):

* ``toy``       -- the NumPy listing of the dataistudio "Mixture of Experts"
  page: 1000 tokens of d=64, 8 two-layer ReLU experts 64->256->64, router
  64x8, all drawn with ``numpy.random.default_rng(42)`` in the page's order
  (W1, W2, router, tokens), N(0, 0.1) weights, N(0, 1) tokens, fp32.
* ``mixtral-*`` -- d=4096, E=8 SwiGLU experts with d_ff=14336, top-2 softmax
  renormalised, weights N(0, 0.02), tokens N(0, 1), bf16.
* ``dsv3-*``    -- d=7168, 256 routed + 1 shared SwiGLU experts, d_ff=2048,
  top-8 sigmoid with a selection-only bias U(-0.1, 0.1) (the DeepSeek-V3
  numbers of the "Основы MoE" page, section on total and active parameters).
* ``capacity-*``-- d=2048, 64 routed + 1 shared, d_ff=1408, top-2 (or the
  Switch top-1 variant), router skewed by per-expert logit offsets
  ``2.0 * ln(Zipf_{1.1} pmf(rank))``, capacity factor 1, 1.25 or none.
* ``v41flash-*``-- d=5120, 384 routed + 1 shared, d_ff=2304, top-6 sigmoid with
  two selection-only bias sets (text, image), Bernoulli(0.3) image flags and
  the +-10 SwiGLU clip (the table of the DeepSeek-V4.1-Flash "Mixture-of-Experts"
  page, and its section on per-modality balancing).
"""
from __future__ import annotations

import dataclasses
from fractions import Fraction
from typing import Optional

import numpy as np
import torch

SOFTMAX, SIGMOID = 0, 1
SWIGLU, RELU = 0, 1
BF16, F32 = 0, 1


@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    N: int
    d: int
    E: int
    k: int
    F: int
    n_shared: int = 0
    score_fn: int = SOFTMAX
    renorm: int = 1
    act: int = SWIGLU
    clamp: float = 0.0            # <= 0: no clip
    dtype: int = BF16
    n_bias_sets: int = 0          # 0: no selection bias; 2: text/image sets
    bias_range: float = 0.1
    capacity_factor: Optional[Fraction] = None   # None: no capacity limit
    zipf_skew: bool = False
    w_std: float = 0.02
    seed: int = 0

    @property
    def G(self) -> int:
        """Number of expert weight slots (routed plus shared)."""
        return self.E + self.n_shared

    @property
    def gu_rows(self) -> int:
        return 2 * self.F if self.act == SWIGLU else self.F

    def with_N(self, N: int) -> "LayerShape":
        return dataclasses.replace(self, N=N)

    def replace(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)

    def weight_bytes(self) -> int:
        el = 2 if self.dtype == BF16 else 4
        return el * (self.G * (self.gu_rows * self.d + self.d * self.F) + self.E * self.d)


def _presets():
    p = {}
    p["toy"] = LayerShape("toy", N=1000, d=64, E=8, k=2, F=256, act=RELU, dtype=F32,
                          w_std=0.1, seed=42)
    mix = LayerShape("mixtral", N=16384, d=4096, E=8, k=2, F=14336, seed=1)
    for n in (16, 256, 4096, 16384):
        p[f"mixtral-n{n}"] = mix.replace(name=f"mixtral-n{n}", N=n)
    v3 = LayerShape("dsv3", N=8192, d=7168, E=256, k=8, F=2048, n_shared=1,
                    score_fn=SIGMOID, n_bias_sets=1, seed=2)
    for n in (64, 8192):
        p[f"dsv3-n{n}"] = v3.replace(name=f"dsv3-n{n}", N=n)
    cap = LayerShape("capacity", N=16384, d=2048, E=64, k=2, F=1408, n_shared=1,
                     zipf_skew=True, seed=3)
    for tag, cf in (("cf1", Fraction(1)), ("cf1.25", Fraction(5, 4)), ("cfinf", None)):
        p[f"capacity-{tag}"] = cap.replace(name=f"capacity-{tag}", capacity_factor=cf)
        p[f"switch-{tag}"] = cap.replace(name=f"switch-{tag}", k=1, renorm=0,
                                         capacity_factor=cf)
    v41 = LayerShape("v41flash", N=16384, d=5120, E=384, k=6, F=2304, n_shared=1,
                     score_fn=SIGMOID, n_bias_sets=2, clamp=10.0, seed=4)
    for n in (64, 16384):
        p[f"v41flash-n{n}"] = v41.replace(name=f"v41flash-n{n}", N=n)
    return p


PRESETS = _presets()


def zipf_logit_offsets(E: int, s: float = 1.1, scale: float = 2.0) -> np.ndarray:
    """Per-expert router skew ``scale * ln(pmf_Zipf(s)(rank))``, rank = e + 1.

    The normalising constant of the Zipf pmf is the same for every expert; it is
    dropped (it shifts every logit equally).  Expert 0 is the hottest.
    """
    ranks = np.arange(1, E + 1, dtype=np.float64)
    return (scale * (-s) * np.log(ranks)).astype(np.float32)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, std, g, device, dtype):
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=g)
    return t.to(dtype)


def make_inputs(shape: LayerShape, device="cpu", seed: Optional[int] = None,
                N: Optional[int] = None) -> dict:
    """Draw one seeded layer instance.

    Returns a dict of torch tensors on ``device``: ``x [N][d]``, ``W_g [E][d]``,
    ``W_gu``, ``W_down``, and where the workload has them ``bias
    [n_bias_sets][E]`` (fp32), ``modality [N]`` (uint8, 1 = image) and
    ``logit_offset [E]`` (fp32).  bf16 workloads draw fp32 values and round them
    to bf16 (round to nearest even).
    """
    seed = shape.seed if seed is None else seed
    N = shape.N if N is None else N
    if shape.name == "toy":
        return _make_toy(shape, device, seed, N)
    dt = torch.bfloat16 if shape.dtype == BF16 else torch.float32
    g = _gen(device, seed)
    out = {}
    out["W_gu"] = _normal_bf16((shape.G, shape.gu_rows, shape.d), shape.w_std, g, device, dt)
    out["W_down"] = _normal_bf16((shape.G, shape.d, shape.F), shape.w_std, g, device, dt)
    out["W_g"] = _normal_bf16((shape.E, shape.d), shape.w_std, g, device, dt)
    out["x"] = _normal_bf16((N, shape.d), 1.0, g, device, dt)
    if shape.n_bias_sets > 0:
        b = torch.empty((shape.n_bias_sets, shape.E), dtype=torch.float32, device=device)
        b.uniform_(-shape.bias_range, shape.bias_range, generator=g)
        out["bias"] = b
    if shape.n_bias_sets > 1:
        u = torch.empty((N,), dtype=torch.float32, device=device)
        u.uniform_(0.0, 1.0, generator=g)
        out["modality"] = (u < 0.3).to(torch.uint8)
    if shape.zipf_skew:
        out["logit_offset"] = torch.from_numpy(zipf_logit_offsets(shape.E)).to(device)
    return out


def _make_toy(shape, device, seed, N):
    rng = np.random.default_rng(seed)
    d, F, E = shape.d, shape.F, shape.E
    W1 = rng.normal(0, shape.w_std, (E, d, F))      # math orientation x . W1
    W2 = rng.normal(0, shape.w_std, (E, F, d))
    router = rng.normal(0, shape.w_std, (d, E))
    tokens = rng.normal(0, 1, (N, d))
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    return {
        "x": f32(tokens),
        "W_g": f32(router.T),                       # [E][d]
        "W_gu": f32(W1.transpose(0, 2, 1)),         # [E][F][d]
        "W_down": f32(W2.transpose(0, 2, 1)),       # [E][d][F]
    }


def random_logits(N: int, E: int, seed: int, scale: float = 1.0,
                  quantum: float = 0.0) -> np.ndarray:
    """Seeded fp32 router logits for routing-only cases.

    ``quantum > 0`` rounds the values to multiples of ``quantum`` so that exact
    ties between experts occur often (for the lowest-index tie-break rule).
    """
    rng = np.random.default_rng(seed)
    z = rng.normal(0.0, scale, (N, E))
    if quantum > 0:
        z = np.round(z / quantum) * quantum
    return z.astype(np.float32)


def random_bias(n_sets: int, E: int, seed: int, rng_range: float = 0.1) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.uniform(-rng_range, rng_range, (n_sets, E)).astype(np.float32)


def random_modality(N: int, seed: int, p_image: float = 0.3) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.uniform(0, 1, N) < p_image).astype(np.uint8)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 / fp32 torch tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float32).numpy().astype(np.float64)


def tokens_per_expert_estimate(shape: LayerShape) -> float:
    return shape.N * shape.k / shape.E


def expected_touched_experts(shape: LayerShape) -> float:
    """Expected number of routed experts hit by N tokens under uniform routing."""
    p_miss = (1 - shape.k / shape.E) ** shape.N
    return shape.E * (1 - p_miss)


__all__ = ["LayerShape", "PRESETS", "make_inputs", "zipf_logit_offsets", "random_logits",
           "random_bias", "random_modality", "bf16_to_f64", "SOFTMAX", "SIGMOID",
           "SWIGLU", "RELU", "BF16", "F32"]
