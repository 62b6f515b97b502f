"""Seeded synthetic workloads for the top-k gated MoE FFN layer.

This module is shared by the float64 oracle's tests, the CUDA parity tests,
``bench.py`` and ``__graft_entry__.smoke()``.  It holds the workload table and
the seeded input generator only: no step of the layer (gating, normalisation,
top-k, capacity, expert MLP, combine) is computed here.

Input recipe (the same for every workload):

* ``numpy.random.default_rng([seed, tensor_id, ...])`` with a fixed tensor id:
  x = 0 (plus a shard index for data-parallel replicas), W_gate = 1,
  W1 = (2, expert), W2 = (3, expert).  Weights are drawn expert by expert so
  that memory stays bounded and any one expert can be regenerated alone.
* x ~ N(0, 1); W_gate, W1 ~ N(0, 1/d_model); W2 ~ N(0, 1/F)  (fan-in scaling).
* Draws are float32; bf16 workloads round them to bfloat16 with
  round-to-nearest-even and keep the raw 16-bit patterns (``numpy.uint16``).
* The fine-grained workloads carry a deterministic gate bias
  b_e = -1.2 * ln(e + 1), i.e. a Zipf(s = 1.2) prior over experts with expert 0
  the most popular (no random draw involved).

The shapes follow the pages' layers: the FastMoE Transformer-XL experiment
(64 experts, 512->1024->512 ReLU MLPs, top-2), the Skywork-MoE gating-logit
normalisation with lambda = 1 (16 experts, top-2), a Mixtral-8x7B-shaped dropless
layer, and a DeepSeekMoE-style fine-grained layer with skewed routing.  No
dataset is used: synthetic tokens stand in for enwik8 and for the code
fine-tuning data by shape only.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional

import numpy as np

RELU = "relu"
SWIGLU = "swiglu"
F32 = "f32"
BF16 = "bf16"

TENSOR_X = 0
TENSOR_WG = 1
TENSOR_W1 = 2
TENSOR_W2 = 3


@dataclasses.dataclass(frozen=True)
class Workload:
    """One MoE layer shape.  ``capacity_factor <= 0`` means dropless and
    ``lam <= 0`` means plain softmax gating (no logit normalisation)."""

    name: str
    T: int
    d: int
    E: int
    F: int
    k: int
    act: str
    dtype: str
    capacity_factor: float = 0.0
    lam: float = 0.0
    zipf_bias: bool = False
    seed: int = 0
    description: str = ""

    @property
    def F1(self) -> int:
        """Rows of W1 per expert: F for ReLU, 2F for SwiGLU (gate rows then up rows)."""
        return self.F if self.act == RELU else 2 * self.F

    @property
    def has_bias(self) -> bool:
        return self.zipf_bias

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_fp32", T=256, d=64, E=8, F=128, k=2, act=RELU, dtype=F32,
                 description="tiny fp32 layer, 8 ReLU experts 64->128->64, top-2, dropless"),
        Workload("fastmoe_txl", T=8192, d=512, E=64, F=1024, k=2, act=RELU, dtype=BF16,
                 capacity_factor=1.25,
                 description="FastMoE Transformer-XL layer, 64 ReLU experts 512->1024->512, "
                             "top-2, capacity factor 1.25"),
        Workload("skywork_lambda1", T=4096, d=4096, E=16, F=8192, k=2, act=SWIGLU, dtype=BF16,
                 capacity_factor=1.0, lam=1.0,
                 description="Skywork-style layer, gating-logit normalisation lambda=1, "
                             "16 SwiGLU experts 4096->2x8192->4096, top-2, capacity factor 1.0"),
        Workload("mixtral_8x7b", T=16384, d=4096, E=8, F=14336, k=2, act=SWIGLU, dtype=BF16,
                 description="Mixtral-8x7B-shaped dropless layer, 8 SwiGLU experts "
                             "4096->2x14336->4096, top-2"),
        Workload("fine_decode_dropless", T=64, d=2048, E=64, F=1408, k=6, act=SWIGLU, dtype=BF16,
                 zipf_bias=True,
                 description="fine-grained layer, 64 SwiGLU experts 2048->2x1408->2048, top-6, "
                             "Zipf(1.2) gate bias, decode-sized T=64, dropless"),
        Workload("fine_decode_cap", T=64, d=2048, E=64, F=1408, k=6, act=SWIGLU, dtype=BF16,
                 zipf_bias=True, capacity_factor=1.0,
                 description="same layer at T=64 with capacity factor 1.0"),
        Workload("fine_large_dropless", T=32768, d=2048, E=64, F=1408, k=6, act=SWIGLU,
                 dtype=BF16, zipf_bias=True,
                 description="fine-grained layer at T=32768, dropless"),
        Workload("fine_large_cap", T=32768, d=2048, E=64, F=1408, k=6, act=SWIGLU, dtype=BF16,
                 zipf_bias=True, capacity_factor=1.0,
                 description="fine-grained layer at T=32768, capacity factor 1.0"),
    ]
}

# The workload the throughput metric is quoted on: the largest layer that fits
# one GPU (Mixtral-8x7B shape, 11.5 TFLOP of expert GEMMs per forward).
BENCH_WORKLOAD = "mixtral_8x7b"
# Further workloads the bench times on the device and reports beside it.
BENCH_EXTRA_WORKLOADS = ("fastmoe_txl", "fine_decode_dropless", "fine_large_dropless")


# ---------------------------------------------------------------- bf16 helpers
def round_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array -> bfloat16 bit patterns (uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 value of a stored input (uint16 = bf16 bits, or float32)."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


# ------------------------------------------------------------------- generator
def _normal(seed_seq, shape, std: float) -> np.ndarray:
    rng = np.random.default_rng(seed_seq)
    a = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return round_to_bf16_bits(a) if dtype == BF16 else a.astype(np.float32, copy=False)


def gen_x(w: Workload, shard: int = 0, T: Optional[int] = None) -> np.ndarray:
    """Token activations x[T, d] (shard = data-parallel replica index)."""
    T = w.T if T is None else T
    return _store(_normal([w.seed, TENSOR_X, shard], (T, w.d), 1.0), w.dtype)


def gen_wg(w: Workload) -> np.ndarray:
    """Gate weight W_gate[E, d] (nn.Linear layout, out x in)."""
    return _store(_normal([w.seed, TENSOR_WG], (w.E, w.d), 1.0 / math.sqrt(w.d)), w.dtype)


def gen_bias(w: Workload) -> Optional[np.ndarray]:
    """Gate bias b[E] (float32) or None.  Zipf(s=1.2) prior: b_e = -1.2 ln(e+1)."""
    if not w.zipf_bias:
        return None
    e = np.arange(w.E, dtype=np.float64)
    return (-1.2 * np.log(e + 1.0)).astype(np.float32)


def gen_w1_expert(w: Workload, e: int) -> np.ndarray:
    """W1[e] of shape [F1, d]; for SwiGLU rows [0,F) are the gate projection and
    rows [F, 2F) the up projection."""
    return _store(_normal([w.seed, TENSOR_W1, e], (w.F1, w.d), 1.0 / math.sqrt(w.d)), w.dtype)


def gen_w2_expert(w: Workload, e: int) -> np.ndarray:
    """W2[e] of shape [d, F]."""
    return _store(_normal([w.seed, TENSOR_W2, e], (w.d, w.F), 1.0 / math.sqrt(w.F)), w.dtype)


def _stack(fn, w: Workload, shape, threads: int) -> np.ndarray:
    dt = np.uint16 if w.dtype == BF16 else np.float32
    out = np.empty((w.E,) + shape, dtype=dt)

    def one(e):
        out[e] = fn(w, e)

    if threads > 1 and w.E > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(w.E)))
    else:
        for e in range(w.E):
            one(e)
    return out


def gen_w1(w: Workload, threads: int = 8) -> np.ndarray:
    return _stack(gen_w1_expert, w, (w.F1, w.d), threads)


def gen_w2(w: Workload, threads: int = 8) -> np.ndarray:
    return _stack(gen_w2_expert, w, (w.d, w.F), threads)


@dataclasses.dataclass
class Inputs:
    """Stored inputs of one workload (bf16 as uint16 bit patterns, else float32)."""

    w: Workload
    x: np.ndarray
    wg: np.ndarray
    bias: Optional[np.ndarray]
    w1: np.ndarray
    w2: np.ndarray


def generate(w: Workload, shard: int = 0, threads: int = 8) -> Inputs:
    return Inputs(w, gen_x(w, shard), gen_wg(w), gen_bias(w), gen_w1(w, threads), gen_w2(w, threads))


def to_device(a: Optional[np.ndarray], device="cuda"):
    """Upload a stored input to a torch tensor (bf16 bit patterns -> torch.bfloat16)."""
    if a is None:
        return None
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


class F64Experts:
    """Lazy float64 view of a stacked [E, ...] bf16/fp32 weight array: ``a[e]``
    returns expert e's matrix as exact float64, one expert at a time."""

    def __init__(self, stored: np.ndarray):
        self.stored = stored

    def __len__(self):
        return self.stored.shape[0]

    def __getitem__(self, e):
        return to_f64(self.stored[e])
