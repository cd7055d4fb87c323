"""Seeded synthetic inputs for the optimizer step (no optimizer arithmetic).

Both the CUDA path and the CPU oracle consume the arrays made here, so the
two sides always see the same bytes.  Every generator is a pure function of
its seed (numpy's counter-based Philox bit generator), so any step's gradient
can be regenerated without replaying earlier steps.

The workloads follow the shapes, sizes and value distributions of the
bitsandbytes issue "Investigate a 256-thread SM103 path for small 32-bit
optimizer tensors" (section "Correctness oracle": n = 1..1,024 boundary sizes
and 1,025/4,095/4,096/4,097 controls, zero / random / mixed-magnitude
gradients, FP16/BF16/FP32 storage; section "B300 benchmark and acceptance":
bias/norm/LoRA-like 64..1,024-element tensors mixed with larger ones).
There is no public dataset behind them: these synthetic collections stand in
for the issue's "fixed, reproducibly recorded" collections.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 0x0E0A0000

_NP = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}


def rng(seed: int, *stream: int) -> np.random.Generator:
    """Counter-based (Philox) generator keyed by (seed, *stream)."""
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, *stream])))


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values -> storage array of ``dtype`` (bf16 as uint16 bits).

    Rounding uses numpy (fp16) and ml_dtypes (bf16), both round-to-nearest-
    even; the generator's values only need to be some valid pattern of the
    storage type, so this is input preparation, not method arithmetic.
    """
    x = np.asarray(x, np.float32)
    if dtype == "f32":
        return x.copy()
    if dtype == "f16":
        return x.astype(np.float16)
    import ml_dtypes
    return x.astype(ml_dtypes.bfloat16).view(np.uint16)


def from_storage(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array -> float32 values (exact)."""
    if dtype == "f32":
        return a.astype(np.float32)
    if dtype == "f16":
        return a.view(np.float16).astype(np.float32)
    return (a.view(np.uint16).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# Value distributions
# --------------------------------------------------------------------------

def normal(seed: int, stream: tuple, n: int, std: float) -> np.ndarray:
    g = rng(seed, *stream)
    return (g.standard_normal(n, dtype=np.float32) * np.float32(std)).astype(np.float32)


def mixed_magnitude(seed: int, stream: tuple, n: int, lo: float = 1e-6,
                    hi: float = 1e2, zero_frac: float = 0.05) -> np.ndarray:
    """|g| log-uniform in [lo, hi], random sign, a fraction of exact zeros."""
    g = rng(seed, *stream)
    mag = np.exp(g.uniform(np.log(lo), np.log(hi), n)).astype(np.float32)
    sign = np.where(g.random(n) < 0.5, np.float32(-1), np.float32(1))
    out = (mag * sign).astype(np.float32)
    out[g.random(n) < zero_frac] = 0.0
    return out


def sparse_mixture(seed: int, stream: tuple, n: int, std: float,
                   zero_frac: float) -> np.ndarray:
    """N(0, std) with each element independently zeroed with ``zero_frac``."""
    g = rng(seed, *stream)
    out = (g.standard_normal(n, dtype=np.float32) * np.float32(std)).astype(np.float32)
    out[g.random(n) < zero_frac] = 0.0
    return out


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

@dataclass
class Workload:
    """A tensor collection, its hyper-parameters and its gradient recipe.

    Two ways to draw values, both pure functions of (seed, tensor, step):
      * direct (collections whose total size is below ``ring_threshold``):
        every step draws fresh values for the whole collection from its own
        Philox stream;
      * ring (larger collections): one seeded pool of ``pool_len`` values per
        quantity, and tensor i at step t reads the pool rotated by a seeded
        offset, ``pool[(offset(i, t) + j) % pool_len]``.  Any element of any
        step can then be rebuilt from its index alone, which lets the oracle
        check a sample of a multi-GB step without regenerating it.
    """
    name: str
    sizes: list
    dtypes: list
    algo: str
    hyper: dict
    steps: int
    seed: int
    grad_kind: str            # 'normal' | 'sparse_mixture' | 'mixed_magnitude'
    grad_std: float = 1e-2
    param_std: float = 1.0
    skip_zeros: bool = False
    ring_threshold: int = 1 << 24
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def numel(self) -> int:
        return int(sum(self.sizes))

    @property
    def ring(self) -> bool:
        return self.numel > self.ring_threshold

    @property
    def pool_len(self) -> int:
        return int(max(max(self.sizes), 1 << 20))

    # ---- direct mode ------------------------------------------------------
    def _grad_values(self, g: np.random.Generator, n: int, std_per_elem=None) -> np.ndarray:
        if self.grad_kind == "normal":
            return (g.standard_normal(n, dtype=np.float32) * np.float32(self.grad_std)).astype(np.float32)
        if self.grad_kind == "sparse_mixture":
            out = (g.standard_normal(n, dtype=np.float32) * std_per_elem).astype(np.float32)
            out[g.random(n) < 0.10] = 0.0
            return out
        if self.grad_kind == "mixed_magnitude":
            mag = np.exp(g.uniform(np.log(1e-6), np.log(1e2), n)).astype(np.float32)
            sign = np.where(g.random(n) < 0.5, np.float32(-1), np.float32(1))
            out = (mag * sign).astype(np.float32)
            out[g.random(n) < 0.05] = 0.0
            return out
        raise ValueError(self.grad_kind)

    def _split(self, flat: np.ndarray) -> list:
        return np.split(flat, np.cumsum(self.sizes)[:-1])

    def _std_per_elem(self) -> np.ndarray:
        """sparse_mixture: tensor i draws from N(0, 1e-3) if i is even, else
        N(0, 10)."""
        stds = np.where(np.arange(len(self.sizes)) % 2 == 0, np.float32(1e-3), np.float32(10.0))
        return np.repeat(stds.astype(np.float32), self.sizes)

    def params_init(self) -> list:
        """Initial param values (float32, already representable in each
        tensor's storage dtype) of every tensor, direct mode."""
        flat = normal(self.seed, (1,), self.numel, self.param_std)
        return [from_storage(to_storage(x, d), d) for x, d in zip(self._split(flat), self.dtypes)]

    def grads(self, step: int) -> list:
        """Gradient values (float32, representable in each storage dtype) of
        every tensor at 1-based ``step``, direct mode."""
        g = rng(self.seed, 2, step)
        std = self._std_per_elem() if self.grad_kind == "sparse_mixture" else None
        flat = self._grad_values(g, self.numel, std)
        return [from_storage(to_storage(x, d), d) for x, d in zip(self._split(flat), self.dtypes)]

    # ---- ring mode --------------------------------------------------------
    def pool(self, which: str) -> np.ndarray:
        """The seeded pool of float32 values for 'param' or 'grad'."""
        key = "_pool_" + which
        if key not in self.extra:
            if which == "param":
                vals = normal(self.seed, (5,), self.pool_len, self.param_std)
            else:
                std = np.full(self.pool_len, np.float32(self.grad_std), np.float32)
                if self.grad_kind == "sparse_mixture":
                    std = np.where(np.arange(self.pool_len) % 2 == 0, np.float32(1e-3),
                                   np.float32(10.0)).astype(np.float32)
                vals = self._grad_values(rng(self.seed, 6), self.pool_len, std)
            self.extra[key] = vals
        return self.extra[key]

    def offset(self, i: int, step: int) -> int:
        """Rotation of the pool for tensor i at ``step`` (step 0 = param init)."""
        return int(rng(self.seed, 7, step, i).integers(0, self.pool_len))

    def ring_values(self, which: str, i: int, step: int, idx: np.ndarray) -> np.ndarray:
        """Values of tensor i at element indices ``idx`` (float32,
        representable in the tensor's storage dtype)."""
        pool = self.pool(which)
        vals = pool[(self.offset(i, step) + idx) % self.pool_len]
        return from_storage(to_storage(vals, self.dtypes[i]), self.dtypes[i])


ADAM_HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, beta3=0.0,
                  alpha=0.0, weight_decay=0.0)
ADEMAMIX_HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8,
                      beta3=0.9999, alpha=5.0, weight_decay=0.0)

BOUNDARY_SIZES = [1, 2, 31, 32, 33, 127, 128, 129, 255, 256, 257, 511, 512,
                  513, 1023, 1024, 1025, 4095, 4096, 4097]

LAYER_SHAPES = [2048 * 2048] * 4 + [2048 * 8192] * 2 + [2048] * 4


def single_small() -> Workload:
    """One fp32 tensor of 1,024 elements, Adam, 10 steps."""
    return Workload("single_f32_n1024_adam", [1024], ["f32"], "adam",
                    dict(ADAM_HYPER), 10, SEED_BASE + 0, "normal")


def small_collection(count: int = 2000) -> Workload:
    """2,000 tensors of 64..1,024 elements, fp32/bf16/fp16 1:1:1, AdamW."""
    seed = SEED_BASE + 1
    sizes = rng(seed, 0).integers(64, 1025, count).tolist()
    dtypes = [("f32", "bf16", "f16")[i % 3] for i in range(count)]
    h = dict(ADAM_HYPER)
    h["weight_decay"] = 0.01
    return Workload("collection_2000_small_mixed_dtype_adamw", sizes, dtypes,
                    "adam", h, 100, seed, "sparse_mixture")


def large_f32(n: int = 268_435_456) -> Workload:
    """One fp32 tensor of 268,435,456 elements, Adam, 20 steps."""
    return Workload(f"single_f32_n{n}_adam", [n], ["f32"], "adam",
                    dict(ADAM_HYPER), 20, SEED_BASE + 2, "normal")


def transformer_bf16(layers: int = 24) -> Workload:
    """24 layers x {4 x 2048^2, 2 x 2048x8192, 4 x 2048}, bf16, AdEMAMix."""
    sizes = LAYER_SHAPES * layers
    h = dict(ADEMAMIX_HYPER)
    h["weight_decay"] = 0.1
    return Workload(f"transformer_{layers}x_bf16_ademamix", sizes,
                    ["bf16"] * len(sizes), "ademamix", h, 10, SEED_BASE + 3,
                    "normal", param_std=0.02)


def boundary_sweep(algo: str, dtype: str, skip_zeros: bool,
                   weight_decay: float = 0.0, big: int = 16_777_216,
                   steps: int = 1000) -> Workload:
    """Boundary sizes plus one large tensor, mixed-magnitude gradients."""
    h = dict(ADAM_HYPER if algo == "adam" else ADEMAMIX_HYPER)
    h["weight_decay"] = weight_decay
    sizes = list(BOUNDARY_SIZES) + ([big] if big else [])
    return Workload(f"boundary_{algo}_{dtype}_skip{int(skip_zeros)}_wd{weight_decay}",
                    sizes, [dtype] * len(sizes), algo, h, steps, SEED_BASE + 4,
                    "mixed_magnitude", skip_zeros=skip_zeros)


def sample_indices(n: int, stride: int = 97, edge: int = 4096) -> np.ndarray:
    """Deterministic index sample of a large tensor: every ``stride``-th
    element plus the first and last ``edge`` elements."""
    idx = np.arange(0, n, stride, dtype=np.int64)
    head = np.arange(0, min(edge, n), dtype=np.int64)
    tail = np.arange(max(0, n - edge), n, dtype=np.int64)
    return np.unique(np.concatenate([idx, head, tail]))
