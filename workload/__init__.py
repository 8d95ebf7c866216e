"""Seeded synthetic workloads for activation-sparse FFN decode.

This module only draws inputs: weights, biases, predictor parameters, the
per-neuron activation profile and decode tokens.  It holds none of the
method's arithmetic (no predictor evaluation, no FFN), so both the CPU oracle
and the CUDA library can be fed from it without sharing any computation.

Shapes follow the models the pages measure: OPT-6.7B (ReLU, >90% activation
sparsity; 53ai.com "sparsity for LLM inference" page, section on the
feasibility of activation sparsity), LLaMA-7B with a ReLU-gated FFN, OPT-30B
and a 70B ReGLU model whose activations follow a power law in which 26% / 43%
of the neurons carry 80% of all activations (hexiedandong.com PowerInfer news
page, the paragraph on figure (a), the power-law distribution of neuron
activations).  The pages publish no trained weights or datasets that this
repository may use, so every tensor here is random with the stated
distributions:

* ``W_up``, ``W_gate``, ``W_down`` entries ~ N(0, 1/d); tokens ``x`` ~ N(0, 1).
* per-neuron activation probability ``p_i`` from a Zipf law over hotness ranks,
  ``p = min(p_max, s * rank^-alpha)``, ``s`` set by bisection so that
  ``mean(p)`` equals the configured mean; ranks are dealt to neurons by a seeded
  permutation so that the library's hotness reordering is a real step.
* bias of the activated projection ``b_i = -Phi^-1(1 - p_i)`` (= ``Phi^-1(p_i)``):
  with unit-norm rows and x ~ N(0, I), ``P(W[i].x + b_i > 0) = p_i``.
* predictor ``A`` [d x r], ``B`` [r x n] entries ~ N(0, 1/r); the predictor bias
  ``c_i`` is calibrated in closed form (Gaussian approximation of
  ``relu(x.A).B[:, i]``) so that neuron i is predicted active with probability
  ``p_i``.

Random numbers come from numpy's PCG64 keyed by ``SeedSequence([seed, layer,
stream, block])``: generation is split in fixed row blocks and is bit-identical
for any number of threads.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
from scipy.special import ndtri

# stream ids of the independent sub-streams of one layer
_S_UP, _S_GATE, _S_DOWN, _S_PERM, _S_A, _S_B, _S_TOKENS = range(7)
_BLOCK = 1 << 22  # elements per independently keyed block
_POOL_THREADS = 8


@dataclass(frozen=True)
class LayerConfig:
    """One synthetic FFN workload.

    ``top_frac``: when set, the Zipf exponent is solved so that the hottest
    ``top_frac`` of neurons carry 80% of the expected activations.
    """

    name: str
    d: int
    n: int
    r: int
    act: str  # "relu" | "reglu"
    dtype: str  # "f32" | "f16"
    mean_p: float
    alpha: float | None = None
    top_frac: float | None = None
    layers: int = 1
    batches: tuple = (1,)
    tokens: int = 64
    p_max: float = 0.99
    description: str = ""

    @property
    def np_dtype(self):
        return np.float16 if self.dtype == "f16" else np.float32

    @property
    def esize(self) -> int:
        return 2 if self.dtype == "f16" else 4

    @property
    def nproj(self) -> int:
        return 3 if self.act == "reglu" else 2


CONFIGS: dict[str, LayerConfig] = {
    "tiny_relu_f32": LayerConfig(
        "tiny_relu_f32", d=512, n=2048, r=64, act="relu", dtype="f32",
        mean_p=0.10, alpha=1.2, tokens=64,
        description="tiny ReLU FFN, fp32, d=512 n=2048 r=64, Zipf 1.2 mean 0.10, batch 1"),
    "opt6.7b_relu": LayerConfig(
        "opt6.7b_relu", d=4096, n=16384, r=1024, act="relu", dtype="f16",
        mean_p=0.10, alpha=1.2, tokens=512,
        description="OPT-6.7B-shaped ReLU FFN layer, fp16, d=4096 n=16384 r=1024, "
                    "Zipf 1.2 mean 0.10, batch 1"),
    "llama7b_reglu_stack": LayerConfig(
        "llama7b_reglu_stack", d=4096, n=11008, r=1024, act="reglu", dtype="f16",
        mean_p=0.15, alpha=1.0, layers=4, tokens=512,
        description="LLaMA-7B-shaped ReGLU FFN, fp16, d=4096 n=11008 r=1024, "
                    "Zipf 1.0 mean 0.15, 4-layer stack with residual, batch 1"),
    "opt30b_relu": LayerConfig(
        "opt30b_relu", d=7168, n=28672, r=1024, act="relu", dtype="f16",
        mean_p=0.10, top_frac=0.26, batches=(1, 2, 4, 8), tokens=256,
        description="OPT-30B-shaped ReLU FFN, fp16, d=7168 n=28672 r=1024, "
                    "26% of neurons carry 80%, mean 0.10, batch 1-8"),
    "70b_reglu": LayerConfig(
        "70b_reglu", d=8192, n=28672, r=1024, act="reglu", dtype="f16",
        mean_p=0.12, top_frac=0.43, batches=(1, 2, 4, 8, 16, 32), tokens=128,
        description="70B-ReGLU-shaped FFN, fp16, d=8192 n=28672 r=1024, "
                    "43% of neurons carry 80%, mean 0.12, batch 1-32"),
}

# order in which the configurations are listed by the workload definition
CONFIG_ORDER = ["tiny_relu_f32", "opt6.7b_relu", "llama7b_reglu_stack",
                "opt30b_relu", "70b_reglu"]


# ---------------------------------------------------------------- profiles
def zipf_profile(n: int, alpha: float, mean: float, p_max: float = 0.99) -> np.ndarray:
    """p by hotness rank (index 0 = hottest): min(p_max, s*rank^-alpha), mean(p) = mean."""
    ranks = np.arange(1, n + 1, dtype=np.float64)
    base = ranks ** (-alpha)
    lo, hi = 0.0, p_max / base[-1] * 2.0 + 1.0
    for _ in range(200):
        s = 0.5 * (lo + hi)
        m = np.minimum(p_max, s * base).mean()
        if m < mean:
            lo = s
        else:
            hi = s
    return np.minimum(p_max, 0.5 * (lo + hi) * base)


def top_share(p_by_rank: np.ndarray, frac: float) -> float:
    """Share of the expected activations carried by the hottest ``frac`` of neurons."""
    k = int(round(frac * p_by_rank.size))
    return float(p_by_rank[:k].sum() / p_by_rank.sum())


def solve_alpha(n: int, top_frac: float, mean: float, p_max: float = 0.99,
                share: float = 0.80) -> float:
    """Zipf exponent for which the hottest ``top_frac`` of neurons carry ``share``."""
    lo, hi = 0.05, 4.0
    for _ in range(80):
        a = 0.5 * (lo + hi)
        if top_share(zipf_profile(n, a, mean, p_max), top_frac) < share:
            lo = a
        else:
            hi = a
    return 0.5 * (lo + hi)


def config_alpha(cfg: LayerConfig) -> float:
    if cfg.alpha is not None:
        return cfg.alpha
    return solve_alpha(cfg.n, cfg.top_frac, cfg.mean_p, cfg.p_max)


def expected_union_density(p: np.ndarray, b: int) -> float:
    """E|U|/n for b independent tokens: mean_i 1-(1-p_i)^b."""
    return float(np.mean(1.0 - (1.0 - p) ** b))


# ---------------------------------------------------------------- drawing
def _gen(seed: int, layer: int, stream: int, block: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer, stream, block])))


def _normal(seed: int, layer: int, stream: int, shape, scale: float, dtype) -> np.ndarray:
    """N(0, scale^2) of ``shape`` in ``dtype``, drawn in fixed keyed blocks (thread-count independent)."""
    total = int(np.prod(shape))
    out = np.empty(total, dtype=dtype)
    nblocks = (total + _BLOCK - 1) // _BLOCK

    def fill(bi):
        lo = bi * _BLOCK
        hi = min(total, lo + _BLOCK)
        v = _gen(seed, layer, stream, bi).standard_normal(hi - lo, dtype=np.float32)
        if scale != 1.0:
            v *= np.float32(scale)
        out[lo:hi] = v.astype(dtype, copy=False)

    if nblocks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(min(_POOL_THREADS, nblocks)) as ex:
            list(ex.map(fill, range(nblocks)))
    return out.reshape(shape)


@dataclass
class Layer:
    """One layer's parameters in PyTorch layouts and the storage dtype."""

    cfg: LayerConfig
    w_up: np.ndarray  # [n, d]
    w_gate: np.ndarray | None  # [n, d] (ReGLU) or None
    b: np.ndarray  # [n] bias of the activated projection
    w_down: np.ndarray  # [d, n]
    A: np.ndarray  # [d, r]
    B: np.ndarray  # [r, n]
    c: np.ndarray  # [n]
    p: np.ndarray  # [n] float64: activation probability (hotness profile)
    alpha: float = 0.0
    extras: dict = field(default_factory=dict)


def activation_profile(cfg: LayerConfig, seed: int, layer: int = 0) -> tuple[np.ndarray, float]:
    """Per-neuron activation probability, Zipf over ranks dealt by a seeded permutation."""
    alpha = config_alpha(cfg)
    p_rank = zipf_profile(cfg.n, alpha, cfg.mean_p, cfg.p_max)
    perm = _gen(seed, layer, _S_PERM).permutation(cfg.n)
    p = np.empty(cfg.n, dtype=np.float64)
    p[perm] = p_rank  # neuron perm[k] gets rank k+1
    return p, alpha


def calibrate_predictor_bias(A: np.ndarray, B: np.ndarray, p: np.ndarray) -> np.ndarray:
    """c_i with P(relu(x.A).B[:, i] + c_i > 0) ~= p_i for x ~ N(0, I).

    u_j = x.A[:, j] ~ N(0, sigma_j^2), sigma_j = ||A[:, j]||; relu(u_j) has mean
    sigma_j/sqrt(2 pi) and variance sigma_j^2 (1/2 - 1/(2 pi)).  Treating the
    sum over j as Gaussian with independent terms gives mean mu_i and
    variance s_i^2, and c_i = s_i Phi^-1(p_i) - mu_i.
    """
    A64 = A.astype(np.float64)
    sig = np.sqrt((A64 * A64).sum(axis=0))  # [r]
    B64 = B.astype(np.float64)
    mu = (sig / math.sqrt(2.0 * math.pi)) @ B64  # [n]
    var = ((sig * sig) * (0.5 - 0.5 / math.pi)) @ (B64 * B64)
    return np.sqrt(var) * ndtri(p) - mu


def make_layer(cfg: LayerConfig, seed: int = 0, layer: int = 0) -> Layer:
    d, n, r, dt = cfg.d, cfg.n, cfg.r, cfg.np_dtype
    p, alpha = activation_profile(cfg, seed, layer)
    w_up = _normal(seed, layer, _S_UP, (n, d), 1.0 / math.sqrt(d), dt)
    w_gate = _normal(seed, layer, _S_GATE, (n, d), 1.0 / math.sqrt(d), dt) if cfg.act == "reglu" else None
    w_down = _normal(seed, layer, _S_DOWN, (d, n), 1.0 / math.sqrt(d), dt)
    b = ndtri(p).astype(dt)  # = -Phi^-1(1 - p)
    A = _normal(seed, layer, _S_A, (d, r), 1.0 / math.sqrt(r), dt)
    B = _normal(seed, layer, _S_B, (r, n), 1.0 / math.sqrt(r), dt)
    c = calibrate_predictor_bias(A, B, p).astype(dt)
    return Layer(cfg, w_up, w_gate, b, w_down, A, B, c, p, alpha)


def make_tokens(cfg: LayerConfig, count: int, seed: int = 0, stream_key: int = 0) -> np.ndarray:
    """``count`` decode tokens x ~ N(0, 1) of shape [count, d] in the storage dtype."""
    return _normal(seed, 1000 + stream_key, _S_TOKENS, (count, cfg.d), 1.0, cfg.np_dtype)


def make_stack(cfg: LayerConfig, seed: int = 0) -> list[Layer]:
    return [make_layer(cfg, seed, layer) for layer in range(cfg.layers)]


def small_config(base: LayerConfig, d: int, n: int, r: int, name: str | None = None) -> LayerConfig:
    """A reduced copy of ``base`` (same activation, dtype and profile shape) for fast tests."""
    return LayerConfig(name or f"{base.name}_small", d=d, n=n, r=r, act=base.act, dtype=base.dtype,
                       mean_p=base.mean_p, alpha=config_alpha(base), layers=base.layers,
                       batches=base.batches, tokens=base.tokens, p_max=base.p_max,
                       description=f"reduced {base.name}")


def touched_bytes(cfg: LayerConfig, active_rows: float, b: int = 1) -> float:
    """Algorithmic bytes one step must move: full predictor, active rows, biases, x and y."""
    e = cfg.esize
    pred = (cfg.d * cfg.r + cfg.r * cfg.n + cfg.n) * e
    rows = active_rows * (cfg.nproj * cfg.d * e + e)
    io = b * cfg.d * (e + 4)
    return float(pred + rows + io)
