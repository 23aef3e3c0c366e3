"""Seeded synthetic inputs for the ReLU-gated FFN layer.

This module only draws random tensors. It performs none of the layer's
arithmetic (no products, no activation, no packing, no routing); the CUDA path
and the CPU oracle both consume exactly what it returns.

What the pages fix and what is read into them:

* The gate is a ReLU so that inactive hidden units are exact zeros, and more
  than 80% of the units rest on each step; a 1.5B model reaches under 2%
  nonzeros and a 2B model has fewer nonzeros than a 0.5B one
  (intellectnews.ru "Sakana AI и NVIDIA ..." -- section "Минимальные изменения
  в рецепте обучения"; gate.com post 20977915 -- the paragraph on the 1.5B
  model).
* Some neurons never activate under the chosen L1 setting ("dead" columns;
  intellectnews.ru -- section "Ограничения и открытые вопросы").

The density is steered per token and per column through two extra input
features: x[:, d-2] carries a per-token shift s_t that multiplies a row of ones
in Wg, and x[:, d-1] = 1 multiplies a per-column offset b_j (0 for live
columns, -64 for dead ones, or a constant offset that sets the density of the
small layer). The remaining d-2 gate features are N(0,1) inputs against
N(0,1/d) weights, so z[t,j] ~ N(s_t + b_j, (d-2)/d) and
P(z > 0) = Phi((s_t + b_j) / sigma_r).

Exactness: x and Wg are drawn on coarse grids (x = k/8, Wg = k * 2^-e with
|k| <= 255, s_t and b_j on 2^-5) so every product is a multiple of 2^-13 and
every partial sum of the gate stays far below 2^11. The gate pre-activation is
then exact in fp32 in any summation order, which makes the packed format,
counts and routing independent of the order the hardware sums in. Wu and Wd
are plain N(0,1/fan_in) values rounded to bf16.

Every array is returned as raw bf16 bit patterns (uint16).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "LayerConfig",
    "CONFIGS",
    "sweep_config",
    "make_layer",
    "f32_to_bf16_bits",
]


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """Shape and density structure of one synthetic FFN layer."""

    name: str
    T: int  # tokens (rows of x)
    d: int  # d_model
    f: int  # d_ff (hidden units)
    tile: int  # TwELL column-tile width
    W: int  # ELL slots per (row, column tile)
    density: float  # mean gate density over all f columns (dead included)
    sigma: float = 0.0  # lognormal spread of the per-token density
    dead_frac: float = 0.0  # fraction of columns that are never active
    heavy_frac: float = 0.0  # fraction of tokens drawn at a high density
    heavy_lo: float = 0.0
    heavy_hi: float = 0.0
    column_offset: bool = False  # density set by a constant per-column offset

    @property
    def nT(self) -> int:
        return self.f // self.tile


CONFIGS: dict[str, LayerConfig] = {
    # T=64, d=128, f=512, 5% fixed, offset carried by the Wg row that meets
    # the constant-1 feature.
    "tiny": LayerConfig("tiny", T=64, d=128, f=512, tile=128, W=16, density=0.05,
                        column_offset=True),
    # 8 sequences of 2048 tokens, 0.5B-like layer.
    "0.5b": LayerConfig("0.5b", T=16384, d=1536, f=4096, tile=128, W=32, density=0.05,
                        sigma=0.5, dead_frac=0.03),
    # 1.5B-like layer at the pages' "under 2%" density.
    "1.5b": LayerConfig("1.5b", T=16384, d=2048, f=5632, tile=128, W=16, density=0.018,
                        sigma=0.5, dead_frac=0.05),
    # 2B-like layer: 92% of tokens around 1.2%, 8% heavy tokens at 25-40% that
    # overflow the ELL width and take the dense branch.
    "2b": LayerConfig("2b", T=32768, d=2304, f=9216, tile=128, W=24, density=0.012,
                      sigma=0.5, heavy_frac=0.08, heavy_lo=0.25, heavy_hi=0.40),
}

SWEEP_T = (1, 16, 256, 4096, 16384)
SWEEP_P = (0.005, 0.01, 0.02, 0.05, 0.10, 0.25, 0.50)


def _sweep_width(T: int, f: int, tile: int, p: float) -> int:
    """ELL width for a sweep point: a multiple of 8 that a Binomial(tile, p)
    tile count exceeds with probability below 1e-3 over the whole batch."""
    from scipy.stats import binom

    ntiles = max(1, T * (f // tile))
    q = 1.0 - 1e-3 / ntiles
    w = int(binom.ppf(q, tile, p))
    w = max(8, -(-w // 8) * 8)
    return min(tile, w)


def sweep_config(T: int, p: float, d: int = 2048, f: int = 8192, tile: int = 128) -> LayerConfig:
    """Density/batch sweep point: uniform per-token density, no dead columns."""
    return LayerConfig(f"sweep_T{T}_p{p:g}", T=T, d=d, f=f, tile=tile,
                       W=_sweep_width(T, f, tile, p), density=p)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _weight_exponent(d: int) -> int:
    # Grid 2^-e for Wg with e = floor(log2 sqrt(d)) + 5: the integer k of
    # Wg = k * 2^-e then has a standard deviation between 16 and 32.
    return int(math.floor(math.log2(math.sqrt(d)))) + 5


def _quantise(values: np.ndarray, step: float, kmax: int = 255) -> np.ndarray:
    k = np.clip(np.rint(values / step), -kmax, kmax)
    return (k * step).astype(np.float32)


def _config_key(cfg: LayerConfig) -> int:
    h = 0
    for ch in cfg.name.encode():
        h = (h * 131 + ch) % (2**31 - 1)
    return h


def make_layer(cfg: LayerConfig, seed: int = 0) -> dict:
    """Draw x [T,d], WgT [f,d], WuT [f,d], Wd [f,d] as bf16 bit arrays.

    WgT and WuT hold the gate and up matrices transposed (row j = column j of
    Wg / Wu, i.e. the weight of an nn.Linear(d, f)); Wd holds the down matrix
    as [f, d] (row j multiplies hidden unit j).
    Also returned: per-token target density ``p_t`` and the ``dead`` column mask.
    """
    T, d, f = cfg.T, cfg.d, cfg.f
    if d < 4:
        raise ValueError("d must be at least 4")
    ss = np.random.SeedSequence([seed, _config_key(cfg)])
    r_x, r_g, r_u, r_d, r_p, r_dead, r_heavy = (np.random.Generator(np.random.PCG64(s))
                                                for s in ss.spawn(7))
    sigma_r = math.sqrt((d - 2) / d)

    # Per-token density and dead columns.
    if cfg.sigma > 0:
        p_t = cfg.density * np.exp(cfg.sigma * r_p.standard_normal(T) - 0.5 * cfg.sigma**2)
    else:
        p_t = np.full(T, cfg.density)
    if cfg.heavy_frac > 0:
        n_heavy = int(round(cfg.heavy_frac * T))
        heavy = r_heavy.permutation(T)[:n_heavy]
        p_t[heavy] = r_heavy.uniform(cfg.heavy_lo, cfg.heavy_hi, size=n_heavy)
    p_t = np.clip(p_t, 0.0, 0.99)
    dead = np.zeros(f, dtype=bool)
    n_dead = int(round(cfg.dead_frac * f))
    if n_dead:
        dead[r_dead.permutation(f)[:n_dead]] = True

    if cfg.column_offset:
        s_t = np.zeros(T)
        b = sigma_r * float(_inv_cdf_vec(np.array([cfg.density]))[0])
        b_j = np.full(f, b)
    else:
        q = np.clip(p_t / (1.0 - cfg.dead_frac), 1e-4, 0.999)
        s_t = sigma_r * _inv_cdf_vec(q)
        b_j = np.where(dead, -64.0, 0.0)
    s_t = _quantise(s_t, 2.0**-5)
    b_j = _quantise(b_j, 2.0**-5, kmax=4095)  # -64 = -2048 * 2^-5, exact in bf16

    # x: quantised N(0,1) features, then the shift and the constant feature.
    x = np.empty((T, d), dtype=np.float32)
    x[:, : d - 2] = _quantise(r_x.standard_normal((T, d - 2), dtype=np.float32), 1.0 / 8)
    x[:, d - 2] = s_t
    x[:, d - 1] = 1.0

    # Wg (stored transposed): quantised N(0,1/d), a row of ones and the offsets.
    e = _weight_exponent(d)
    wgt = np.empty((f, d), dtype=np.float32)
    wgt[:, : d - 2] = _quantise(r_g.standard_normal((f, d - 2), dtype=np.float32) / math.sqrt(d),
                                2.0**-e)
    wgt[:, d - 2] = 1.0
    wgt[:, d - 1] = b_j

    wut = r_u.standard_normal((f, d), dtype=np.float32) / np.float32(math.sqrt(d))
    wd = r_d.standard_normal((f, d), dtype=np.float32) / np.float32(math.sqrt(f))

    return {
        "x": f32_to_bf16_bits(x),
        "WgT": f32_to_bf16_bits(wgt),
        "WuT": f32_to_bf16_bits(wut),
        "Wd": f32_to_bf16_bits(wd),
        "p_t": p_t,
        "dead": dead,
        "config": cfg,
        "seed": seed,
    }


def _inv_cdf_vec(q: np.ndarray) -> np.ndarray:
    from scipy.special import ndtri

    return ndtri(q)


def make_dy(T: int, d: int, seed: int = 0) -> np.ndarray:
    """Seeded upstream gradient for the backward pass, [T, d]: N(0, 1) drawn
    in fp32 and rounded to bf16 (uint16 bit patterns)."""
    rng = np.random.default_rng(1000 + seed)
    return f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
