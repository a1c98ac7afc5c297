"""Seeded synthetic inputs for the QE linear layer.

This module is shared by the tests, the benchmark and the oracle checks. It
holds none of the layer's arithmetic. It only draws numbers:

* activations with the outlier structure the Quant Experts pages describe: a
  few channels that are large on every token, plus per-token outliers drawn
  from one of two modality pools (image tokens vs text tokens);
* Gaussian weights, adapters and router weights;
* the per-channel smoothing factor taken from a separate calibration draw.
  This is SmoothQuant-style migration strength 0.5, computed once before
  the layer runs. Both the oracle and the GPU path receive it as an input.

Every array is rounded once to its stored dtype (fp32 or bf16). The oracle
and the GPU then read identical values. bf16 tensors are returned as torch
CPU tensors, and fp32 arrays as numpy float32.

The workload shapes follow the model shapes named on the pages (Qwen2VL-2B,
InternVL2-8B, Qwen2VL-72B) and the decode regime. The calibration and
benchmark datasets the pages use are not available, so these draws stand in
for them.
"""
from __future__ import annotations

import dataclasses
import numpy as np
import torch

__all__ = [
    "LayerConfig", "Projection", "CONFIGS", "config_by_name",
    "outlier_activations", "gaussian", "layer_inputs", "to_bf16", "topk_like_sets", "sparse_routed",
]


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """Round a float array to bf16 (round-to-nearest-even) as a torch CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


@dataclasses.dataclass(frozen=True)
class OutlierSpec:
    n_always: int          # channels that are large on every token
    always_mult: float     # multiplier on those channels
    pool_size: int         # channels in each modality pool
    draws: int             # outlier channels per token, drawn from its pool
    draw_lo: float         # per-draw multiplier ~ U(draw_lo, draw_hi)
    draw_hi: float


def spec_tiny() -> OutlierSpec:
    """The tiny layer: 4 always-on channels x20, two pools of 64 channels, 2 draws x30 per token."""
    return OutlierSpec(4, 20.0, 64, 2, 30.0, 30.0)


def spec_scaled(d: int) -> OutlierSpec:
    """The tiny recipe with every channel count scaled by d/256 (multipliers unchanged)."""
    f = d / 256.0
    return OutlierSpec(max(1, int(round(4 * f))), 20.0, max(1, int(round(64 * f))),
                       max(1, int(round(2 * f))), 30.0, 30.0)


def spec_qwen2b() -> OutlierSpec:
    """Qwen2VL-2B-shaped layers: 16 always-on x20, pools of 256 channels, 4 draws x U(10,50)."""
    return OutlierSpec(16, 20.0, 256, 4, 10.0, 50.0)


def outlier_activations(T: int, d: int, seed: int, spec: OutlierSpec) -> np.ndarray:
    """X ~ N(0,1) [T, d] in fp32 with the two-modality outlier structure.

    The first T//2 tokens are 'image' tokens and draw their outliers from pool A.
    The rest are 'text' tokens and draw from pool B. Channel sets are disjoint
    and chosen by the same seeded generator.
    """
    g = _rng(seed)
    x = g.standard_normal((T, d), dtype=np.float32)
    need = spec.n_always + 2 * spec.pool_size
    perm = g.permutation(d)
    if need > d:  # tiny widths: let pools overlap the always-on set
        perm = np.concatenate([perm, g.permutation(d)])
    always = perm[:spec.n_always]
    pool_a = perm[spec.n_always:spec.n_always + spec.pool_size] % d
    pool_b = perm[spec.n_always + spec.pool_size:spec.n_always + 2 * spec.pool_size] % d
    x[:, always] *= np.float32(spec.always_mult)
    half = T // 2
    for t in range(T):
        pool = pool_a if t < half else pool_b
        k = min(spec.draws, len(pool))
        ch = g.choice(pool, size=k, replace=False)
        mult = g.uniform(spec.draw_lo, spec.draw_hi, size=k).astype(np.float32) \
            if spec.draw_hi > spec.draw_lo else np.full(k, spec.draw_lo, np.float32)
        x[t, ch] *= mult
    return x


def topk_like_sets(T: int, d: int, k: int, seed: int) -> np.ndarray:
    """Seeded int32 [T, k] rows of k distinct channels in [0, d), shaped like Top-k sets.

    A quarter of each row is a fixed always-important set; half comes from the token's modality
    pool (image tokens first, then text tokens; pools of 8k channels, weights falling as
    1/(rank+1), so a few channels co-occur often); the rest is uniform over the other channels.
    """
    g = _rng(seed)
    n_always, n_pool = k // 4, k // 2
    n_rest = k - n_always - n_pool
    perm = g.permutation(d)
    always = perm[:n_always]
    psz = min(8 * k, max(n_pool, (d - n_always) // 2))
    pools = [perm[n_always:n_always + psz], perm[n_always + psz:n_always + 2 * psz]]
    w = 1.0 / np.arange(1, psz + 1)
    w /= w.sum()
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        pool = pools[0] if t < T // 2 else pools[1]
        ch = np.concatenate([always, g.choice(pool, size=n_pool, replace=False, p=w)])
        taken = set(ch.tolist())
        rest = []
        while len(rest) < n_rest:          # uniform draws, skipping channels already in the row
            c = int(g.integers(0, d))
            if c not in taken:
                taken.add(c)
                rest.append(c)
        out[t] = g.permutation(np.concatenate([ch, np.asarray(rest, dtype=ch.dtype)]))
    return out


def sparse_routed(d: int, n_routed: int, kc: int, r_r: int, seed: int):
    """Cluster-sparse routed experts: disjoint seeded channel clusters and their down-projections.

    Returns channels int32 [n_routed][kc] (expert e's cluster, distinct channels, disjoint across
    experts while d allows) and A_r bf16 [n_routed][kc][r_r] ~ N(0, 0.02).
    """
    g = _rng(seed)
    perm = g.permutation(d)
    if n_routed * kc > d:
        perm = np.concatenate([perm] + [g.permutation(d) for _ in range((n_routed * kc) // d)])
    ch = np.empty((n_routed, kc), dtype=np.int32)
    for e in range(n_routed):
        ch[e] = np.sort(perm[e * kc:(e + 1) * kc])
    A = (g.standard_normal((n_routed, kc, r_r), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    return ch, to_bf16(A)


def gaussian(shape, std: float, seed: int) -> np.ndarray:
    return (_rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class Projection:
    name: str
    d_in: int
    d_out: int


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    projections: tuple
    w_bits: int
    a_bits: int
    group: int
    rank_shared: int
    n_routed: int
    rank_routed: int
    topk: int
    x_dtype: str           # "f32" or "bf16"
    spec: str              # outlier recipe: "tiny" | "qwen2b" | "scaled"
    seed_base: int
    scale_fp16: bool = False   # weight group scales stored as fp16

    def outlier_spec(self, d: int) -> OutlierSpec:
        if self.spec == "tiny":
            return spec_tiny()
        if self.spec == "qwen2b":
            return spec_qwen2b()
        return spec_scaled(d)

    def with_(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": LayerConfig("tiny", 64, (Projection("x", 256, 256),), 4, 8, 64, 8, 4, 4, 8, "f32", "tiny", 1),
    "qwen2vl2b": LayerConfig(
        "qwen2vl2b", 2048,
        (Projection("q", 1536, 1536), Projection("o", 1536, 1536), Projection("gate", 1536, 8960),
         Projection("up", 1536, 8960), Projection("down", 8960, 1536)),
        4, 6, 128, 32, 8, 4, 32, "bf16", "qwen2b", 2),
    "internvl2_8b": LayerConfig(
        "internvl2_8b", 4096,
        (Projection("qkv", 4096, 6144), Projection("o", 4096, 4096), Projection("gate", 4096, 14336),
         Projection("up", 4096, 14336), Projection("down", 14336, 4096)),
        4, 8, 128, 32, 8, 4, 32, "bf16", "scaled", 3),
    "qwen2vl72b": LayerConfig(
        "qwen2vl72b", 8192,
        (Projection("q", 8192, 8192), Projection("k", 8192, 1024), Projection("v", 8192, 1024),
         Projection("o", 8192, 8192), Projection("gate", 8192, 29568), Projection("up", 8192, 29568),
         Projection("down", 29568, 8192)),
        4, 6, 128, 32, 8, 4, 32, "bf16", "scaled", 4),
    # weight-only prefill variants of the 2B layer set (W4A16 and W3A16 tables)
    "qwen2vl2b_w4a16": LayerConfig(
        "qwen2vl2b_w4a16", 2048,
        (Projection("q", 1536, 1536), Projection("o", 1536, 1536), Projection("gate", 1536, 8960),
         Projection("up", 1536, 8960), Projection("down", 8960, 1536)),
        4, 16, 128, 32, 8, 4, 32, "bf16", "qwen2b", 7),
    "qwen2vl2b_w3a16": LayerConfig(
        "qwen2vl2b_w3a16", 2048,
        (Projection("q", 1536, 1536), Projection("o", 1536, 1536), Projection("gate", 1536, 8960),
         Projection("up", 1536, 8960), Projection("down", 8960, 1536)),
        3, 16, 128, 32, 8, 4, 32, "bf16", "qwen2b", 8),
    "qwen2vl72b_rr32": LayerConfig(
        "qwen2vl72b_rr32", 8192,
        (Projection("q", 8192, 8192), Projection("k", 8192, 1024), Projection("v", 8192, 1024),
         Projection("o", 8192, 8192), Projection("gate", 8192, 29568), Projection("up", 8192, 29568),
         Projection("down", 29568, 8192)),
        4, 6, 128, 32, 8, 32, 32, "bf16", "scaled", 9),
    "decode72b_w4a8": LayerConfig(
        "decode72b_w4a8", 16,
        (Projection("gate", 8192, 29568), Projection("up", 8192, 29568), Projection("down", 29568, 8192)),
        4, 8, 128, 32, 8, 4, 32, "bf16", "scaled", 5),
    # W4A8 with fp16 group scales (the W4A8 rows of the pages' tables, half the scale bytes)
    "qwen2vl2b_w4a8_s16": LayerConfig(
        "qwen2vl2b_w4a8_s16", 2048,
        (Projection("q", 1536, 1536), Projection("o", 1536, 1536), Projection("gate", 1536, 8960),
         Projection("up", 1536, 8960), Projection("down", 8960, 1536)),
        4, 8, 128, 32, 8, 4, 32, "bf16", "qwen2b", 10, True),
    "decode72b_w4a8_s16": LayerConfig(
        "decode72b_w4a8_s16", 16,
        (Projection("gate", 8192, 29568), Projection("up", 8192, 29568), Projection("down", 29568, 8192)),
        4, 8, 128, 32, 8, 4, 32, "bf16", "scaled", 11, True),
    "decode72b_w3a16": LayerConfig(
        "decode72b_w3a16", 16,
        (Projection("gate", 8192, 29568), Projection("up", 8192, 29568), Projection("down", 29568, 8192)),
        3, 16, 128, 32, 8, 4, 32, "bf16", "scaled", 6),
}


def config_by_name(name: str) -> LayerConfig:
    return CONFIGS[name]


def layer_inputs(cfg: LayerConfig, proj: Projection, T: int | None = None, proj_index: int = 0,
                 calib_tokens: int = 256, adapter_std: float = 0.02) -> dict:
    """All inputs of one projection, rounded to their stored dtypes.

    Returns numpy fp32 arrays for fp32-stored tensors and torch bf16 CPU tensors
    for bf16-stored ones. Seeds: X 1000+, W 2000+, adapters 3000+, G 4000+,
    calibration X 5000+. Each is offset by the config seed base and the
    projection index.
    """
    T = cfg.T if T is None else T
    K, N = proj.d_in, proj.d_out
    sb = cfg.seed_base * 100 + proj_index
    spec = cfg.outlier_spec(K)
    x = outlier_activations(T, K, 1000 + sb, spec)
    xc = outlier_activations(calib_tokens, K, 5000 + sb, spec)
    w = gaussian((N, K), 0.02, 2000 + sb)
    if cfg.x_dtype == "bf16":
        w_store = to_bf16(w)
        w_f = w_store.float().numpy()
    else:
        w_store = w
        w_f = w
    if cfg.x_dtype == "bf16":
        x_store = to_bf16(x)
        xc_f = to_bf16(xc).float().numpy()
    else:
        x_store = x
        xc_f = xc
    # calibration-side smoothing factor (migration strength 0.5)
    amax_x = np.abs(xc_f).max(axis=0).astype(np.float64)
    amax_w = np.abs(w_f).max(axis=0).astype(np.float64)
    ok = (amax_x > 0) & (amax_w > 0)
    s = np.ones(K, np.float64)
    s[ok] = np.sqrt(amax_x[ok] / amax_w[ok])
    s = s.astype(np.float32)
    rs, nr, rr = cfg.rank_shared, cfg.n_routed, cfg.rank_routed
    A_s = to_bf16(gaussian((K, rs), adapter_std, 3000 + sb))
    B_s = to_bf16(gaussian((rs, N), adapter_std, 3100 + sb))
    A_r = to_bf16(gaussian((nr, K, rr), adapter_std, 3200 + sb))
    B_r = to_bf16(gaussian((nr, rr, N), adapter_std, 3300 + sb))
    G = to_bf16(gaussian((K, nr), 0.02, 4000 + sb))
    return dict(X=x_store, W=w_store, s=s, A_s=A_s, B_s=B_s, A_r=A_r, B_r=B_r, G=G,
                T=T, K=K, N=N)
