"""Workload shapes and the seeded synthetic inputs for each.

The workloads follow the configurations the pages' method is measured on:
a lab-scale toy (width 8, 11 tokens), a single full-width block, a mid-size
model, the full-width 32-block model and a large multi-reference edit. The
test-only workloads (``small*``) are sized so that the fp64 oracle finishes in
seconds while every GPU tile shape still sees several tiles and ragged tails.

Nothing here computes a layer: these are shapes, segment lists and draws.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import numpy as np

from .gen import normal

TURBO_SIGMAS = (1.0, 0.978453, 0.95418, 0.926626, 0.89508, 0.845148, 0.704534, 0.414568, 0.0)
LAB_SIGMAS = (1.0, 0.85, 0.45, 0.0)

# Segment kinds (same codes as the C-ABI header).
SEG_TEXT = 0
SEG_IMAGE = 1


@dataclass(frozen=True)
class ModelShape:
    d_model: int
    n_heads: int
    head_dim: int
    n_layers: int
    mlp_hidden: int
    latent_ch: int
    time_dim: int
    rope: str = "axial"          # "axial" (16,56,56)-style split, or "lab" (micro split)
    use_shift: int = 0
    ln_eps: float = 1e-6
    qk_eps: float = 1e-6

    @property
    def n_chunks(self) -> int:
        return 6 if self.use_shift else 4


@dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    batch: int
    segments: Tuple[Tuple[int, int, int], ...]   # (kind, n_text | h, w)
    sigmas: Tuple[float, ...]
    seed: int
    weight_std: float = 0.02
    # (weight name, std) pairs that replace weight_std for those weights
    std_overrides: Tuple[Tuple[str, float], ...] = ()

    def std_of(self, name: str) -> float:
        for n, s in self.std_overrides:
            if n == name:
                return s
        return self.weight_std

    @property
    def n_prefix(self) -> int:
        return sum(s[1] if s[0] == SEG_TEXT else s[1] * s[2] for s in self.segments[:-1])

    @property
    def n_target(self) -> int:
        s = self.segments[-1]
        return s[1] * s[2]


def _text(n):
    return (SEG_TEXT, n, 0)


def _img(h, w):
    return (SEG_IMAGE, h, w)


TOY = ModelShape(8, 2, 4, 2, 16, 4, 8, rope="lab")
SMALL = ModelShape(256, 2, 128, 2, 768, 64, 256)
SMALL64 = ModelShape(256, 4, 64, 2, 768, 64, 256)
MID = ModelShape(1024, 16, 64, 8, 3072, 64, 256)
FULL = ModelShape(4096, 32, 128, 32, 12288, 64, 256)
BLOCK = ModelShape(4096, 32, 128, 1, 12288, 64, 256)

def parity_stds(shape: ModelShape) -> Tuple[Tuple[str, float], ...]:
    """Weight stds of the parity-test recipe (the benchmark keeps N(0, 0.02)).

    With every weight at N(0, 0.02) the timestep MLP produces modulation rows
    of order 1e-2, so tanh(gate) ~ 1e-2 scales every residual update down and
    v_theta is almost img_in + proj_out alone: a wrong attention or MLP would
    hide under the bf16 tolerance. These stds give modulation rows of order 1
    (timestep MLP and modulation at 1/sqrt(fan_in) and 2/sqrt(fan_in)) and an
    attention branch of the same order as the residual stream (W_v, W_o at
    2/sqrt(d)), so that every block, its attention included, moves v_theta and
    the cached K/V by far more than the tolerance.
    """
    d, t = shape.d_model, shape.time_dim
    return (("w_t1", 1.0 / t ** 0.5), ("w_t2", 2.0 / d ** 0.5), ("w_mod", 2.0 / d ** 0.5),
            ("w_fin", 2.0 / d ** 0.5), ("w_v", 2.0 / d ** 0.5), ("w_o", 2.0 / d ** 0.5))


WORKLOADS: Dict[str, Workload] = {
    # Lab-scale toy: [text, text, cond 2x2, text] + target 2x2 = 7 + 4 tokens.
    "toy": Workload("toy", TOY, 1, (_text(2), _img(2, 2), _text(1), _img(2, 2)), LAB_SIGMAS, 21),
    # Test-only (parity recipe): several 128-row tiles with ragged tails, two batch items.
    "small": Workload("small", SMALL, 2, (_text(77), _img(11, 11), _img(15, 20)), TURBO_SIGMAS, 1234,
                      std_overrides=parity_stds(SMALL)),
    "small64": Workload("small64", SMALL64, 2, (_text(40), _img(9, 10), _img(10, 13)), TURBO_SIGMAS, 1234,
                        std_overrides=parity_stds(SMALL64)),
    # Test-only (parity recipe): every attention pass fits one 128-key tile (P 56, N 64).
    "small_t1": Workload("small_t1", SMALL, 1, (_text(20), _img(6, 6), _img(8, 8)), TURBO_SIGMAS, 1234,
                         std_overrides=parity_stds(SMALL)),
    # Single full-width block.
    "block": Workload("block", BLOCK, 1, (_text(512), _img(64, 64), _img(64, 64)), TURBO_SIGMAS, 1234),
    "mid": Workload("mid", MID, 8, (_text(256), _img(16, 16), _img(16, 16)), TURBO_SIGMAS, 1234),
    "full": Workload("full", FULL, 1, (_text(512), _img(64, 64), _img(64, 64)), TURBO_SIGMAS, 1234),
    "large": Workload("large", FULL, 1,
                      (_text(1024), _img(128, 128), _img(128, 128), _img(128, 128)), TURBO_SIGMAS, 1234),
}


def make_workload(name: str) -> Workload:
    return WORKLOADS[name]


def parity_workload(name: str, **changes) -> Workload:
    """The named workload with the parity-test weight recipe (``parity_stds``)
    and any field replaced by ``changes`` (e.g. batch)."""
    import dataclasses
    w = make_workload(name)
    return dataclasses.replace(w, std_overrides=parity_stds(w.shape), **changes)


def weight_specs(shape: ModelShape) -> List[Tuple[str, Tuple[int, ...]]]:
    """Names and shapes of every weight, [out][in] (torch.nn.Linear) order.

    Per-layer tensors are stacked on a leading layer axis.
    """
    d, f, c, L, dh = shape.d_model, shape.mlp_hidden, shape.latent_ch, shape.n_layers, shape.head_dim
    return [
        ("w_img_in", (d, c)),
        ("w_out", (c, d)),
        ("w_t1", (d, shape.time_dim)),
        ("w_t2", (d, d)),
        ("w_mod", (shape.n_chunks * d, d)),
        ("w_fin", (d, d)),
        ("w_q", (L, d, d)),
        ("w_k", (L, d, d)),
        ("w_v", (L, d, d)),
        ("w_o", (L, d, d)),
        ("w_gate", (L, f, d)),
        ("w_up", (L, f, d)),
        ("w_down", (L, d, f)),
        ("q_norm", (L, dh)),
        ("k_norm", (L, dh)),
    ]


def _stream_name(name: str, layer: int | None) -> str:
    return name if layer is None else f"L{layer}.{name}"


def host_weights(w: Workload, store_dtype: str = "float32") -> Dict[str, np.ndarray]:
    """All weights as float64 arrays holding exactly the stored values.

    ``store_dtype`` is the dtype the CUDA path keeps them in ("float32" or
    "bfloat16"); each draw is rounded once to it, so the oracle and the GPU see
    the same numbers. The norm weights stay float32 on both sides.
    """
    out = {}
    for name, shp in weight_specs(w.shape):
        per_layer = len(shp) == 3 or name in ("q_norm", "k_norm")
        if per_layer:
            arr = np.stack([normal(w.seed, _stream_name(name, l), shp[1:], std=w.std_of(name))
                            for l in range(shp[0])])
        else:
            arr = normal(w.seed, name, shp, std=w.std_of(name))
        sd = "float32" if name in ("q_norm", "k_norm") else store_dtype
        out[name] = round_to(arr, sd)
    return out


def device_weights(w: Workload, torch_dtype, device) -> Dict[str, "object"]:
    """All weights drawn directly on a CUDA device (for models too large to
    draw on the host): the same named streams as ``host_weights``, each draw
    computed in float64 on the device and rounded once to ``torch_dtype``
    (norm weights float32). Returns torch tensors keyed by weight name."""
    import torch

    from .gen import normal_torch
    out = {}
    for name, shp in weight_specs(w.shape):
        sdt = torch.float32 if name in ("q_norm", "k_norm") else torch_dtype
        if len(shp) == 3 or name in ("q_norm", "k_norm"):
            t = torch.empty(shp, dtype=sdt, device=device)
            for l in range(shp[0]):
                t[l] = normal_torch(w.seed, _stream_name(name, l), shp[1:], std=w.std_of(name), device=device,
                                    dtype=torch.float32).to(sdt)
        else:
            t = normal_torch(w.seed, name, shp, std=w.std_of(name), device=device, dtype=torch.float32).to(sdt)
        out[name] = t
    return out


def round_to(a: np.ndarray, store_dtype: str) -> np.ndarray:
    """Round float64 values to float32 or bfloat16 (RNE) and return float64."""
    if store_dtype == "float64":
        return np.asarray(a, dtype=np.float64)
    f = np.asarray(a, dtype=np.float32)
    if store_dtype == "float32":
        return f.astype(np.float64)
    if store_dtype == "bfloat16":
        u = f.view(np.uint32).astype(np.uint64)
        # round to nearest even on the upper 16 bits (inputs are finite)
        rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
        b = (rounded << np.uint64(16)).astype(np.uint32)
        return b.view(np.float32).astype(np.float64)
    raise ValueError(store_dtype)


def host_prefix_hidden(w: Workload) -> np.ndarray:
    """Prefix hidden states [B][P][d], N(0,1), stored float32."""
    return round_to(normal(w.seed, "prefix_hidden", (w.batch, w.n_prefix, w.shape.d_model)), "float32")


def host_noise(w: Workload) -> np.ndarray:
    """Initial latent x_0 [B][N][C], N(0,1), stored float32."""
    return round_to(normal(w.seed, "noise", (w.batch, w.n_target, w.shape.latent_ch)), "float32")
