"""Replay of the NumPy lab's micro model through the fp64 oracle.

TEST INFRASTRUCTURE (same import rule as ``qi21_oracle``).

The lab page ("Bài Lab tổng hợp — Qwen-Image-2.1 Architecture", script
``qwen-image-21.py``) draws its untrained weights once from
``numpy.random.default_rng(21)`` in a fixed order and prints, among other
checks, the prefix-K drift when the prefix reads the t_step modulation row
(End-to-end lab §4 "Profiling": 9.61e-01 at layer 0 and 1.68e+00 at layer 1).
Reproducing those numbers needs the same draws in the same order and the same
micro front-end (VAE encode, latent standardisation, txt_in), so this module
re-creates the draw sequence (shapes, scales and order must match the lab's,
which is why this part is alike) and feeds the resulting inputs to the
oracle's own block, attention, cache and Euler functions.

Lab-only differences from the production reading, all confined here:
6 modulation chunks with shifts and a two-row bias table, time_dim 8 with a
linear embedding-to-table map, a linear final scale with a bias, SwiGLU width
24, one QK-norm vector shared by both layers, and the micro RoPE split.
"""
from __future__ import annotations

import numpy as np

from . import qi21_oracle as O

DIM = 8
N_HEADS = 2
HEAD_DIM = 4
N_LAYERS = 2
MLP_DIM = 24
LATENT = 4
RGBA = 4
TIME_DIM = 8
EPS = 1e-6
SIGMAS = (1.0, 0.85, 0.45, 0.0)
# [text, text, cond 2x2, text] + target 2x2 (lab [2A]: repeats [1, 1, 4, 1])
SEGMENTS = ((O.SEG_TEXT, 2, 0), (O.SEG_IMAGE, 2, 2), (O.SEG_TEXT, 1, 0), (O.SEG_IMAGE, 2, 2))


def draw_lab_weights(seed: int = 21):
    """The lab's draws in its order; matrices stay in the lab's [in][out] form."""
    rng = np.random.default_rng(seed)

    def n(shape, s):
        return rng.normal(0.0, s, shape)

    w = {}
    w["latent_mean"] = n((LATENT,), 0.20)
    w["latent_std"] = 0.5 + np.abs(n((LATENT,), 0.25))
    w["w_enc"] = n((RGBA, LATENT), 0.45)
    w["b_enc"] = n((LATENT,), 0.20)
    w["w_dec"] = n((LATENT, RGBA), 0.45)
    w["b_dec"] = n((RGBA,), 0.20)
    w["w_img_in"] = n((LATENT, DIM), 0.35)
    w["context"] = n((4, DIM), 0.40)
    w["rms_ctx"] = n((DIM,), 0.30)
    w["w_txt1"] = n((DIM, DIM), 0.30)
    w["w_txt2"] = n((DIM, DIM), 0.30)
    w["w_t_mod"] = n((TIME_DIM, 6 * DIM), 0.20)
    w["mod_bias"] = n((2, 6 * DIM), 0.15)
    w["w_out_mod"] = n((TIME_DIM, DIM), 0.20)
    for name, shape, s in (("w_q", (DIM, DIM), 0.30), ("w_k", (DIM, DIM), 0.30),
                           ("w_v", (DIM, DIM), 0.30), ("w_o", (DIM, DIM), 0.30),
                           ("gate1_unused", (DIM,), 0.30),
                           ("w_gate", (DIM, MLP_DIM), 0.30), ("w_up", (DIM, MLP_DIM), 0.30),
                           ("w_down", (MLP_DIM, DIM), 0.25), ("gate2_unused", (DIM,), 0.30)):
        w[name] = np.stack([n(shape, s) for _ in range(N_LAYERS)])
    w["rms_q"] = n((HEAD_DIM,), 0.30)
    w["rms_k"] = n((HEAD_DIM,), 0.30)
    w["w_unpatch"] = n((DIM, LATENT), 0.35)
    w["noise"] = n((4, LATENT), 1.0)
    w["scale_out_base"] = n((DIM,), 0.15)
    return w


def _gelu_tanh(x):
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def text_slot_tokens(w) -> np.ndarray:
    """Lab [1B]: the text slots 0, 1, 3 of the VLM context -> zero-centred RMSNorm -> GELU MLP."""
    return np.stack([_gelu_tanh(O.rmsnorm_zero_centre(w["context"][i], w["rms_ctx"], EPS) @ w["w_txt1"])
                     @ w["w_txt2"] for i in (0, 1, 3)])


def cond_image_tokens(w, demo_rgba: np.ndarray) -> np.ndarray:
    """Lab [1A]: cond latent = standardise(rgba W_enc + b_enc), then img_in (4 tokens)."""
    z = np.asarray(demo_rgba, dtype=np.float64).reshape(-1, RGBA) @ w["w_enc"] + w["b_enc"]
    z_std = (z - w["latent_mean"]) / w["latent_std"]
    return z_std @ w["w_img_in"]


def slot_vectors(w) -> np.ndarray:
    """The 4 VLM slots as the packing reads them: txt_in of the text slots, the
    image slot (index 2) as the VLM left it (lab [1B], [2A])."""
    txt = text_slot_tokens(w)
    return np.stack([txt[0], txt[1], w["context"][2], txt[2]])


def prefix_tokens(w, demo_rgba: np.ndarray) -> np.ndarray:
    """The lab's 7 prefix rows, laid out as the lab does it: two text rows, the
    image slot vector added to each of the 4 img_in tokens, the last text row."""
    txt = text_slot_tokens(w)
    cond = cond_image_tokens(w, demo_rgba) + w["context"][2]
    return np.concatenate([txt[:2], cond, txt[2:]], axis=0)


def lab_model(w) -> O.Model:
    """Oracle model with the lab's weights, converted to [out][in]."""
    wts = {
        "w_img_in": w["w_img_in"].T,
        "w_out": w["w_unpatch"].T,
        "w_q": np.transpose(w["w_q"], (0, 2, 1)),
        "w_k": np.transpose(w["w_k"], (0, 2, 1)),
        "w_v": np.transpose(w["w_v"], (0, 2, 1)),
        "w_o": np.transpose(w["w_o"], (0, 2, 1)),
        "w_gate": np.transpose(w["w_gate"], (0, 2, 1)),
        "w_up": np.transpose(w["w_up"], (0, 2, 1)),
        "w_down": np.transpose(w["w_down"], (0, 2, 1)),
        "q_norm": np.stack([w["rms_q"]] * N_LAYERS),
        "k_norm": np.stack([w["rms_k"]] * N_LAYERS),
    }
    return O.Model(N_HEADS, N_LAYERS, 6, EPS, EPS, O.rope_omega_lab(), wts)


def lab_mod_fn(w, causal_row: bool = True):
    """The lab's two-row table: t_step row = emb(t) W + bias0, t = 0 row = emb(0) W + bias1.

    Returns f(t) -> (mod_row, scale_final). For t == 0 the second bias row is
    used, which is the row every prefix token reads (lab [3B]).
    """
    def f(t):
        emb = O.timestep_embedding(t, TIME_DIM)
        row = 1 if (t == 0.0 and causal_row) else 0
        mod = emb @ w["w_t_mod"] + w["mod_bias"][row]
        sf = emb @ w["w_out_mod"] + w["scale_out_base"]
        return mod, sf
    return f


def prefix_k_drift(w, demo_rgba) -> list:
    """Per-layer max |K_prefix(t=1000 row) - K_prefix(t=850 row)| with the
    prefix reading the t_step row (End-to-end lab §4, second bullet)."""
    model = lab_model(w)
    seq = O.make_sequence(SEGMENTS)
    pre = prefix_tokens(w, demo_rgba)
    f = lab_mod_fn(w)
    k1, _ = O.prefix_extract(model, seq, pre, f(1000.0)[0])
    k2, _ = O.prefix_extract(model, seq, pre, f(850.0)[0])
    return [float(np.max(np.abs(k1[l] - k2[l]))) for l in range(N_LAYERS)]
