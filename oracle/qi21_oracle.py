"""fp64 CPU oracle of the cached Flow-Matching Euler step (Qwen-Image-2.1 style DiT).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference arm of ``bench.py`` may import or run this module.
The product (the C-ABI library and its Python binding) never calls it, and it
shares no code with the CUDA path.

Everything is float64 numpy, written as the plain definitions the pages give,
in the pages' order; numpy's matmul is the only library primitive used as a
step. Page citations name the page and its section (the pages are five course
pages on Qwen-Image-2.1; the lab page carries the NumPy lab ``qwen-image-21.py``
whose blocks are labelled [1A] .. [6B]):

* "End-to-end lab" = "Lab tổng hợp Qwen-Image-2.1 — chạy toàn trình 1A → 6B bằng NumPy"
* "6B page" = "6B · Scale-Only Final AdaLN, Dự đoán vận tốc v_θ & Vòng lặp 8-Step Euler"
* "3B page" = "3B · Điều kiện nhân quả (t=0 vs t) & Bộ điều biến dùng chung"
* "2A page" = "2A · Mở rộng 4× Slot ảnh & Ghép chuỗi đồng nhất"
* "Lab page" = "Bài Lab tổng hợp — Qwen-Image-2.1 Architecture" (the 1:1 mapping
  table and the lab script)

Readings taken where the pages are silent or disagree (each is listed with its
reason in the design notes of the repository):

* modulation has 4 chunks [scale1, gate1, scale2, gate2] and no shift (3B page,
  §1 and §2); the lab's 6-chunk form with shift1/shift2 is kept as
  ``n_chunks == 6`` (order shift1, scale1, gate1, shift2, scale2, gate2) for the
  lab replay only;
* residual gates are tanh(gate) (End-to-end lab §3; lab [4A], [5A]);
* QK-RMSNorm is zero-centred, x * rsqrt(mean x^2 + eps) * (1 + w), per head,
  before RoPE (lab [4A]);
* masked attention scores are excluded (the lab's -1e9 gives exp() == 0 in fp64);
* the timestep MLP is Linear(time_dim->d) -> SiLU -> Linear(d->d); the shared
  modulation is SiLU -> Linear(d -> n_chunks*d); the final scale is
  SiLU -> Linear(d->d) of the same embedding; no biases (3B page §1 names
  "sin-cos then MLP" without its shape);
* sin-cos embedding: cos half then sin half, frequencies 10000^(-2i/time_dim)
  (lab [3B]);
* RoPE pairs are adjacent dims (2j, 2j+1), angle = sum over axes of coord * omega
  (lab [3A]); image grids are centred with integer n//2 (lab [3A], End-to-end
  lab §3); text tokens take (i, i, i) counting text tokens only;
* joint packing of the prefix values: every VLM image slot stands for
  IMG_TOKENS_PER_SLOT = 4 latent cells (2A page), so an image of h*w cells
  (h*w divisible by 4) has h*w/4 slots; repeat_interleave writes each slot's
  vector at 4 consecutive positions of the image's token run (raster order).
  At image positions the 2A page replaces the slot value by the img_in token
  (the default, PACK_SUBSTITUTE); the lab adds the two (its COND_TOKENS,
  PACK_ADD).

Parity unpinned: nothing. Each function has a pin in ``tests/test_oracle_pins.py``
(page-printed values, closed forms, library routines or brute force); the
output head (``final_velocity``, ``img_in``), which the lab replay's drift
check never reaches, is pinned by closed-form LayerNorm rows through a
non-symmetric one-hot W_out and by hand-worked products, and
``tests/test_oracle_mutations.py`` shows each pin catching planted mistakes.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Sequence, Tuple

import numpy as np

SEG_TEXT = 0
SEG_IMAGE = 1

# ---------------------------------------------------------------------------
# [2A] packing metadata, [3A] RoPE coordinates, [3C] block-causal mask
# ---------------------------------------------------------------------------


def token_metadata(segments: Sequence[Tuple[int, int, int]]):
    """image_ids and target_token_mask of the packed sequence.

    2A page §1: text tokens carry id -1, condition images 0..K-1 in order, the
    image being generated carries K and is the only one whose tokens have
    target_token_mask True; the target is placed last (2A page §2, "Chữ → Ảnh
    tham chiếu → Ảnh đích"). Each image segment contributes h*w tokens.
    Returns (image_ids int64[S], target_mask bool[S], S, P, N).
    """
    if not segments or segments[-1][0] != SEG_IMAGE:
        raise ValueError("the last segment must be the target image")
    n_images = sum(1 for s in segments if s[0] == SEG_IMAGE)
    ids: List[int] = []
    mask: List[bool] = []
    img = 0
    for kind, a, b in segments:
        if kind == SEG_TEXT:
            ids += [-1] * a
            mask += [False] * a
        else:
            ids += [img] * (a * b)
            mask += [img == n_images - 1] * (a * b)
            img += 1
    ids_a = np.array(ids, dtype=np.int64)
    mask_a = np.array(mask, dtype=bool)
    n = int(mask_a.sum())
    return ids_a, mask_a, len(ids), len(ids) - n, n


def rope_coords(segments, frame_mode: int = 0) -> np.ndarray:
    """(frame, height, width) integer coordinate of every token.

    Lab [3A] and End-to-end lab §3: text tokens advance on all three axes
    together, (i, i, i), where i counts text tokens only; every image pins
    frame = 0 and centres its grid, rows h - H//2 (outer) and columns w - W//2
    (inner, row-major). ``frame_mode=1`` is the alternative reading with
    frame = image id.
    """
    coords = []
    text_i = 0
    img = 0
    for kind, a, b in segments:
        if kind == SEG_TEXT:
            for _ in range(a):
                coords.append((text_i, text_i, text_i))
                text_i += 1
        else:
            f = img if frame_mode == 1 else 0
            for r in range(a):
                for c in range(b):
                    coords.append((f, r - a // 2, c - b // 2))
            img += 1
    return np.array(coords, dtype=np.int64)


# Joint packing of the prefix values (2A page; lab [2A])
IMG_TOKENS_PER_SLOT = 4        # 2A page: one VLM image slot <-> a 2x2 block of latent cells
PACK_SUBSTITUTE = 0            # 2A page, mechanism (2): img_in replaces the slot value
PACK_ADD = 1                   # lab [2A]: COND_TOKENS = img_in(latent) + image slot vector


def slot_expansion(segments):
    """Index tables of the 4x slot expansion over the prefix (every segment but
    the last, which is the target).

    2A page, mechanism (1): repeat_interleave repeats each VLM slot vector
    consecutively, once for a text slot and IMG_TOKENS_PER_SLOT times for an
    image slot (repeats = where(img_mask, 4, 1)); (2): image positions take the
    img_in token of their latent cell. Returns slot_of int64[P] (the slot each
    prefix token expands), img_row int64[P] (row of the table of image tokens,
    reference images concatenated in order, raster order inside an image; -1 at
    text positions), n_slots and n_img.
    """
    repeats: List[int] = []
    img_row: List[int] = []
    n_img = 0
    for kind, a, b in segments[:-1]:
        if kind == SEG_TEXT:
            repeats += [1] * a
            img_row += [-1] * a
        else:
            cells = a * b
            if cells % IMG_TOKENS_PER_SLOT:
                raise ValueError("an image slot covers 4 latent cells: h*w must be divisible by 4")
            repeats += [IMG_TOKENS_PER_SLOT] * (cells // IMG_TOKENS_PER_SLOT)
            img_row += list(range(n_img, n_img + cells))
            n_img += cells
    slot_of = np.repeat(np.arange(len(repeats), dtype=np.int64), repeats)
    return slot_of, np.array(img_row, dtype=np.int64), len(repeats), n_img


def pack_prefix(ctx: np.ndarray, img_tokens: np.ndarray, segments, mode: int = PACK_SUBSTITUTE) -> np.ndarray:
    """Prefix hidden states [P, d] from the VLM slot vectors ctx [n_slots, d]
    (text slots after txt_in, image slots as the VLM left them) and the img_in
    tokens of the reference images img_tokens [n_img, d] (2A page, mechanism
    (1)-(2); lab [2A])."""
    slot_of, img_row, _, _ = slot_expansion(segments)
    out = ctx[slot_of].copy()
    m = img_row >= 0
    if mode == PACK_SUBSTITUTE:
        out[m] = img_tokens[img_row[m]]
    else:
        out[m] = out[m] + img_tokens[img_row[m]]
    return out


def block_causal_allowed(image_ids: np.ndarray) -> np.ndarray:
    """allowed[q, kv] = (q >= kv) or (id[q] == id[kv] >= 0).

    Lab [3C] and the Lab page's 1:1 table row 3C: text attends causally, the
    tokens of one image see each other both ways.
    """
    s = len(image_ids)
    allowed = np.zeros((s, s), dtype=bool)
    for q in range(s):
        for kv in range(s):
            same = image_ids[q] >= 0 and image_ids[q] == image_ids[kv]
            allowed[q, kv] = (q >= kv) or same
    return allowed


# ---------------------------------------------------------------------------
# [3A] RoPE frequencies and rotation
# ---------------------------------------------------------------------------


def rope_omega_axial(head_dim: int, base: float = 10000.0) -> np.ndarray:
    """Per-pair angular frequency per axis, shape [head_dim/2][3].

    Lab [3A] notes: production splits head_dim 128 as (frame 16, height 56,
    width 56) -> 8 + 28 + 28 rotation pairs, base 10000. Reading: axis a of
    width dim_a owns dim_a/2 consecutive pairs with omega = base^(-2j/dim_a);
    for other head dims the split scales with head_dim/128.
    """
    if head_dim % 16:
        raise ValueError("axial RoPE needs head_dim divisible by 16")
    dims = (head_dim // 8, head_dim * 7 // 16, head_dim * 7 // 16)
    omega = np.zeros((head_dim // 2, 3), dtype=np.float64)
    p = 0
    for axis, dim_a in enumerate(dims):
        for j in range(dim_a // 2):
            omega[p, axis] = base ** (-2.0 * j / dim_a)
            p += 1
    assert p == head_dim // 2
    return omega


def rope_omega_lab(base: float = 10000.0) -> np.ndarray:
    """The lab's micro split for head_dim 4 (lab [3A]).

    Pair 0 turns with the frame axis at rate 1; pair 1 is shared by height
    (rate base^-1) and width (rate base^-1.5), the angles adding.
    """
    return np.array([[1.0, 0.0, 0.0],
                     [0.0, base ** (-2.0 * 2.0 / 4), base ** (-2.0 * 3.0 / 4)]], dtype=np.float64)


def rope_angles(coords: np.ndarray, omega: np.ndarray) -> np.ndarray:
    """angle[s, j] = sum_a coords[s, a] * omega[j, a]."""
    return coords.astype(np.float64) @ omega.T


def rope_rotate(x: np.ndarray, coords: np.ndarray, omega: np.ndarray) -> np.ndarray:
    """Rotate adjacent pairs (2j, 2j+1) of the last axis of x [..., S, Dh].

    Lab [3A] ``rope_rotate_heads``: (x0, x1) -> (x0 c - x1 s, x0 s + x1 c) with
    c, s the cos/sin of the pair's angle at that token.
    """
    ang = rope_angles(coords, omega)          # [S, Dh/2]
    c = np.cos(ang)
    s = np.sin(ang)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ---------------------------------------------------------------------------
# Elementwise definitions
# ---------------------------------------------------------------------------


def layernorm(x: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm without affine parameters, biased variance (lab helpers)."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def rmsnorm_zero_centre(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """Zero-centred RMSNorm x * rsqrt(mean(x^2) + eps) * (1 + w) (lab helpers)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * (1.0 + w)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def masked_softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                             allowed: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(Dh) over allowed keys) v, per head.

    q [H, Sq, Dh], k/v [H, Sk, Dh], allowed [Sq, Sk] (lab [4A]; masked keys are
    excluded, which is what the lab's -1e9 score offset gives in fp64).
    """
    dh = q.shape[-1]
    scores = q @ np.swapaxes(k, -1, -2) / np.sqrt(dh)          # [H, Sq, Sk]
    scores = np.where(allowed[None], scores, -np.inf)
    m = scores.max(axis=-1, keepdims=True)
    e = np.where(allowed[None], np.exp(scores - m), 0.0)
    w = e / e.sum(axis=-1, keepdims=True)
    return w @ v


# ---------------------------------------------------------------------------
# [3B] timestep embedding and the shared modulation
# ---------------------------------------------------------------------------


def timestep_embedding(t: float, time_dim: int, base: float = 10000.0) -> np.ndarray:
    """[cos(t f_i) ..., sin(t f_i) ...] with f_i = base^(-2i/time_dim) (lab [3B])."""
    freqs = base ** (-2.0 * np.arange(time_dim // 2) / time_dim)
    ang = float(t) * freqs
    return np.concatenate([np.cos(ang), np.sin(ang)])


def modulation(t: float, wts: Dict[str, np.ndarray], n_chunks: int):
    """Shared modulation row and final scale at timestep t = 1000 * sigma.

    3B page §1: sin-cos of 1000*sigma, then an MLP to width d; one shared
    SiLU -> Linear(d -> n_chunks*d) produces the chunks read by every block.
    6B page §3: the final scale comes from the same t row. Weights are [out][in].
    Returns (mod_row [n_chunks*d], scale_final [d]).
    """
    emb = timestep_embedding(t, wts["w_t1"].shape[1])
    e = wts["w_t2"] @ silu(wts["w_t1"] @ emb)
    se = silu(e)
    mod_row = wts["w_mod"] @ se
    scale_final = wts["w_fin"] @ se
    assert mod_row.shape[0] == n_chunks * e.shape[0]
    return mod_row, scale_final


def split_chunks(mod_row: np.ndarray, n_chunks: int) -> Dict[str, np.ndarray]:
    """Name the chunks of one modulation row (3B page §2; lab [3B] for 6)."""
    d = mod_row.shape[0] // n_chunks
    parts = [mod_row[i * d:(i + 1) * d] for i in range(n_chunks)]
    if n_chunks == 4:
        names = ("scale1", "gate1", "scale2", "gate2")
        out = dict(zip(names, parts))
        out["shift1"] = np.zeros(d)
        out["shift2"] = np.zeros(d)
        return out
    if n_chunks == 6:
        names = ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")
        return dict(zip(names, parts))
    raise ValueError(n_chunks)


def select_modulation_rows(target_mask: np.ndarray, row_prefix: Dict[str, np.ndarray],
                           row_target: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """Per-token chunks: mask False -> the prefix row (t = 0), True -> t_step row.

    3B page §1/§2 (``_select_modulation_rows``).
    """
    out = {}
    for key in row_prefix:
        out[key] = np.where(target_mask[:, None], row_target[key][None, :], row_prefix[key][None, :])
    return out


# ---------------------------------------------------------------------------
# [4A] + [5A] one single-stream DiT block
# ---------------------------------------------------------------------------


@dataclass
class BlockOut:
    h: np.ndarray        # [S, d]
    k_rot: np.ndarray    # [S, H, Dh] post QK-norm, post RoPE
    v: np.ndarray        # [S, H, Dh]


def _heads(x: np.ndarray, n_heads: int) -> np.ndarray:
    s, d = x.shape
    return x.reshape(s, n_heads, d // n_heads).transpose(1, 0, 2)   # [H, S, Dh]


def dit_block(h: np.ndarray, mods: Dict[str, np.ndarray], lw: Dict[str, np.ndarray],
              n_heads: int, coords: np.ndarray, omega: np.ndarray,
              kv_extra: Tuple[np.ndarray, np.ndarray] | None, allowed: np.ndarray,
              ln_eps: float, qk_eps: float) -> BlockOut:
    """One block over the rows of h (lab [4A] then [5A]).

    x = LN(h)(1 + scale1) + shift1; q, k, v = x Wq, x Wk, x Wv; q, k get the
    per-head zero-centred RMSNorm then RoPE; attention over [kv_extra; own k/v]
    restricted by ``allowed``; h += tanh(gate1) (attn Wo); then
    x2 = LN(h)(1 + scale2) + shift2; h += tanh(gate2) ((silu(x2 Wg) * (x2 Wu)) Wd).
    ``kv_extra`` is the cached prefix (k_rot, v) [P, H, Dh] for the cached mode
    (lab [6A]); ``allowed`` is [S_q, P_extra + S_q].
    """
    s, d = h.shape
    x_mod = layernorm(h, ln_eps) * (1.0 + mods["scale1"]) + mods["shift1"]
    q = _heads(x_mod @ lw["w_q"].T, n_heads)
    k = _heads(x_mod @ lw["w_k"].T, n_heads)
    v = _heads(x_mod @ lw["w_v"].T, n_heads)
    q = rmsnorm_zero_centre(q, lw["q_norm"], qk_eps)
    k = rmsnorm_zero_centre(k, lw["k_norm"], qk_eps)
    q = rope_rotate(q, coords, omega)
    k = rope_rotate(k, coords, omega)
    if kv_extra is not None:
        k_all = np.concatenate([kv_extra[0].transpose(1, 0, 2), k], axis=1)
        v_all = np.concatenate([kv_extra[1].transpose(1, 0, 2), v], axis=1)
    else:
        k_all, v_all = k, v
    attn = masked_softmax_attention(q, k_all, v_all, allowed)         # [H, S, Dh]
    attn_flat = attn.transpose(1, 0, 2).reshape(s, d)
    h = h + np.tanh(mods["gate1"]) * (attn_flat @ lw["w_o"].T)
    x2 = layernorm(h, ln_eps) * (1.0 + mods["scale2"]) + mods["shift2"]
    hidden = silu(x2 @ lw["w_gate"].T) * (x2 @ lw["w_up"].T)
    h = h + np.tanh(mods["gate2"]) * (hidden @ lw["w_down"].T)
    return BlockOut(h, k.transpose(1, 0, 2), v.transpose(1, 0, 2))


def layer_weights(wts: Dict[str, np.ndarray], l: int) -> Dict[str, np.ndarray]:
    return {k: wts[k][l] for k in ("w_q", "w_k", "w_v", "w_o", "w_gate", "w_up", "w_down",
                                   "q_norm", "k_norm")}


# ---------------------------------------------------------------------------
# [6B] output head and the Euler update
# ---------------------------------------------------------------------------


def final_velocity(h_target: np.ndarray, scale_final: np.ndarray, w_out: np.ndarray,
                   ln_eps: float) -> np.ndarray:
    """v = (LN(h)(1 + scale_final)) W_out: scale-only final AdaLN, no shift.

    6B page §1 and §3; lab [6B].
    """
    return (layernorm(h_target, ln_eps) * (1.0 + scale_final)) @ w_out.T


def img_in(x: np.ndarray, w_img_in: np.ndarray) -> np.ndarray:
    """Target tokens = latent x W_img_in, patch size 1 (lab [1A], End-to-end lab §3)."""
    return x @ w_img_in.T


def euler_step(x: np.ndarray, v: np.ndarray, sigma_k: float, sigma_k1: float) -> np.ndarray:
    """x_{k+1} = x_k + (sigma_{k+1} - sigma_k) v (6B page §1)."""
    return x + (float(sigma_k1) - float(sigma_k)) * v


# ---------------------------------------------------------------------------
# Whole-sequence forward, prefix extract, cached step
# ---------------------------------------------------------------------------


@dataclass
class Model:
    """Shapes plus weights (float64 arrays holding the stored values)."""
    n_heads: int
    n_layers: int
    n_chunks: int
    ln_eps: float
    qk_eps: float
    omega: np.ndarray
    wts: Dict[str, np.ndarray]


@dataclass
class Sequence_:
    segments: tuple
    image_ids: np.ndarray
    target_mask: np.ndarray
    coords: np.ndarray
    allowed: np.ndarray
    S: int
    P: int
    N: int


def make_sequence(segments, frame_mode: int = 0) -> Sequence_:
    ids, mask, s, p, n = token_metadata(segments)
    coords = rope_coords(segments, frame_mode)
    return Sequence_(tuple(segments), ids, mask, coords, block_causal_allowed(ids), s, p, n)


def joint_forward(model: Model, seq: Sequence_, prefix_hidden: np.ndarray, x: np.ndarray,
                  mod_prefix: np.ndarray, mod_target: np.ndarray, scale_final: np.ndarray,
                  perturb=None):
    """Full recomputation over all S tokens of one batch item (lab ``forward``, extract).

    prefix_hidden [P, d], x [N, C]; every token runs every block with the
    literal block-causal mask; prefix tokens read ``mod_prefix`` and target
    tokens ``mod_target`` (3B page). ``perturb`` = list of (token, dim, delta)
    added to the joint input (lab checks, isolation experiment).
    Returns dict(v [N, C], h_final [S, d], k [L][S, H, Dh], v_cache [L][S, H, Dh]).
    """
    joint = np.concatenate([prefix_hidden, img_in(x, model.wts["w_img_in"])], axis=0)
    if perturb:
        joint = joint.copy()
        for (idx, dim, delta) in perturb:
            joint[idx, dim] += delta
    mods = select_modulation_rows(seq.target_mask, split_chunks(mod_prefix, model.n_chunks),
                                  split_chunks(mod_target, model.n_chunks))
    h = joint
    ks, vs = [], []
    for l in range(model.n_layers):
        out = dit_block(h, mods, layer_weights(model.wts, l), model.n_heads, seq.coords,
                        model.omega, None, seq.allowed, model.ln_eps, model.qk_eps)
        h = out.h
        ks.append(out.k_rot)
        vs.append(out.v)
    v = final_velocity(h[seq.P:], scale_final, model.wts["w_out"], model.ln_eps)
    return {"v": v, "h_final": h, "k": ks, "v_cache": vs}


def prefix_extract(model: Model, seq: Sequence_, prefix_hidden: np.ndarray,
                   mod_prefix: np.ndarray):
    """K/V of the prefix tokens for every layer (lab [6A], mode "extract").

    Runs the blocks over the P prefix rows only with the block-causal mask
    restricted to them. Prefix rows never attend to target keys (target is
    last, and its id differs), so this equals the prefix part of the joint pass.
    Returns (K [L, P, H, Dh], V [L, P, H, Dh]).
    """
    p = seq.P
    mods = split_chunks(mod_prefix, model.n_chunks)
    h = prefix_hidden
    ks, vs = [], []
    for l in range(model.n_layers):
        out = dit_block(h, mods, layer_weights(model.wts, l), model.n_heads, seq.coords[:p],
                        model.omega, None, seq.allowed[:p, :p], model.ln_eps, model.qk_eps)
        h = out.h
        ks.append(out.k_rot)
        vs.append(out.v)
    return np.stack(ks), np.stack(vs)


def cached_step(model: Model, seq: Sequence_, cache_k: np.ndarray, cache_v: np.ndarray,
                x: np.ndarray, mod_target: np.ndarray, scale_final: np.ndarray):
    """v_theta for the N target tokens using the prefix cache (lab [6A], mode "cached").

    Only the target rows run the blocks; their keys are [cached prefix; own].
    The target rows' mask row allows all P + N keys (target is last).
    Returns (v [N, C], target K [L, N, H, Dh], target V [L, N, H, Dh]): the K/V
    rows this step appends to each layer's cache after the prefix.
    """
    p, n = seq.P, seq.N
    mods = split_chunks(mod_target, model.n_chunks)
    h = img_in(x, model.wts["w_img_in"])
    allowed = seq.allowed[p:, :]
    tk, tv = [], []
    for l in range(model.n_layers):
        out = dit_block(h, mods, layer_weights(model.wts, l), model.n_heads, seq.coords[p:],
                        model.omega, (cache_k[l], cache_v[l]), allowed, model.ln_eps, model.qk_eps)
        h = out.h
        tk.append(out.k_rot)
        tv.append(out.v)
    v = final_velocity(h, scale_final, model.wts["w_out"], model.ln_eps)
    return v, np.stack(tk), np.stack(tv)


def run_image(model: Model, seq: Sequence_, prefix_hidden: np.ndarray, x0: np.ndarray,
              sigmas: Sequence[float], use_cache: bool, causal_condition: bool = True,
              mod_fn=None):
    """The denoising loop of one batch item (lab ``run_pipeline``).

    ``mod_fn(t) -> (mod_row, scale_final)`` defaults to :func:`modulation`.
    With ``use_cache`` the first step extracts the prefix cache and the later
    steps run cached; otherwise every step recomputes all S tokens.
    ``causal_condition=False`` makes the prefix read the t_step row (3B page §3).
    Returns dict(velocities, xs, cache_k, cache_v, modes).
    """
    if mod_fn is None:
        def mod_fn(t):
            return modulation(t, model.wts, model.n_chunks)
    x = x0
    vels, xs, modes = [], [], []
    ck = cv = None
    mod0, _ = mod_fn(0.0)
    for k in range(len(sigmas) - 1):
        t = 1000.0 * float(sigmas[k])
        mod_t, sf = mod_fn(t)
        mod_p = mod0 if causal_condition else mod_t
        if use_cache and k == 0:
            ck, cv = prefix_extract(model, seq, prefix_hidden, mod_p)
        if use_cache:
            v = cached_step(model, seq, ck, cv, x, mod_t, sf)[0]
            modes.append("extract" if k == 0 else "cached")
        else:
            v = joint_forward(model, seq, prefix_hidden, x, mod_p, mod_t, sf)["v"]
            modes.append("extract")
        vels.append(v)
        x = euler_step(x, v, sigmas[k], sigmas[k + 1])
        xs.append(x)
    return {"velocities": vels, "xs": xs, "cache_k": ck, "cache_v": cv, "modes": modes}


def kv_limit_from_mask(allowed: np.ndarray) -> np.ndarray:
    """Row limits of a mask whose every row is a prefix [0, limit); raises otherwise."""
    lim = allowed.sum(axis=1)
    for q in range(allowed.shape[0]):
        if not (allowed[q, :lim[q]].all() and not allowed[q, lim[q]:].any()):
            raise ValueError(f"row {q} of the mask is not a prefix")
    return lim.astype(np.int64)
