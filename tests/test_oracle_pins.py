"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every oracle function has at least one check here that does not retype its
own formula: page-printed values (tests/golden, each with its citation),
closed forms, library routines (torch fp64), brute force over tiny inputs, or
an invariant such as cache equivalence. ``test_oracle_mutations.py`` plants
plausible mistakes in the oracle and shows that these pins catch them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import qi21_oracle as O
from oracle import lab_replay as LR
from qi21_synth import configs as C


# ---------------------------------------------------------------- metadata

def test_toy_sequence_matches_page(golden):
    g = golden("toy_sequence.json")
    segs = [tuple(s) for s in g["segments"]]
    ids, mask, s, p, n = O.token_metadata(segs)
    assert ids.tolist() == g["image_ids"]
    assert mask.tolist() == g["target_mask"]
    assert (s, p, n) == (g["S"], g["P"], g["N"])
    # length = text tokens + 4 * total image slots (2A page §3): 3 text + 4*(1+1)
    assert s == 3 + 4 * 2


def test_mask_row_counts_match_page(golden):
    g = golden("toy_sequence.json")
    allowed = O.block_causal_allowed(np.array(g["image_ids"]))
    assert allowed.sum(axis=1).tolist() == g["mask_row_key_counts"]
    assert int(allowed.sum()) == 78
    # target rows never lose a key; no prefix row sees a target key
    assert not allowed[:7, 7:].any()


def test_rope_coords_match_page(golden):
    g = golden("toy_sequence.json")
    coords = O.rope_coords([tuple(s) for s in g["segments"]])
    text_pos = [0, 1, 6]
    assert coords[text_pos].tolist() == g["coords_text"]
    assert coords[2:6].tolist() == g["coords_image_grid"]
    assert coords[7:11].tolist() == g["coords_image_grid"]


def test_rope_coords_large_grid_centring():
    coords = O.rope_coords([(O.SEG_TEXT, 3, 0), (O.SEG_IMAGE, 64, 64)])
    img = coords[3:]
    assert img[:, 1].min() == -32 and img[:, 1].max() == 31
    assert img[:, 2].min() == -32 and img[:, 2].max() == 31
    # row-major: width is the inner index
    assert img[1].tolist() == [0, -32, -31] and img[64].tolist() == [0, -31, -32]
    fm = O.rope_coords([(O.SEG_IMAGE, 2, 2), (O.SEG_TEXT, 1, 0), (O.SEG_IMAGE, 2, 2)], frame_mode=1)
    assert fm[:, 0].tolist() == [0, 0, 0, 0, 0, 1, 1, 1, 1]


@pytest.mark.parametrize("seed", range(20))
def test_kv_limit_is_exact_for_segment_layouts(seed):
    rng = np.random.default_rng(seed)
    segs = []
    for _ in range(rng.integers(1, 5)):
        if rng.random() < 0.5:
            segs.append((O.SEG_TEXT, int(rng.integers(1, 5)), 0))
        else:
            segs.append((O.SEG_IMAGE, int(rng.integers(1, 4)), int(rng.integers(1, 4))))
    segs.append((O.SEG_IMAGE, int(rng.integers(1, 4)), int(rng.integers(1, 4))))
    ids, _, s, p, n = O.token_metadata(segs)
    allowed = O.block_causal_allowed(ids)
    lim = O.kv_limit_from_mask(allowed)
    # brute-force definition: text rows q+1, image rows the end of their run
    for q in range(s):
        if ids[q] < 0:
            assert lim[q] == q + 1
        else:
            run_end = max(i for i in range(s) if ids[i] == ids[q]) + 1
            assert lim[q] == run_end
    assert (lim[p:] == s).all()


# ---------------------------------------------------------------- sigmas / Euler

def test_turbo_delta_sigma_matches_page(golden):
    g = golden("turbo_sigmas.json")
    sig = np.array(g["sigmas"])
    d = np.diff(sig)
    assert np.allclose(-d, g["abs_delta_sigma"], atol=5e-7)
    assert math.isclose(float(-d.sum()), g["abs_delta_sum"], abs_tol=1e-12)
    assert round(float(-d[0]), 4) == 0.0215 and round(float(-d[-1]), 4) == 0.4146
    assert tuple(sig) == C.TURBO_SIGMAS
    lab = np.diff(np.array(g["lab_sigmas"]))
    assert np.allclose(lab, g["lab_delta_sigma"], atol=1e-15)


def test_euler_constant_velocity_reaches_x0_minus_v(golden):
    sig = golden("turbo_sigmas.json")["sigmas"]
    x0 = np.linspace(-1, 1, 12).reshape(3, 4)
    v = np.arange(12.0).reshape(3, 4) / 7.0
    x = x0
    for k in range(8):
        x = O.euler_step(x, v, sig[k], sig[k + 1])
    np.testing.assert_allclose(x, x0 - v, atol=1e-14)
    # one step is a straight move by (sigma_{k+1} - sigma_k) along v
    np.testing.assert_allclose(O.euler_step(x0, v, 1.0, 0.85), x0 - 0.15 * v, atol=1e-15)


# ---------------------------------------------------------------- RoPE

def _complex_rope(x, coords, omega):
    # independent formulation: pairs as complex numbers times e^{i angle}
    z = x[..., 0::2] + 1j * x[..., 1::2]
    out = np.empty_like(x)
    for s in range(coords.shape[0]):
        for j in range(omega.shape[0]):
            ang = sum(float(coords[s, a]) * float(omega[j, a]) for a in range(3))
            r = z[..., s, j] * complex(math.cos(ang), math.sin(ang))
            out[..., s, 2 * j] = r.real
            out[..., s, 2 * j + 1] = r.imag
    return out


def test_rope_against_complex_multiplication():
    rng = np.random.default_rng(0)
    coords = np.array([[0, 0, 0], [3, -2, 5], [1, 31, -32], [7, 7, 7]])
    for omega in (O.rope_omega_axial(32), O.rope_omega_lab()):
        x = rng.normal(size=(2, 4, omega.shape[0] * 2))
        np.testing.assert_allclose(O.rope_rotate(x, coords, omega), _complex_rope(x, coords, omega),
                                   atol=1e-13)


def test_rope_invariants():
    rng = np.random.default_rng(1)
    omega = O.rope_omega_axial(128)
    assert omega.shape == (64, 3)
    # 8 frame pairs, 28 height pairs, 28 width pairs, each starting at rate 1
    assert (omega[:8, 0] > 0).all() and (omega[8:36, 1] > 0).all() and (omega[36:, 2] > 0).all()
    assert omega[0, 0] == 1.0 and omega[8, 1] == 1.0 and omega[36, 2] == 1.0
    assert np.count_nonzero(omega) == 64
    coords = rng.integers(-40, 40, size=(6, 3))
    q = rng.normal(size=(1, 6, 128))
    k = rng.normal(size=(1, 6, 128))
    rq = O.rope_rotate(q, coords, omega)
    rk = O.rope_rotate(k, coords, omega)
    # norm preserving
    np.testing.assert_allclose(np.linalg.norm(rq, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-13)
    # identity at the origin
    zero = np.zeros((1, 3), dtype=np.int64)
    np.testing.assert_array_equal(O.rope_rotate(q[:, :1], zero, omega), q[:, :1])
    # <R(p) q, R(p') k> depends only on p - p'
    shift = np.array([[5, -3, 11]])
    rq2 = O.rope_rotate(q, coords + shift, omega)
    rk2 = O.rope_rotate(k, coords + shift, omega)
    np.testing.assert_allclose(np.einsum("hsd,htd->st", rq, rk), np.einsum("hsd,htd->st", rq2, rk2),
                               atol=1e-11)


# ---------------------------------------------------------------- norms, activations

def test_layernorm_against_torch_and_constant_rows():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(5, 64)) * 3 + 1
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (64,), eps=1e-6).numpy()
    np.testing.assert_allclose(O.layernorm(x, 1e-6), ref, atol=1e-12)
    np.testing.assert_array_equal(O.layernorm(np.full((2, 8), 3.5), 1e-6), np.zeros((2, 8)))


def test_rmsnorm_against_torch():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(3, 7, 16))
    w = rng.normal(size=16) * 0.3
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (16,), weight=torch.from_numpy(1.0 + w),
                                       eps=1e-6).numpy()
    np.testing.assert_allclose(O.rmsnorm_zero_centre(x, w, 1e-6), ref, atol=1e-12)


def test_silu_against_torch():
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(O.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(),
                               atol=1e-14)


# ---------------------------------------------------------------- attention

def _attention_loops(q, k, v, allowed):
    h_, sq, dh = q.shape
    out = np.zeros_like(q)
    for h in range(h_):
        for i in range(sq):
            scores = []
            for j in range(k.shape[1]):
                if allowed[i, j]:
                    scores.append((j, sum(q[h, i, t] * k[h, j, t] for t in range(dh)) / math.sqrt(dh)))
            m = max(s for _, s in scores)
            z = sum(math.exp(s - m) for _, s in scores)
            for j, s in scores:
                out[h, i] += math.exp(s - m) / z * v[h, j]
    return out


def test_attention_against_loops():
    rng = np.random.default_rng(4)
    ids = np.array([-1, -1, 0, 0, 0, -1, 1, 1])
    allowed = O.block_causal_allowed(ids)
    q = rng.normal(size=(2, 8, 4))
    k = rng.normal(size=(2, 8, 4))
    v = rng.normal(size=(2, 8, 4))
    np.testing.assert_allclose(O.masked_softmax_attention(q, k, v, allowed),
                               _attention_loops(q, k, v, allowed), atol=1e-13)


def test_attention_special_cases():
    rng = np.random.default_rng(5)
    q = rng.normal(size=(1, 3, 4))
    k = rng.normal(size=(1, 3, 4))
    v = rng.normal(size=(1, 3, 4))
    only_first = np.zeros((3, 3), dtype=bool)
    only_first[:, 0] = True
    np.testing.assert_array_equal(O.masked_softmax_attention(q, k, v, only_first)[0],
                                  np.repeat(v[0, :1], 3, axis=0))
    # equal scores -> plain mean of the allowed values
    same = O.masked_softmax_attention(np.zeros((1, 3, 4)), k, v, np.ones((3, 3), dtype=bool))
    np.testing.assert_allclose(same[0], np.repeat(v[0].mean(axis=0, keepdims=True), 3, 0), atol=1e-15)


# ---------------------------------------------------------------- output head and img_in

def test_final_velocity_closed_forms():
    """6B page §1 and §3: v = (LN(h)(1 + scale_final)) W_out, scale-only (no
    shift, no bias). Two rows whose LayerNorm is known in closed form:
    an alternating row (+a, -a, ...) has mean 0 and variance a^2, so LN gives
    +-a / sqrt(a^2 + eps); the row 1, 2, ..., 8 has mean 4.5 and biased
    variance (8^2 - 1) / 12 = 5.25. W_out picks dimension (c + 1) mod 8 for
    output c (a cyclic shift, so W_out and its transpose differ), which makes
    v[c] = LN(h)[j] (1 + s[j]) with j = (c + 1) mod 8."""
    d, a, eps = 8, 2.0, 1e-6
    h = np.array([[a, -a] * 4, list(range(1, 9))], dtype=np.float64)
    s = np.array([0.5, -0.25, 2.0, 0.0, -1.5, 0.75, 1.0, -0.5])
    w_out = np.zeros((d, d))
    for c in range(d):
        w_out[c, (c + 1) % d] = 1.0
    ln0 = np.array([1.0, -1.0] * 4) * a / math.sqrt(a * a + eps)
    ln1 = (np.arange(1, 9) - 4.5) / math.sqrt(5.25 + eps)
    for row, ln in ((0, ln0), (1, ln1)):
        want = np.array([ln[(c + 1) % d] * (1.0 + s[(c + 1) % d]) for c in range(d)])
        np.testing.assert_allclose(O.final_velocity(h[row:row + 1], s, w_out, eps)[0], want, rtol=1e-13,
                                   atol=1e-15)
    # scale_final = 0 leaves the plain LayerNorm through W_out
    np.testing.assert_allclose(O.final_velocity(h[1:], np.zeros(d), w_out, eps)[0], np.roll(ln1, -1),
                               rtol=1e-13)


def test_img_in_hand_worked():
    """img_in with patch size 1 (lab [1A]; End-to-end lab §3): token = latent
    times W_img_in^T, W_img_in [d][C]. Worked by hand for C = 3, d = 4."""
    x = np.array([[1.0, 2.0, 3.0], [0.0, -1.0, 2.0]])
    w_img_in = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 0.0], [0.0, 0.0, 1.0], [1.0, 1.0, 1.0]])
    np.testing.assert_array_equal(O.img_in(x, w_img_in), np.array([[1.0, 2.0, 3.0, 6.0], [0.0, -1.0, 2.0, 1.0]]))
    w2 = np.array([[2.0, -1.0, 0.5], [0.0, 0.0, 0.0], [1.0, 1.0, -1.0], [0.0, 3.0, 0.0]])
    np.testing.assert_array_equal(O.img_in(x, w2), np.array([[1.5, 0.0, 0.0, 6.0], [2.0, 0.0, -3.0, -3.0]]))


# ---------------------------------------------------------------- modulation

def test_timestep_embedding_closed_forms():
    e0 = O.timestep_embedding(0.0, 256)
    np.testing.assert_array_equal(e0, np.concatenate([np.ones(128), np.zeros(128)]))
    e = O.timestep_embedding(850.0, 256)
    assert math.isclose(e[0], math.cos(850.0), abs_tol=1e-15)       # frequency 1 first
    assert math.isclose(e[128], math.sin(850.0), abs_tol=1e-15)
    np.testing.assert_allclose(e[:128] ** 2 + e[128:] ** 2, np.ones(128), atol=1e-15)


def test_modulation_identity_weights_closed_form():
    d = 8
    eye = np.eye(d)
    wts = {"w_t1": eye, "w_t2": eye, "w_mod": np.vstack([eye] * 4), "w_fin": 2 * eye}
    mod, sf = O.modulation(0.0, wts, 4)
    s1 = 1.0 / (1.0 + math.exp(-1.0))            # silu(1)
    a = s1 / (1.0 + math.exp(-s1))               # silu(silu(1))
    expect = np.array([a] * 4 + [0.0] * 4)       # emb(0) = [1,1,1,1,0,0,0,0]
    np.testing.assert_allclose(mod, np.tile(expect, 4), atol=1e-15)
    np.testing.assert_allclose(sf, 2 * expect, atol=1e-15)
    ch = O.split_chunks(np.arange(24.0), 6)
    assert ch["shift1"][0] == 0 and ch["scale1"][0] == 4 and ch["gate2"][0] == 20
    ch4 = O.split_chunks(np.arange(16.0), 4)
    assert ch4["gate1"][0] == 4 and ch4["scale2"][0] == 8 and not ch4["shift2"].any()


def test_modulation_parameter_count(golden):
    g = golden("modulation.json")
    shapes = dict(C.weight_specs(C.FULL))
    assert shapes["w_mod"] == (g["n_chunks"] * g["d_model"], g["d_model"])
    assert shapes["w_mod"][0] * shapes["w_mod"][1] == g["params"]


def test_prefix_row_is_identical_across_steps():
    w = C.make_workload("toy")
    wts = C.host_weights(w)
    a, _ = O.modulation(0.0, wts, 4)
    b, _ = O.modulation(0.0, wts, 4)
    assert np.max(np.abs(a - b)) == 0.0
    r1, _ = O.modulation(1000.0, wts, 4)
    r2, _ = O.modulation(850.0, wts, 4)
    assert np.max(np.abs(r1 - r2)) > 1e-6


# ---------------------------------------------------------------- lab replay (page numbers)

def test_lab_replay_prefix_k_drift_matches_page(golden):
    g = golden("lab_checks.json")
    w = LR.draw_lab_weights()
    drift = LR.prefix_k_drift(w, np.array(g["demo_rgba"]))
    assert [float(f"{d:.3g}") for d in drift] == g["prefix_k_drift_3sf"]


def _lab_pipelines(g):
    w = LR.draw_lab_weights()
    model = LR.lab_model(w)
    seq = O.make_sequence(LR.SEGMENTS)
    pre = LR.prefix_tokens(w, np.array(g["demo_rgba"]))
    f = LR.lab_mod_fn(w)
    cached = O.run_image(model, seq, pre, w["noise"], LR.SIGMAS, True, mod_fn=f)
    recomp = O.run_image(model, seq, pre, w["noise"], LR.SIGMAS, False, mod_fn=f)
    return w, model, seq, pre, f, cached, recomp


def test_lab_cached_equals_recompute(golden):
    g = golden("lab_checks.json")
    w, model, seq, pre, f, cached, recomp = _lab_pipelines(g)
    assert cached["modes"] == ["extract", "cached", "cached"]
    for step in (1, 2):
        assert np.max(np.abs(cached["velocities"][step] - recomp["velocities"][step])) < g["cache_threshold"]
    assert np.max(np.abs(cached["xs"][-1] - recomp["xs"][-1])) < g["cache_threshold"]
    # prefix K cached at step 1 vs the prefix K a recompute produces at step 2
    x1 = recomp["xs"][0]
    mod_t, sf = f(1000.0 * LR.SIGMAS[1])
    joint = O.joint_forward(model, seq, pre, x1, f(0.0)[0], mod_t, sf)
    for l in range(LR.N_LAYERS):
        assert np.max(np.abs(cached["cache_k"][l] - joint["k"][l][:seq.P])) < g["cache_threshold"]
    assert cached["cache_k"].shape == (2, 7, 2, 4)


def test_lab_isolation(golden):
    g = golden("lab_checks.json")
    w, model, seq, pre, f, _, _ = _lab_pipelines(g)
    mod_t, sf = f(1000.0)
    base = O.joint_forward(model, seq, pre, w["noise"], f(0.0)[0], mod_t, sf)["h_final"]
    pt = O.joint_forward(model, seq, pre, w["noise"], f(0.0)[0], mod_t, sf,
                         perturb=[(g["isolation_target_token"], 0, 0.5)])["h_final"]
    assert np.max(np.abs(pt[:7] - base[:7])) == 0.0
    assert np.max(np.abs(pt[7:] - base[7:])) > 0.0
    pc = O.joint_forward(model, seq, pre, w["noise"], f(0.0)[0], mod_t, sf,
                         perturb=[(g["isolation_cond_token"], 0, 0.5)])["h_final"]
    d2 = np.abs(pc - base).max(axis=1)
    assert (d2[2:6] > 0).all()
    assert d2[0] == 0.0 and d2[1] == 0.0


def test_lab_t0_row_change_is_zero(golden):
    g = golden("lab_checks.json")
    w = LR.draw_lab_weights()
    f = LR.lab_mod_fn(w)
    assert float(np.max(np.abs(f(0.0)[0] - f(0.0)[0]))) == g["t0_row_change"]
    assert np.max(np.abs(f(1000.0)[0] - f(850.0)[0])) > 0


# ---------------------------------------------------------------- production reading, synthetic weights

def _toy_model_and_inputs(name="toy"):
    w = C.make_workload(name)
    sh = w.shape
    wts = C.host_weights(w, "float32")
    omega = O.rope_omega_lab() if sh.rope == "lab" else O.rope_omega_axial(sh.head_dim)
    model = O.Model(sh.n_heads, sh.n_layers, sh.n_chunks, sh.ln_eps, sh.qk_eps, omega, wts)
    seq = O.make_sequence(w.segments)
    return w, model, seq, C.host_prefix_hidden(w), C.host_noise(w)


def test_toy_cached_equals_recompute_and_causal_drift():
    w, model, seq, pre, x0 = _toy_model_and_inputs()
    c = O.run_image(model, seq, pre[0], x0[0], w.sigmas, True)
    r = O.run_image(model, seq, pre[0], x0[0], w.sigmas, False)
    for a, b in zip(c["velocities"], r["velocities"]):
        assert np.max(np.abs(a - b)) < 1e-9
    assert np.max(np.abs(c["xs"][-1] - r["xs"][-1])) < 1e-9
    # prefix reading t_step instead of t = 0: K drifts between steps
    m1, _ = O.modulation(1000.0, model.wts, 4)
    m2, _ = O.modulation(850.0, model.wts, 4)
    k1, _ = O.prefix_extract(model, seq, pre[0], m1)
    k2, _ = O.prefix_extract(model, seq, pre[0], m2)
    for l in range(model.n_layers):
        assert np.max(np.abs(k1[l] - k2[l])) > 1e-9


def test_velocity_depends_on_sigma():
    w, model, seq, pre, x0 = _toy_model_and_inputs()
    m0, _ = O.modulation(0.0, model.wts, 4)
    ck, cv = O.prefix_extract(model, seq, pre[0], m0)
    vs = []
    for s in (1.0, 0.7, 0.3):
        mt, sf = O.modulation(1000.0 * s, model.wts, 4)
        vs.append(O.cached_step(model, seq, ck, cv, x0[0], mt, sf)[0])
    for a, b in itertools.combinations(vs, 2):
        assert np.max(np.abs(a - b)) > 1e-8


# ---------------------------------------------------------------------------- joint packing (2A page)
def _random_layouts(n=20, seed=5):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        segs = []
        for _ in range(rng.integers(1, 5)):
            if rng.random() < 0.5:
                segs.append((O.SEG_TEXT, int(rng.integers(1, 6)), 0))
            else:
                segs.append((O.SEG_IMAGE, 2 * int(rng.integers(1, 4)), 2 * int(rng.integers(1, 4))))
        segs.append((O.SEG_IMAGE, 2, 2))                        # target last
        out.append(segs)
    return out


def test_slot_expansion_matches_page_repeats(golden):
    """Lab page 1:1 table, row 2A: repeats = [1, 1, 4, 1] over the slots [text, text, image, text]."""
    g = golden("toy_sequence.json")
    slot_of, img_row, n_slots, n_img = O.slot_expansion([tuple(s) for s in g["segments"]])
    assert slot_of.tolist() == np.repeat(np.arange(4), g["repeats"]).tolist()
    assert img_row.tolist() == [-1, -1, 0, 1, 2, 3, -1]
    assert (n_slots, n_img, len(slot_of)) == (4, 4, g["P"])


def test_packed_length_formula():
    """2A page: length = text tokens + 4 x (image slots), and the packing covers exactly the prefix."""
    for segs in _random_layouts():
        slot_of, img_row, n_slots, n_img = O.slot_expansion(segs)
        n_text = sum(a for k, a, _ in segs[:-1] if k == O.SEG_TEXT)
        image_slots = sum(a * b // 4 for k, a, b in segs[:-1] if k == O.SEG_IMAGE)
        assert len(slot_of) == n_text + 4 * image_slots == O.token_metadata(segs)[3]
        assert n_slots == n_text + image_slots and n_img == 4 * image_slots


def test_slot_expansion_brute_force():
    """Walk the prefix position by position: a text token takes the next slot; an
    image takes the next slot every 4 cells and the next image-token row every cell."""
    for segs in _random_layouts():
        want_slot, want_row = [], []
        slot = row = 0
        for kind, a, b in segs[:-1]:
            if kind == O.SEG_TEXT:
                for _ in range(a):
                    want_slot.append(slot)
                    want_row.append(-1)
                    slot += 1
            else:
                for cell in range(a * b):
                    want_slot.append(slot + cell // 4)
                    want_row.append(row)
                    row += 1
                slot += a * b // 4
        slot_of, img_row, _, _ = O.slot_expansion(segs)
        assert slot_of.tolist() == want_slot and img_row.tolist() == want_row


def test_pack_add_reproduces_the_lab_prefix_rows(golden):
    """Lab [2A]: PREFIX_TOKENS = [txt0, txt1, img_in(cond) + slot2, txt3] — built there by concatenation."""
    g = golden("lab_checks.json")
    w = LR.draw_lab_weights()
    demo = np.array(g["demo_rgba"])
    segs = [tuple(s) for s in golden("toy_sequence.json")["segments"]]
    got = O.pack_prefix(LR.slot_vectors(w), LR.cond_image_tokens(w, demo), segs, O.PACK_ADD)
    assert np.array_equal(got, LR.prefix_tokens(w, demo))


def test_pack_substitute_takes_img_in_at_image_positions():
    """2A page, mechanism (2): image positions hold the img_in token of their cell, text positions their slot."""
    rng = np.random.default_rng(8)
    for segs in _random_layouts(8):
        slot_of, img_row, n_slots, n_img = O.slot_expansion(segs)
        ctx = rng.standard_normal((n_slots, 6))
        img = rng.standard_normal((n_img, 6))
        out = O.pack_prefix(ctx, img, segs, O.PACK_SUBSTITUTE)
        pos = 0
        for kind, a, b in segs[:-1]:
            n = a if kind == O.SEG_TEXT else a * b
            for t in range(n):
                if kind == O.SEG_TEXT:
                    assert np.array_equal(out[pos], ctx[slot_of[pos]])
                else:
                    assert np.array_equal(out[pos], img[img_row[pos]])
                pos += 1
        image_slots = set(slot_of[img_row >= 0].tolist())
        for s_ in image_slots:                       # an image slot's own vector never survives
            assert not any(np.array_equal(r, ctx[s_]) for r in out)
