"""Plant plausible mistakes in the oracle (on the CPU) and show the pins catch them.

Each case rewrites one line of an oracle function's source (a dropped term, a
flipped sign, a transposed operand, a wrong index), installs the mutant in the
oracle module for the duration of the test, and checks that at least one pin
from ``test_oracle_pins.py`` now fails: chiefly the page-printed prefix-K
drift of the lab replay (9.61e-01 / 1.68e+00), which runs the whole block.
"""
import inspect
import textwrap

import numpy as np
import pytest

from oracle import qi21_oracle as O
from oracle import lab_replay as LR
from tests.conftest import load_golden


def _mutant(func, old, new):
    src = textwrap.dedent(inspect.getsource(func))
    assert old in src, f"mutation anchor not found in {func.__name__}: {old!r}"
    src = src.replace(old, new, 1)
    ns = dict(O.__dict__)
    exec(compile(src, f"<mutant {func.__name__}>", "exec"), ns)
    return ns[func.__name__]


def _drift():
    g = load_golden("lab_checks.json")
    d = LR.prefix_k_drift(LR.draw_lab_weights(), np.array(g["demo_rgba"]))
    return [float(f"{x:.3g}") for x in d], g["prefix_k_drift_3sf"]


MUTATIONS = [
    # (function, anchor, replacement)
    ("dit_block", "(1.0 + mods[\"scale1\"])", "(mods[\"scale1\"])"),                     # dropped 1 +
    ("dit_block", "+ mods[\"shift1\"]", "- mods[\"shift1\"]"),                           # sign
    ("dit_block", "x_mod @ lw[\"w_q\"].T", "x_mod @ lw[\"w_q\"]"),                       # transposed operand
    ("dit_block", "np.tanh(mods[\"gate1\"])", "mods[\"gate1\"]"),                        # no tanh
    ("dit_block", "np.tanh(mods[\"gate2\"])", "np.tanh(mods[\"gate1\"])"),               # wrong chunk
    ("dit_block", "silu(x2 @ lw[\"w_gate\"].T) * (x2 @ lw[\"w_up\"].T)",
     "silu(x2 @ lw[\"w_up\"].T) * (x2 @ lw[\"w_gate\"].T)"),                             # gate/up swapped
    ("dit_block", "k = rope_rotate(k, coords, omega)", "k = k"),                         # RoPE dropped on k
    ("dit_block", "lw[\"k_norm\"]", "lw[\"q_norm\"]"),                                   # wrong norm weight
    ("rope_rotate", "x0 * s + x1 * c", "x0 * s - x1 * c"),                               # sign in rotation
    ("rope_rotate", "out[..., 0::2] = x0 * c - x1 * s", "out[..., 0::2] = x0 * c + x1 * s"),
    ("layernorm", "((x - mu) ** 2).mean(axis=-1, keepdims=True)",
     "((x - mu) ** 2).sum(axis=-1, keepdims=True) / (x.shape[-1] - 1)"),                 # unbiased var
    ("rmsnorm_zero_centre", "* (1.0 + w)", "* w"),                                      # dropped 1 +
    ("masked_softmax_attention", "/ np.sqrt(dh)", ""),                                   # dropped scale
    ("block_causal_allowed", "(q >= kv) or same", "(q <= kv) or same"),                  # transposed mask
    ("rope_coords", "coords.append((f, r - a // 2, c - b // 2))",
     "coords.append((f, c - b // 2, r - a // 2))"),                                      # h/w swapped
    ("split_chunks", "names = (\"shift1\", \"scale1\", \"gate1\", \"shift2\", \"scale2\", \"gate2\")",
     "names = (\"shift1\", \"gate1\", \"scale1\", \"shift2\", \"scale2\", \"gate2\")"),  # chunk order
    ("timestep_embedding", "np.concatenate([np.cos(ang), np.sin(ang)])",
     "np.concatenate([np.sin(ang), np.cos(ang)])"),                                      # sin/cos order
]


@pytest.mark.parametrize("fname,old,new", MUTATIONS, ids=[f"{m[0]}:{i}" for i, m in enumerate(MUTATIONS)])
def test_pin_catches_mutation(monkeypatch, fname, old, new):
    monkeypatch.setattr(O, fname, _mutant(getattr(O, fname), old, new))
    got, want = _drift()
    caught = got != want
    g = load_golden("toy_sequence.json")
    if not caught and fname == "block_causal_allowed":
        ids = np.array(g["image_ids"])
        caught = O.block_causal_allowed(ids).sum(axis=1).tolist() != g["mask_row_key_counts"]
    if not caught and fname == "rope_coords":
        # the lab's height/width rates are ~1e-4 rad, so the page's coordinate table is the pin
        coords = O.rope_coords([tuple(s) for s in g["segments"]])
        caught = coords[2:6].tolist() != g["coords_image_grid"]
    assert caught, f"mutation in {fname} not caught: drift {got}"


def test_euler_sign_mutation_caught(monkeypatch):
    monkeypatch.setattr(O, "euler_step", _mutant(O.euler_step, "(float(sigma_k1) - float(sigma_k))",
                                                 "(float(sigma_k) - float(sigma_k1))"))
    x0 = np.ones(4)
    v = np.full(4, 0.5)
    sig = load_golden("turbo_sigmas.json")["sigmas"]
    x = x0
    for k in range(8):
        x = O.euler_step(x, v, sig[k], sig[k + 1])
    assert not np.allclose(x, x0 - v)


PACK_MUTATIONS = [
    ("slot_expansion", "repeats += [IMG_TOKENS_PER_SLOT] * (cells // IMG_TOKENS_PER_SLOT)",
     "repeats += [1] * (cells // IMG_TOKENS_PER_SLOT)"),                                  # no 4x expansion
    ("slot_expansion", "img_row += list(range(n_img, n_img + cells))",
     "img_row += list(range(n_img + cells - 1, n_img - 1, -1))"),                         # cells reversed
    ("pack_prefix", "out[m] = img_tokens[img_row[m]]", "out[m] = out[m] + img_tokens[img_row[m]]"),  # add
    ("pack_prefix", "out[m] = out[m] + img_tokens[img_row[m]]", "out[m] = img_tokens[img_row[m]]"),  # replace
]


@pytest.mark.parametrize("fname,old,new", PACK_MUTATIONS, ids=[f"{m[0]}:{i}" for i, m in enumerate(PACK_MUTATIONS)])
def test_packing_pins_catch_mutation(monkeypatch, fname, old, new):
    from tests import test_oracle_pins as P
    from tests.conftest import load_golden as lg
    monkeypatch.setattr(O, fname, _mutant(getattr(O, fname), old, new))
    pins = [lambda: P.test_slot_expansion_matches_page_repeats(lg), P.test_packed_length_formula,
            P.test_slot_expansion_brute_force, lambda: P.test_pack_add_reproduces_the_lab_prefix_rows(lg),
            P.test_pack_substitute_takes_img_in_at_image_positions]
    failed = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, IndexError, ValueError):   # a pin that fails or breaks catches it
            failed += 1
    assert failed > 0, f"mutation in {fname} not caught by any packing pin"


HEAD_MUTATIONS = [
    ("final_velocity", "(1.0 + scale_final)", "(scale_final)"),                          # dropped 1 +
    ("final_velocity", "(1.0 + scale_final))", "(1.0 + scale_final) + scale_final)"),    # added shift
    ("final_velocity", "@ w_out.T", "@ w_out"),                                          # transposed W_out
    ("final_velocity", "layernorm(h_target, ln_eps)", "h_target"),                       # LN dropped
    ("img_in", "return x @ w_img_in.T", "return 2.0 * (x @ w_img_in.T)"),                # doubled img_in
    ("img_in", "return x @ w_img_in.T", "return x @ w_img_in[::-1].T"),                  # wrong row order
]


@pytest.mark.parametrize("fname,old,new", HEAD_MUTATIONS, ids=[f"{m[0]}:{i}" for i, m in enumerate(HEAD_MUTATIONS)])
def test_head_pins_catch_mutation(monkeypatch, fname, old, new):
    from tests import test_oracle_pins as P
    monkeypatch.setattr(O, fname, _mutant(getattr(O, fname), old, new))
    failed = 0
    for pin in (P.test_final_velocity_closed_forms, P.test_img_in_hand_worked):
        try:
            pin()
        except (AssertionError, ValueError):
            failed += 1
    assert failed > 0, f"mutation in {fname} not caught by the output-head pins"
