"""The parity tests can fail: a guard on their inputs, run on the CPU.

For every workload the GPU parity tests compare with the oracle, replacing the
oracle's attention output by zeros (a planted mistake, on the CPU) must move
every tensor those tests compare by at least ten times the tolerance it is
compared with: 10 x 2e-2 relative L2 (bf16) and 10 x 1e-4 max relative error
(fp32). The compared tensors are the prefix K/V of every layer >= 1 (the
extract's masked attention feeds them), the target K/V of every layer >= 1 of
each cached step (the cached attention over prefix + target keys feeds them),
v_theta of each step, and the final latent of a whole 8-step image. Layer 0's
K/V and the latent after one Euler step (x + dsigma v with |dsigma| ~ 0.02)
do not depend on the attention by construction and are excluded.
"""
import dataclasses

import numpy as np
import pytest

from oracle import qi21_oracle as O
from qi21_synth import configs as C
from tests._harness import BF16_TOL, F32_TOL, max_rel, oracle_item, oracle_model, rel_l2

FACTOR = 10.0


def _outputs(w, n_steps, items, zero_attention, monkeypatch):
    model, _ = oracle_model(w, "bfloat16")
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    with monkeypatch.context() as m:
        if zero_attention:
            m.setattr(O, "masked_softmax_attention", lambda q, k, v, allowed: np.zeros_like(q))
        return [oracle_item(model, seq, pre[b], x0[b], w.sigmas, n_steps) for b in items]


def _assert_moves(a, b, what):
    assert rel_l2(b, a) >= FACTOR * BF16_TOL, f"{what}: zeroed attention moves it by {rel_l2(b, a):.3g} rel-L2"
    assert max_rel(b, a) >= FACTOR * F32_TOL, f"{what}: zeroed attention moves it by {max_rel(b, a):.3g} max-rel"


CASES = [
    # (label, workload, cached steps compared, items)
    ("small", C.make_workload("small"), 3, (0, 1)),
    ("small64", C.make_workload("small64"), 3, (0, 1)),
    ("small_t1", C.make_workload("small_t1"), 3, (0,)),
    ("shared prefix (small, 3 requests)", dataclasses.replace(C.make_workload("small"), batch=3), 2, (0, 1, 2)),
    ("mid", dataclasses.replace(C.parity_workload("mid"), batch=1), 1, (0,)),
    ("toy_parity", C.parity_workload("toy"), 3, (0,)),
]


@pytest.mark.parametrize("label,w,n_steps,items", CASES, ids=[c[0] for c in CASES])
def test_zeroed_attention_moves_every_compared_tensor(monkeypatch, label, w, n_steps, items):
    if label.startswith("shared"):
        # requests share the prefix of item 0 (the shared-prefix tests extract it once)
        one = dataclasses.replace(w, batch=1)
        pre1 = C.host_prefix_hidden(one)
        model, _ = oracle_model(w, "bfloat16")
        seq = O.make_sequence(w.segments)
        x0 = C.host_noise(w)
        outs = []
        for zero in (False, True):
            with monkeypatch.context() as m:
                if zero:
                    m.setattr(O, "masked_softmax_attention", lambda q, k, v, allowed: np.zeros_like(q))
                outs.append([oracle_item(model, seq, pre1[0], x0[b], w.sigmas, n_steps) for b in items])
        ref, mut = outs
    else:
        ref = _outputs(w, n_steps, items, False, monkeypatch)
        mut = _outputs(w, n_steps, items, True, monkeypatch)
    n_layers = w.shape.n_layers
    assert n_layers >= 2
    for i, b in enumerate(items):
        a, z = ref[i], mut[i]
        for l in range(1, n_layers):
            _assert_moves(a["ck"][l], z["ck"][l], f"{label} item {b} prefix K layer {l}")
            _assert_moves(a["cv"][l], z["cv"][l], f"{label} item {b} prefix V layer {l}")
        for k in range(n_steps):
            for l in range(1, n_layers):
                _assert_moves(a["tk"][k][l], z["tk"][k][l], f"{label} item {b} target K step {k} layer {l}")
                _assert_moves(a["tv"][k][l], z["tv"][k][l], f"{label} item {b} target V step {k} layer {l}")
            _assert_moves(a["v"][k], z["v"][k], f"{label} item {b} v step {k}")


def test_zeroed_attention_moves_the_final_latent_of_an_image(monkeypatch):
    """The whole-image tests compare the latent after all 8 Turbo steps."""
    w = dataclasses.replace(C.make_workload("small"), batch=1)
    n = len(w.sigmas) - 1
    a = _outputs(w, n, (0,), False, monkeypatch)[0]["x"][-1]
    z = _outputs(w, n, (0,), True, monkeypatch)[0]["x"][-1]
    _assert_moves(a, z, "final latent")


def test_benchmark_recipe_would_hide_the_attention(monkeypatch):
    """Why the parity recipe exists: with every weight at N(0, 0.02) the
    modulation gates are ~1e-2 and zeroing the attention moves v_theta by less
    than the bf16 tolerance, so a test on those inputs could not fail."""
    w = dataclasses.replace(C.make_workload("small"), std_overrides=(), batch=1)
    a = _outputs(w, 1, (0,), False, monkeypatch)[0]["v"][0]
    z = _outputs(w, 1, (0,), True, monkeypatch)[0]["v"][0]
    assert rel_l2(z, a) < BF16_TOL
