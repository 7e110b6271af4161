"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances (stated by the target of this work): fp32 storage must match the
fp64 oracle within 1e-4 max relative error (max|a-b| / max|b| per tensor) on
v_theta and the latent; bf16 storage within 2e-2 relative L2. Integer
metadata is bit-exact.
"""
import numpy as np
import pytest
import torch

from oracle import qi21_oracle as O
from qi21_synth import configs as C
from tests._harness import (BF16_TOL, F32_TOL, assert_item_matches, gpu_steps, max_rel, oracle_item,
                            oracle_model, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from prefix_kv_cached_b200 import binding
    return binding


def _runner(w, dtype, wts):
    from prefix_kv_cached_b200.runner import Qi21Runner
    return Qi21Runner(w, dtype, host_weights=wts)


def _oracle_image(model, seq, pre, x0, sigmas, n_steps):
    m0, _ = O.modulation(0.0, model.wts, model.n_chunks)
    ck, cv = O.prefix_extract(model, seq, pre, m0)
    x = x0
    vs, xs = [], []
    for k in range(n_steps):
        mt, sf = O.modulation(1000.0 * sigmas[k], model.wts, model.n_chunks)
        v = O.cached_step(model, seq, ck, cv, x, mt, sf)[0]
        x = O.euler_step(x, v, sigmas[k], sigmas[k + 1])
        vs.append(v)
        xs.append(x)
    return ck, cv, vs, xs, m0


def _gpu_image(r, pre_t, x0_t, sigmas, n_steps):
    r.set_prefix_row()
    r.prefix_extract(pre_t)
    x = x0_t.clone()
    v = torch.empty_like(x)
    vs, xs = [], []
    for k in range(n_steps):
        r.set_target_row(sigmas[k])
        r.cached_step(x, v)
        vs.append(v.double().cpu().numpy())
        r.euler(x, v, sigmas[k], sigmas[k + 1], x)
        xs.append(x.double().cpu().numpy())
    torch.cuda.synchronize()
    r.check_device()
    return vs, xs


@pytest.mark.parametrize("name,n_steps", [("toy", 3), ("toy_parity", 3), ("small", 8), ("small64", 3)])
def test_f32_denoise_matches_oracle(B, name, n_steps):
    """Every layer's prefix K/V, every step's target K/V of every layer, v_theta
    and the latent, F32 storage within 1e-4 max relative error. toy is the
    lab-scale configuration with N(0, 0.02) weights; toy_parity the same shape
    with the parity weight recipe."""
    w = C.parity_workload("toy") if name == "toy_parity" else C.make_workload(name)
    model, wts = oracle_model(w, "float32")
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    r = _runner(w, B.QI21_DTYPE_F32, wts)
    got = gpu_steps(r, torch.from_numpy(pre.astype(np.float32)).cuda(),
                    torch.from_numpy(x0.astype(np.float32)).cuda(), w.sigmas, n_steps)
    for b in range(w.batch):
        want = oracle_item(model, seq, pre[b], x0[b], w.sigmas, n_steps)
        assert_item_matches(got, want, b, n_steps, max_rel, F32_TOL, name)
    assert max_rel(r.mod_prefix.double().cpu().numpy(), want["m0"]) < F32_TOL


@pytest.mark.parametrize("name", ["toy", "small"])
def test_f32_full_recompute_matches_oracle_and_cache(B, name):
    w = C.make_workload(name)
    model, wts = oracle_model(w, "float32")
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    r = _runner(w, B.QI21_DTYPE_F32, wts)
    pre_t = torch.from_numpy(pre.astype(np.float32)).cuda()
    x_t = torch.from_numpy(x0.astype(np.float32)).cuda()
    sigma = w.sigmas[1]
    r.set_prefix_row()
    r.set_target_row(sigma)
    v_full = torch.empty_like(x_t)
    r.full_recompute(pre_t, x_t, v_full)
    r.prefix_extract(pre_t)
    v_cached = torch.empty_like(x_t)
    r.cached_step(x_t, v_cached)
    torch.cuda.synchronize()
    m0, _ = O.modulation(0.0, model.wts, 4)
    mt, sf = O.modulation(1000.0 * sigma, model.wts, 4)
    for b in range(w.batch):
        ref = O.joint_forward(model, seq, pre[b], x0[b], m0, mt, sf)["v"]
        assert max_rel(v_full[b].double().cpu().numpy(), ref) < F32_TOL
    # cache equivalence on the GPU: same math, different launch shapes
    assert max_rel(v_cached.double().cpu().numpy(), v_full.double().cpu().numpy()) < 1e-5


def test_bf16_cuda_core_family_matches_oracle(B):
    w = C.make_workload("small")
    model, wts = oracle_model(w, "bfloat16")
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    B.qi21_set_tensor_cores(0)
    try:
        r = _runner(w, B.QI21_DTYPE_BF16, wts)
        gvs, gxs = _gpu_image(r, torch.from_numpy(pre.astype(np.float32)).cuda(),
                              torch.from_numpy(x0.astype(np.float32)).cuda(), w.sigmas, 3)
    finally:
        B.qi21_set_tensor_cores(1)
    for b in range(w.batch):
        _, _, vs, xs, _ = _oracle_image(model, seq, pre[b], x0[b], w.sigmas, 3)
        for k in range(3):
            assert rel_l2(gvs[k][b], vs[k]) < BF16_TOL
            assert rel_l2(gxs[k][b], xs[k]) < BF16_TOL


def test_euler_update_exact(B):
    n = 1003
    x = torch.randn(n, device="cuda")
    v = torch.randn(n, device="cuda")
    out = torch.empty_like(x)
    B.check("euler", B.qi21_euler_update(x, v, 0.95418, 0.926626, out, n,
                                         torch.cuda.current_stream().cuda_stream))
    dsig = np.float32(0.926626 - 0.95418)
    ref = (x.cpu().numpy() + dsig * v.cpu().numpy()).astype(np.float32)
    got = out.cpu().numpy()
    assert np.max(np.abs(got - ref)) <= 1e-6 * np.max(np.abs(ref))
    # n == 0 is a no-op that succeeds
    assert B.qi21_euler_update(x, v, 1.0, 0.5, out, 0, 0) == B.QI21_OK


def test_degenerate_one_token_image(B):
    shape = C.SMALL
    w = C.Workload("tiny", shape, 1, ((C.SEG_TEXT, 1, 0), (C.SEG_IMAGE, 1, 1)), C.TURBO_SIGMAS, 99)
    model, wts = oracle_model(w, "float32")
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    r = _runner(w, B.QI21_DTYPE_F32, wts)
    gvs, gxs = _gpu_image(r, torch.from_numpy(pre.astype(np.float32)).cuda(),
                          torch.from_numpy(x0.astype(np.float32)).cuda(), w.sigmas, 2)
    _, _, vs, xs, _ = _oracle_image(model, seq, pre[0], x0[0], w.sigmas, 2)
    for k in range(2):
        assert max_rel(gvs[k][0], vs[k]) < F32_TOL
