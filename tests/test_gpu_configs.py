"""BF16 tensor-core path at the benchmark's own sizes.

* mid (d 1024, 8 blocks, batch 8, P 512, N 256): extract + one cached step +
  Euler against the fp64 oracle, relative L2 < 2e-2 (exercises split-K of the
  residual GEMMs and head_dim 64).
* block (d 4096, one block, P 4608, N 4096): the exact per-layer launch
  configuration the benchmark times, against the fp64 oracle.
* full (d 4096, 32 blocks): too large for the oracle; checked through
  properties that hold at any size — the cached step equals the full
  recomputation (relative L2 < 2e-2) and every output is finite.
"""
import numpy as np
import pytest
import torch

from oracle import qi21_oracle as O
from qi21_synth import configs as C
from tests._harness import oracle_model, rel_l2

pytestmark = pytest.mark.gpu
BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from prefix_kv_cached_b200 import binding
    return binding


def _one_step(B, w, wts):
    from prefix_kv_cached_b200.runner import Qi21Runner
    r = Qi21Runner(w, B.QI21_DTYPE_BF16, host_weights=wts)
    pre = torch.from_numpy(C.host_prefix_hidden(w).astype(np.float32)).cuda()
    x = torch.from_numpy(C.host_noise(w).astype(np.float32)).cuda()
    v = torch.empty_like(x)
    r.set_prefix_row()
    r.prefix_extract(pre)
    r.set_target_row(w.sigmas[0])
    r.cached_step(x, v)
    r.euler(x, v, w.sigmas[0], w.sigmas[1], x)
    torch.cuda.synchronize()
    r.check_device()
    K, V = r.cache_kv()
    return (v.double().cpu().numpy(), x.double().cpu().numpy(), K[:, :, :r.P].double().cpu().numpy(),
            V[:, :, :r.P].double().cpu().numpy())


@pytest.mark.parametrize("name", ["mid", "block"])
def test_bf16_matches_oracle_at_benchmark_sizes(B, name):
    w = C.make_workload(name)
    model, wts = oracle_model(w, "bfloat16")
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    gv, gx, gk, gvv = _one_step(B, w, wts)
    m0, _ = O.modulation(0.0, model.wts, 4)
    mt, sf = O.modulation(1000.0 * w.sigmas[0], model.wts, 4)
    items = range(w.batch) if w.batch <= 2 else (0, w.batch - 1)
    for b in items:
        ck, cv = O.prefix_extract(model, seq, pre[b], m0)
        assert rel_l2(gk[:, b], ck) < BF16_TOL
        assert rel_l2(gvv[:, b], cv) < BF16_TOL
        v, _ = O.cached_step(model, seq, ck, cv, x0[b], mt, sf)
        assert rel_l2(gv[b], v) < BF16_TOL
        assert rel_l2(gx[b], O.euler_step(x0[b], v, w.sigmas[0], w.sigmas[1])) < BF16_TOL


def test_full_width_cached_step_equals_recompute(B):
    from prefix_kv_cached_b200.runner import Qi21Runner
    from qi21_synth.gen import normal_torch
    w = C.make_workload("full")
    r = Qi21Runner(w, B.QI21_DTYPE_BF16)           # weights drawn on the device (14 GB)
    pre = normal_torch(w.seed, "prefix_hidden", (1, w.n_prefix, 4096), device="cuda", dtype=torch.float32)
    x = normal_torch(w.seed, "noise", (1, w.n_target, 64), device="cuda", dtype=torch.float32)
    r.set_prefix_row()
    r.prefix_extract(pre)
    r.set_target_row(w.sigmas[2])
    v_c = torch.empty_like(x)
    v_f = torch.empty_like(x)
    r.cached_step(x, v_c)
    r.full_recompute(pre, x, v_f)
    torch.cuda.synchronize()
    r.check_device()
    assert torch.isfinite(v_c).all() and torch.isfinite(v_f).all()
    a, b = v_c.double().cpu().numpy(), v_f.double().cpu().numpy()
    assert rel_l2(a, b) < BF16_TOL
    assert np.linalg.norm(a) > 0


@pytest.mark.parametrize("name", ["mid", "block"])
def test_f32_matches_oracle_at_benchmark_sizes(B, name):
    """F32 storage (CUDA-core kernels) against the fp64 oracle at the benchmark's
    block sizes: max relative error < 1e-4 on v_theta, the latent and the prefix K/V."""
    from prefix_kv_cached_b200.runner import Qi21Runner
    from tests._harness import max_rel
    w = C.make_workload(name)
    model, wts = oracle_model(w, "float32")
    r = Qi21Runner(w, B.QI21_DTYPE_F32, host_weights=wts)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    x = torch.from_numpy(x0.astype(np.float32)).cuda()
    v = torch.empty_like(x)
    r.set_prefix_row()
    r.prefix_extract(torch.from_numpy(pre.astype(np.float32)).cuda())
    r.set_target_row(w.sigmas[0])
    r.cached_step(x, v)
    r.euler(x, v, w.sigmas[0], w.sigmas[1], x)
    torch.cuda.synchronize()
    r.check_device()
    K, V = r.cache_kv()
    gv, gx = v.double().cpu().numpy(), x.double().cpu().numpy()
    seq = O.make_sequence(w.segments)
    m0, _ = O.modulation(0.0, model.wts, 4)
    mt, sf = O.modulation(1000.0 * w.sigmas[0], model.wts, 4)
    for b in ((0, w.batch - 1) if w.batch > 1 else (0,)):
        ck, cv = O.prefix_extract(model, seq, pre[b], m0)
        assert max_rel(K[:, b, :r.P].double().cpu().numpy(), ck) < 1e-4
        assert max_rel(V[:, b, :r.P].double().cpu().numpy(), cv) < 1e-4
        vo, _ = O.cached_step(model, seq, ck, cv, x0[b], mt, sf)
        assert max_rel(gv[b], vo) < 1e-4
        assert max_rel(gx[b], O.euler_step(x0[b], vo, w.sigmas[0], w.sigmas[1])) < 1e-4
