"""BF16 mode on the tcgen05 tensor-core kernels: parity with the fp64 oracle
(2e-2 relative L2) and agreement with the CUDA-core kernel family on the same
bf16 storage (same roundings up to accumulation order)."""
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


def _run(B, w, wts, tc: int, n_steps: int):
    from prefix_kv_cached_b200.runner import Qi21Runner
    B.qi21_set_tensor_cores(tc)
    try:
        r = Qi21Runner(w, B.QI21_DTYPE_BF16, host_weights=wts)
        pre = torch.from_numpy(C.host_prefix_hidden(w).astype(np.float32)).cuda()
        x = torch.from_numpy(C.host_noise(w).astype(np.float32)).cuda()
        v = torch.empty_like(x)
        r.set_prefix_row()
        r.prefix_extract(pre)
        vs, xs = [], []
        for k in range(n_steps):
            r.set_target_row(w.sigmas[k])
            r.cached_step(x, v)
            vs.append(v.double().cpu().numpy())
            r.euler(x, v, w.sigmas[k], w.sigmas[k + 1], x)
            xs.append(x.double().cpu().numpy())
        torch.cuda.synchronize()
        r.check_device()
        K, V = r.cache_kv()
        kv = (K[:, :, :r.P].double().cpu().numpy(), V[:, :, :r.P].double().cpu().numpy())
        vf = torch.empty_like(x)
        r.full_recompute(pre, x, vf)
        torch.cuda.synchronize()
        r.check_device()
        return vs, xs, kv, vf.double().cpu().numpy(), x.double().cpu().numpy(), r
    finally:
        B.qi21_set_tensor_cores(1)


@pytest.mark.parametrize("name", ["small", "small64"])
def test_tc_family_agrees_with_cuda_core_family(B, name):
    w = C.make_workload(name)
    _, wts = oracle_model(w, "bfloat16")
    a = _run(B, w, wts, 1, 2)
    b = _run(B, w, wts, 0, 2)
    assert rel_l2(a[2][0], b[2][0]) < 1e-2     # prefix K of every layer
    assert rel_l2(a[2][1], b[2][1]) < 1e-2     # prefix V
    for k in range(2):
        assert rel_l2(a[0][k], b[0][k]) < 1e-2
    assert rel_l2(a[3], b[3]) < 1e-2           # full recompute


@pytest.mark.parametrize("name", ["small", "small64", "small_t1"])
def test_tc_matches_oracle(B, name):
    w = C.make_workload(name)
    model, wts = oracle_model(w, "bfloat16")
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    n_steps = 3
    vs, xs, (gk, gv), vfull, xlast, r = _run(B, w, wts, 1, n_steps)
    m0, _ = O.modulation(0.0, model.wts, 4)
    for b in range(w.batch):
        ck, cv = O.prefix_extract(model, seq, pre[b], m0)
        assert rel_l2(gk[:, b], ck) < BF16_TOL
        assert rel_l2(gv[:, b], cv) < BF16_TOL
        x = x0[b]
        for k in range(n_steps):
            mt, sf = O.modulation(1000.0 * w.sigmas[k], model.wts, 4)
            v, _ = O.cached_step(model, seq, ck, cv, x, mt, sf)
            x = O.euler_step(x, v, w.sigmas[k], w.sigmas[k + 1])
            assert rel_l2(vs[k][b], v) < BF16_TOL, f"v step {k} item {b}"
            assert rel_l2(xs[k][b], x) < BF16_TOL, f"x step {k} item {b}"
        # full recompute at sigma_{n_steps} on the last latent
        mt, sf = O.modulation(1000.0 * w.sigmas[n_steps - 1], model.wts, 4)
        ref = O.joint_forward(model, seq, pre[b], xlast[b], m0, mt, sf)["v"]
        assert rel_l2(vfull[b], ref) < BF16_TOL
