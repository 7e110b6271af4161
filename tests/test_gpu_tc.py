"""BF16 mode on the tcgen05 tensor-core kernels: parity with the fp64 oracle
(2e-2 relative L2) on every layer's prefix K/V, every layer's target K/V of
each cached step, v_theta and the latent; and agreement with the CUDA-core
kernel family on the same bf16 storage (same roundings up to accumulation
order).

The workloads use the parity weight recipe (O(1) modulation gates, an
attention branch as large as the residual stream): replacing the attention by
zeros moves every compared tensor by more than ten times the tolerance
(tests/test_parity_strength.py), so these tests fail for a wrong attention.
"""
import numpy as np
import pytest
import torch

from oracle import qi21_oracle as O
from qi21_synth import configs as C
from tests._harness import BF16_TOL, assert_item_matches, gpu_steps, oracle_item, oracle_model, rel_l2

pytestmark = pytest.mark.gpu


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
        fam = B.qi21_kernel_family(r.cfg)
        assert fam == (B.QI21_FAMILY_TENSOR_CORES if tc else B.QI21_FAMILY_CUDA_CORES)
        pre = torch.from_numpy(C.host_prefix_hidden(w).astype(np.float32)).cuda()
        x0 = torch.from_numpy(C.host_noise(w).astype(np.float32)).cuda()
        got = gpu_steps(r, pre, x0, w.sigmas, n_steps)
        vf = torch.empty_like(x0)
        xl = torch.from_numpy(got["x"][-1].astype(np.float32)).cuda()
        r.full_recompute(pre, xl, vf)
        torch.cuda.synchronize()
        r.check_device()
        got["vfull"] = vf.double().cpu().numpy()
        return got
    finally:
        B.qi21_set_tensor_cores(1)


@pytest.mark.parametrize("name", ["small", "small64"])
def test_tc_family_agrees_with_cuda_core_family(B, name):
    w = C.make_workload(name)
    _, wts = oracle_model(w, "bfloat16")
    a = _run(B, w, wts, 1, 2)
    b = _run(B, w, wts, 0, 2)
    for key in ("pk", "pv"):
        assert rel_l2(a[key], b[key]) < 1e-2, key
    for k in range(2):
        for key in ("tk", "tv", "v"):
            assert rel_l2(a[key][k], b[key][k]) < 1e-2, f"{key} step {k}"
    assert rel_l2(a["vfull"], b["vfull"]) < 1e-2


@pytest.mark.parametrize("name", ["small", "small64", "small_t1"])
def test_tc_matches_oracle(B, name):
    w = C.make_workload(name)
    model, wts = oracle_model(w, "bfloat16")
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    n_steps = 3
    got = _run(B, w, wts, 1, n_steps)
    for b in range(w.batch):
        want = oracle_item(model, seq, pre[b], x0[b], w.sigmas, n_steps)
        assert_item_matches(got, want, b, n_steps, rel_l2, BF16_TOL, name)
        # full recompute at sigma_{n_steps - 1} on the last latent
        mt, sf = O.modulation(1000.0 * w.sigmas[n_steps - 1], model.wts, 4)
        ref = O.joint_forward(model, seq, pre[b], got["x"][-1][b], want["m0"], mt, sf)["v"]
        assert rel_l2(got["vfull"][b], ref) < BF16_TOL
