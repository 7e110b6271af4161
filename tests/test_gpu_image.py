"""Whole-image driver (qi21_denoise_image: extract once, then the cached steps
with Euler, 6B page §4) and its CUDA-graph replay with the sigma schedule read
from a device table.

* One call equals the step-by-step path through the separate entry points:
  the kernels are the same; only the timestep embedding is formed on the device
  from the sigma table (fp64, like the host helper) instead of on the host.
* It matches the fp64 oracle's denoising loop: F32 storage within 1e-4 max
  relative error, BF16 (tensor cores) within 2e-2 relative L2.
* A captured graph replays to exactly the eager result, and after another
  schedule is written into the device table a replay of the same graph follows
  the new schedule (checked against the oracle on that schedule).
"""
import numpy as np
import pytest
import torch

from oracle import qi21_oracle as O
from qi21_synth import configs as C
from tests._harness import oracle_model, max_rel, rel_l2

pytestmark = pytest.mark.gpu
F32_TOL = 1e-4
BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from prefix_kv_cached_b200 import binding
    return binding


def _setup(B, name, dtype, store):
    from prefix_kv_cached_b200.runner import Qi21Runner
    w = C.make_workload(name)
    model, wts = oracle_model(w, store)
    r = Qi21Runner(w, dtype, host_weights=wts)
    pre = torch.from_numpy(C.host_prefix_hidden(w).astype(np.float32)).cuda()
    x0 = torch.from_numpy(C.host_noise(w).astype(np.float32)).cuda()
    return w, model, r, pre, x0


def _oracle_final(w, model, sigmas):
    seq = O.make_sequence(w.segments)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    return np.stack([O.run_image(model, seq, pre[b], x0[b], sigmas, use_cache=True)["xs"][-1]
                     for b in range(w.batch)])


def test_image_call_matches_step_path_and_oracle_f32(B):
    w, model, r, pre, x0 = _setup(B, "small", B.QI21_DTYPE_F32, "float32")
    sig = torch.tensor(w.sigmas, dtype=torch.float64, device="cuda")
    x = x0.clone()
    r.denoise_image(pre, x, sig)
    torch.cuda.synchronize()
    r.check_device()
    steps = r.denoise(pre, x0, w.sigmas)        # host-side loop over the separate entry points
    torch.cuda.synchronize()
    a, b = x.double().cpu().numpy(), steps.double().cpu().numpy()
    assert rel_l2(a, b) < 1e-6
    assert max_rel(a, _oracle_final(w, model, w.sigmas)) < F32_TOL


def test_graph_replay_is_exact_and_follows_a_new_schedule(B):
    w, model, r, pre, x0 = _setup(B, "small", B.QI21_DTYPE_F32, "float32")
    sig = torch.tensor(w.sigmas, dtype=torch.float64, device="cuda")
    x = x0.clone()
    g = r.capture_image(pre, x, sig)
    x.copy_(x0)
    g.replay()
    torch.cuda.synchronize()
    r.check_device()
    replayed = x.clone()
    eager = x0.clone()
    r.denoise_image(pre, eager, sig)
    torch.cuda.synchronize()
    assert torch.equal(replayed, eager)
    # another 8-step schedule through the same graph
    other = np.linspace(1.0, 0.0, len(w.sigmas)).tolist()
    sig.copy_(torch.tensor(other, dtype=torch.float64))
    x.copy_(x0)
    g.replay()
    torch.cuda.synchronize()
    r.check_device()
    got = x.double().cpu().numpy()
    assert not np.allclose(got, replayed.double().cpu().numpy())
    assert max_rel(got, _oracle_final(w, model, other)) < F32_TOL
    del g


def test_graph_bf16_tensor_cores_matches_oracle(B):
    w, model, r, pre, x0 = _setup(B, "small", B.QI21_DTYPE_BF16, "bfloat16")
    sig = torch.tensor(w.sigmas, dtype=torch.float64, device="cuda")
    x = x0.clone()
    g = r.capture_image(pre, x, sig)
    x.copy_(x0)
    g.replay()
    torch.cuda.synchronize()
    r.check_device()
    assert rel_l2(x.double().cpu().numpy(), _oracle_final(w, model, w.sigmas)) < BF16_TOL
    del g
