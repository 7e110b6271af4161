"""qi21_modulation_noalloc: the modulation call for callers that cannot allocate.

Some users of the library cannot give it a workspace: their device memory is
owned by another allocator, or their loop must never call cudaMalloc because
it can block. This entry point keeps its scratch in a fixed device array
inside the library instead. The test calls it through the C ABI twice in a
row (two timesteps, so the second call overwrites what the first left in the
shared array) and checks each result against qi21_modulation, which uses a
caller workspace, within the fp32 tolerance of the parity tests (1e-4 max
relative error). It also checks that a model wider than the array's limit is
refused before anything runs.

The tests do not depend on test order: each builds its own runner and reads
only what its own calls wrote (both calls of the array are fully written before
they are read), so they pass alone in a fresh process and after every other
test. The file name makes pytest collect it last only so that, should it fail,
a run that stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from qi21_synth import configs as C

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _max_rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


@pytest.mark.parametrize("name,dtype_name,store", [("toy", "f32", "float32"), ("small", "bf16", "bfloat16")])
def test_noalloc_modulation_matches_workspace_version(name, dtype_name, store):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from prefix_kv_cached_b200 import build
    build.build()
    from prefix_kv_cached_b200 import binding as B
    from prefix_kv_cached_b200.runner import Qi21Runner

    dtype = B.QI21_DTYPE_F32 if dtype_name == "f32" else B.QI21_DTYPE_BF16
    w = C.make_workload(name)
    r = Qi21Runner(w, dtype, host_weights=C.host_weights(w, store))
    d, nch = w.shape.d_model, w.shape.n_chunks
    stream = torch.cuda.current_stream().cuda_stream
    for t in (1000.0 * w.sigmas[1], 0.0):          # two calls in a row
        ref_mod = torch.empty(nch * d, device="cuda")
        ref_sf = torch.empty(d, device="cuda")
        B.check("qi21_modulation", B.qi21_modulation(r.cfg, r.wstruct, t, ref_mod, ref_sf, r.ws, r.ws_bytes,
                                                     stream))
        got_mod = torch.full((nch * d,), float("nan"), device="cuda")
        got_sf = torch.full((d,), float("nan"), device="cuda")
        B.check("qi21_modulation_noalloc", B.qi21_modulation_noalloc(r.cfg, r.wstruct, t, got_mod, got_sf,
                                                                     stream))
        torch.cuda.synchronize()
        assert torch.isfinite(got_mod).all() and torch.isfinite(got_sf).all()
        assert _max_rel(got_mod, ref_mod) < TOL
        assert _max_rel(got_sf, ref_sf) < TOL


def test_noalloc_rejects_width_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from prefix_kv_cached_b200 import binding as B
    from prefix_kv_cached_b200.runner import make_config

    wide = C.ModelShape(16384, 128, 128, 1, 512, 64, 256)
    cfg = make_config(wide, B.QI21_DTYPE_BF16)
    fake = 0x10000
    w = B.qi21_weights(*([fake] * 15))
    assert B.qi21_modulation_noalloc(cfg, w, 500.0, fake, fake, 0) == B.QI21_ERR_UNSUPPORTED
