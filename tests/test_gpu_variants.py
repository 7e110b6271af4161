"""Variants of the path (F32 storage, against the fp64 oracle within 1e-4 max
relative error):

* frame_mode = 1: the RoPE frame axis carries the image id instead of 0 (the
  target statement's "(image_id, h, w)" reading; the pages pin frame = 0);
* a 40-step schedule through the whole-image graph (3B page §2: "8-40 denoising
  steps"; the pages print only the 8-step Turbo table, so the 40-step one is
  read as sigma uniform from 1 to 0);
* ten reference images in the prefix (the End-to-end lab's note on "up to 10
  reference images"), each with its own image id and block-causal run.
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import qi21_oracle as O
from qi21_synth import configs as C
from tests._harness import oracle_model, max_rel

pytestmark = pytest.mark.gpu
F32_TOL = 1e-4


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from prefix_kv_cached_b200 import binding
    return binding


def _one_step(B, w, frame_mode=0, steps=1):
    """Extract + `steps` cached steps with Euler on the GPU and in the oracle; returns the max-rel errors."""
    from prefix_kv_cached_b200.runner import Qi21Runner
    model, wts = oracle_model(w, "float32")
    r = Qi21Runner(w, B.QI21_DTYPE_F32, host_weights=wts, frame_mode=frame_mode)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    x = torch.from_numpy(x0.astype(np.float32)).cuda()
    v = torch.empty_like(x)
    r.set_prefix_row()
    r.prefix_extract(torch.from_numpy(pre.astype(np.float32)).cuda())
    vs = []
    for k in range(steps):
        r.set_target_row(w.sigmas[k])
        r.cached_step(x, v)
        vs.append(v.double().cpu().numpy())
        r.euler(x, v, w.sigmas[k], w.sigmas[k + 1], x)
    torch.cuda.synchronize()
    r.check_device()
    seq = O.make_sequence(w.segments, frame_mode)
    errs = []
    for b in range(w.batch):
        out = O.run_image(model, seq, pre[b], x0[b], w.sigmas[:steps + 1], use_cache=True)
        errs += [max_rel(vs[k][b], out["velocities"][k]) for k in range(steps)]
        errs.append(max_rel(x.double().cpu().numpy()[b], out["xs"][-1]))
    return max(errs)


def test_frame_axis_as_image_id(B):
    w = C.make_workload("small")
    assert _one_step(B, w, frame_mode=1, steps=2) < F32_TOL
    # the two readings really differ on this layout (two images)
    c0 = O.rope_coords(w.segments, 0)
    c1 = O.rope_coords(w.segments, 1)
    assert not np.array_equal(c0, c1)


def test_ten_reference_images(B):
    segs = [C._text(6)]
    for i in range(10):
        segs += [C._img(2 + i % 3, 3), C._text(1 + i % 2)]
    segs.append(C._img(6, 5))
    w = dataclasses.replace(C.make_workload("small"), name="ten_refs", segments=tuple(segs), batch=1)
    ids = O.token_metadata(w.segments)[0]
    assert sorted(set(ids.tolist())) == [-1] + list(range(11))
    assert _one_step(B, w, steps=1) < F32_TOL


def test_forty_step_schedule_through_the_graph(B):
    from prefix_kv_cached_b200.runner import Qi21Runner
    sig40 = tuple(np.linspace(1.0, 0.0, 41).tolist())
    w = dataclasses.replace(C.make_workload("small64"), name="small64_40", sigmas=sig40, batch=1)
    model, wts = oracle_model(w, "float32")
    r = Qi21Runner(w, B.QI21_DTYPE_F32, host_weights=wts)
    pre = C.host_prefix_hidden(w)
    x0 = C.host_noise(w)
    pre_d = torch.from_numpy(pre.astype(np.float32)).cuda()
    x = torch.from_numpy(x0.astype(np.float32)).cuda()
    sig = torch.tensor(sig40, dtype=torch.float64, device="cuda")
    g = r.capture_image(pre_d, x, sig)
    x.copy_(torch.from_numpy(x0.astype(np.float32)))
    g.replay()
    torch.cuda.synchronize()
    r.check_device()
    want = O.run_image(model, O.make_sequence(w.segments), pre[0], x0[0], sig40, use_cache=True)["xs"][-1]
    assert max_rel(x.double().cpu().numpy()[0], want) < F32_TOL
    del g
