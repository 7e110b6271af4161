"""Joint packing of the prefix values on the GPU (2A page, mechanisms (1)-(2);
lab [2A]) against the oracle.

* qi21_pack_prefix is pure data movement plus, in the lab's mode, one float32
  add per element: bit-exact with the oracle run on the same float32 inputs.
* The whole on-device prefix construction — img_in of the reference latents,
  packing, then the extract — matches the oracle's pack_prefix + prefix_extract
  within the F32 tolerance (1e-4 max relative error) on every layer's K and V.
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import qi21_oracle as O
from qi21_synth import configs as C
from tests._harness import oracle_model, max_rel

pytestmark = pytest.mark.gpu

# several reference images with text between them; every image's cell count is whole slots
SEGMENTS = ((C.SEG_TEXT, 20, 0), (C.SEG_IMAGE, 6, 6), (C.SEG_TEXT, 5, 0), (C.SEG_IMAGE, 4, 2),
            (C.SEG_IMAGE, 8, 8))


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from prefix_kv_cached_b200 import binding
    return binding


def _tables(B, segs):
    t = B.qi21_build_packing(list(segs))
    dev = {k: torch.from_numpy(t[k]).cuda() for k in ("slot_of", "img_row")}
    return t, dev


@pytest.mark.parametrize("mode", [0, 1])
def test_pack_bit_exact(B, mode):
    rng = np.random.default_rng(3 + mode)
    t, dev = _tables(B, SEGMENTS)
    batch, d = 2, 256
    ctx = rng.standard_normal((batch, t["n_slots"], d)).astype(np.float32)
    img = rng.standard_normal((batch, t["n_img"], d)).astype(np.float32)
    out = torch.full((batch, t["P"], d), float("nan"), device="cuda")
    B.check("qi21_pack_prefix", B.qi21_pack_prefix(batch, t["P"], d, t["n_slots"], t["n_img"],
                                                   torch.from_numpy(ctx).cuda(), torch.from_numpy(img).cuda(),
                                                   dev["slot_of"], dev["img_row"], mode, out))
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for b in range(batch):
        want = O.pack_prefix(ctx[b], img[b], SEGMENTS, mode)      # float32 in, float32 arithmetic
        assert want.dtype == np.float32
        assert np.array_equal(got[b], want)


@pytest.mark.parametrize("mode", [0, 1])
def test_packed_prefix_feeds_the_extract(B, mode):
    from prefix_kv_cached_b200.runner import Qi21Runner
    w = dataclasses.replace(C.make_workload("small"), name="packing", segments=SEGMENTS)
    model, wts = oracle_model(w, "float32")
    r = Qi21Runner(w, B.QI21_DTYPE_F32, host_weights=wts)
    t, dev = _tables(B, SEGMENTS)
    sh = w.shape
    rng = np.random.default_rng(9)
    ctx = rng.standard_normal((w.batch, t["n_slots"], sh.d_model)).astype(np.float32)
    lat = rng.standard_normal((w.batch, t["n_img"], sh.latent_ch)).astype(np.float32)
    img_tok = torch.empty(w.batch * t["n_img"], sh.d_model, device="cuda")
    B.check("qi21_img_in_tokens", B.qi21_img_in_tokens(r.cfg, r.wstruct, torch.from_numpy(lat).cuda(),
                                                       w.batch * t["n_img"], img_tok))
    pre = torch.empty(w.batch, t["P"], sh.d_model, device="cuda")
    B.check("qi21_pack_prefix", B.qi21_pack_prefix(w.batch, t["P"], sh.d_model, t["n_slots"], t["n_img"],
                                                   torch.from_numpy(ctx).cuda(), img_tok, dev["slot_of"],
                                                   dev["img_row"], mode, pre))
    r.set_prefix_row()
    r.prefix_extract(pre)
    torch.cuda.synchronize()
    r.check_device()
    K, V = r.cache_kv()
    gk, gv = K[:, :, :r.P].double().cpu().numpy(), V[:, :, :r.P].double().cpu().numpy()
    seq = O.make_sequence(w.segments)
    m0, _ = O.modulation(0.0, model.wts, model.n_chunks)
    for b in range(w.batch):
        tokens = O.img_in(lat[b].astype(np.float64), model.wts["w_img_in"])
        pre_o = O.pack_prefix(ctx[b].astype(np.float64), tokens, SEGMENTS, mode)
        ck, cv = O.prefix_extract(model, seq, pre_o, m0)
        assert max_rel(gk[:, b], ck) < 1e-4
        assert max_rel(gv[:, b], cv) < 1e-4


@pytest.mark.parametrize("dtype_name", ["float32", "bfloat16"])
def test_pack_weights_from_canonical_layout(B, dtype_name):
    """qi21_pack_weights: canonical [in][out] weights become exactly the [out][in]
    tensors the kernels read (bit-exact), and a cached step through them gives
    the same result (to the run-to-run variation of the residual GEMMs, whose
    partial sums reach h in a non-deterministic order: rel-L2 < 1e-3; a
    packing mistake moves it by order 1)."""
    from prefix_kv_cached_b200.runner import Qi21Runner
    w = C.make_workload("small")
    dtype = B.QI21_DTYPE_F32 if dtype_name == "float32" else B.QI21_DTYPE_BF16
    _, wts = oracle_model(w, dtype_name)
    r = Qi21Runner(w, dtype, host_weights=wts)
    canon = {}
    for name, _ in C.weight_specs(w.shape):
        t = r.weights[name]
        canon[name] = t if name in ("q_norm", "k_norm") else t.transpose(-1, -2).contiguous()
    cw = B.qi21_weights_canonical(*[canon[n].data_ptr() for n in (
        "w_img_in", "w_out", "w_t1", "w_t2", "w_mod", "w_fin", "w_q", "w_k", "w_v", "w_o", "w_gate", "w_up",
        "w_down", "q_norm", "k_norm")])
    nbytes = B.qi21_packed_weights_bytes(r.cfg)
    packed = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    st, pw = B.qi21_pack_weights(r.cfg, cw, packed, nbytes)
    assert st == 0
    torch.cuda.synchronize()
    base = packed.data_ptr()
    for name, shp in C.weight_specs(w.shape):
        ref = r.weights[name]
        off = getattr(pw, name) - base
        got = packed[off: off + ref.numel() * ref.element_size()].view(ref.dtype).view(ref.shape)
        assert torch.equal(got, ref), name
    # a cached step through the packed weights equals the step through the original tensors
    pre = torch.from_numpy(C.host_prefix_hidden(w).astype(np.float32)).cuda()
    x = torch.from_numpy(C.host_noise(w).astype(np.float32)).cuda()
    outs = []
    for wstruct in (r.wstruct, pw):
        r.wstruct = wstruct
        v = torch.empty_like(x)
        r.set_prefix_row()
        r.prefix_extract(pre)
        r.set_target_row(w.sigmas[0])
        r.cached_step(x, v)
        torch.cuda.synchronize()
        outs.append(v.clone())
    r.check_device()
    a, b = outs[0].double(), outs[1].double()
    assert float(torch.linalg.norm(a - b) / torch.linalg.norm(b)) < 1e-3
