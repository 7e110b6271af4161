"""C-ABI library checks that need no GPU: it builds, loads, exports every
symbol include/*.h declares, its host helpers agree with the oracle (bit-exact
for integer metadata), and host-detectable errors return before any launch."""
import ctypes as ct
import glob
import os
import re

import numpy as np
import pytest

from tests.conftest import ROOT
from oracle import qi21_oracle as O
from qi21_synth import configs as C


@pytest.fixture(scope="module")
def B():
    from prefix_kv_cached_b200 import build
    build.build()
    from prefix_kv_cached_b200 import binding
    return binding


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(qi21_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported(B):
    names = _declared_symbols()
    assert len(names) >= 20
    for n in names:
        assert hasattr(B.lib, n), f"{n} declared in include/ but not exported"
    assert set(B.EXPORTED) <= set(names)


@pytest.mark.parametrize("name", ["toy", "small", "small64", "full", "large"])
def test_metadata_bit_exact_vs_oracle(B, name):
    w = C.make_workload(name)
    m = B.qi21_build_metadata(list(w.segments))
    ids, mask, s, p, n = O.token_metadata(w.segments)
    assert (m["S"], m["P"], m["N"]) == (s, p, n)
    np.testing.assert_array_equal(m["image_ids"], ids)
    np.testing.assert_array_equal(m["target_mask"].astype(bool), mask)
    np.testing.assert_array_equal(m["coords"], O.rope_coords(w.segments))
    if s <= 2000:
        np.testing.assert_array_equal(m["kv_limit"], O.kv_limit_from_mask(O.block_causal_allowed(ids)))
    m1 = B.qi21_build_metadata(list(w.segments), frame_mode=1)
    np.testing.assert_array_equal(m1["coords"], O.rope_coords(w.segments, frame_mode=1))


def test_toy_metadata_matches_page(B, golden):
    g = golden("toy_sequence.json")
    m = B.qi21_build_metadata([tuple(s) for s in g["segments"]])
    assert m["image_ids"].tolist() == g["image_ids"]
    assert m["kv_limit"].tolist() == g["mask_row_key_counts"]


def test_rope_helpers_vs_oracle(B):
    for dh in (64, 128):
        np.testing.assert_array_equal(B.qi21_rope_omega_axial(dh), O.rope_omega_axial(dh))
    w = C.make_workload("small")
    m = B.qi21_build_metadata(list(w.segments))
    om = O.rope_omega_axial(128)
    cs = B.qi21_rope_table(128, m["coords"], om)
    ang = O.rope_angles(m["coords"], om)
    np.testing.assert_allclose(cs[..., 0], np.cos(ang), atol=6e-8)
    np.testing.assert_allclose(cs[..., 1], np.sin(ang), atol=6e-8)
    emb = B.qi21_timestep_embedding(850.0, 256)
    np.testing.assert_allclose(emb, O.timestep_embedding(850.0, 256), atol=6e-8)


def test_metadata_errors(B):
    segs = (B.qi21_segment * 2)(B.qi21_segment(B.QI21_SEG_IMAGE, 0, 2, 2), B.qi21_segment(B.QI21_SEG_TEXT, 3, 0, 0))
    S, P, N = ct.c_int32(), ct.c_int32(), ct.c_int32()
    st = B.lib.qi21_build_metadata(segs, 2, 0, 0, None, None, None, None, ct.byref(S), ct.byref(P), ct.byref(N))
    assert st == B.QI21_ERR_METADATA          # target must be last
    segs2 = (B.qi21_segment * 1)(B.qi21_segment(B.QI21_SEG_IMAGE, 0, 0, 3))
    assert B.lib.qi21_build_metadata(segs2, 1, 0, 0, None, None, None, None, ct.byref(S), ct.byref(P),
                                     ct.byref(N)) == B.QI21_ERR_METADATA
    ids = np.zeros(2, np.int32)
    segs3 = (B.qi21_segment * 1)(B.qi21_segment(B.QI21_SEG_IMAGE, 0, 2, 2))
    assert B.lib.qi21_build_metadata(segs3, 1, 0, 2, ids.ctypes.data, None, None, None, ct.byref(S), ct.byref(P),
                                     ct.byref(N)) == B.QI21_ERR_METADATA    # capacity < S


def _cfg(B, dtype=0):
    from prefix_kv_cached_b200.runner import make_config
    return make_config(C.SMALL, dtype)


def test_host_validation_returns_before_launch(B):
    cfg = _cfg(B)
    fake = 0x10000          # aligned, never dereferenced on these paths
    w = B.qi21_weights(*([fake] * 15))
    cache = B.qi21_kv_cache_init(fake, cfg, 1, 8, 4)
    ws_bytes = B.qi21_workspace_bytes(cfg, 1, 8, 4)
    assert ws_bytes > 0 and B.qi21_kv_cache_bytes(cfg, 1, 8, 4) == 4 * 2 * 2 * 12 * 256
    # cached step before any extract
    assert B.qi21_cached_step(cfg, w, cache, fake, fake, fake, fake, fake, fake, ws_bytes, 0) == \
        B.QI21_ERR_CACHE_STATE
    # misaligned input pointer
    cache.state = B.QI21_CACHE_EXTRACTED
    assert B.qi21_cached_step(cfg, w, cache, fake + 4, fake, fake, fake, fake, fake, ws_bytes, 0) == \
        B.QI21_ERR_INVALID_ARG
    # workspace too small
    assert B.qi21_cached_step(cfg, w, cache, fake, fake, fake, fake, fake, fake, ws_bytes - 1, 0) == \
        B.QI21_ERR_WORKSPACE_TOO_SMALL
    # cache built for another model
    other = _cfg(B)
    other.n_layers = 3
    assert B.qi21_cached_step(other, w, cache, fake, fake, fake, fake, fake, fake, ws_bytes, 0) == \
        B.QI21_ERR_CACHE_STATE
    # inconsistent config
    bad = _cfg(B)
    bad.n_heads = 3
    assert B.qi21_cached_step(bad, w, cache, fake, fake, fake, fake, fake, fake, ws_bytes, 0) == B.QI21_ERR_SHAPE
    # null weight pointer
    w2 = B.qi21_weights(*([fake] * 14 + [0]))
    assert B.qi21_prefix_extract(cfg, w2, cache, fake, fake, fake, fake, fake, ws_bytes, 0) == \
        B.QI21_ERR_INVALID_ARG
    assert B.qi21_full_recompute_step(cfg, w, 0, 8, 4, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                      ws_bytes, 0) == B.QI21_ERR_SHAPE
    assert B.qi21_euler_update(fake, fake, 1.0, float("nan"), fake, 4, 0) == B.QI21_ERR_INVALID_ARG
    # device-indexed forms and the whole-image call: bad sigma tables, steps and configs
    mod = fake
    assert B.qi21_modulation_at(cfg, w, 0, 0, 1000.0, mod, mod, fake, ws_bytes, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_modulation_at(cfg, w, fake + 4, 0, 1000.0, mod, mod, fake, ws_bytes, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_modulation_at(cfg, w, fake, -1, 1000.0, mod, mod, fake, ws_bytes, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_modulation_at(bad, w, fake, 0, 1000.0, mod, mod, fake, ws_bytes, 0) == B.QI21_ERR_SHAPE
    assert B.qi21_euler_update_at(fake, fake, fake, -1, fake, 4, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_euler_update_at(fake + 4, fake, fake, 0, fake, 4, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_euler_update_at(fake, fake, 0, 0, fake, 4, 0) == B.QI21_ERR_INVALID_ARG
    args = (fake, fake, fake, fake)
    assert B.qi21_denoise_image(cfg, w, cache, *args, fake, 0, 1000.0, fake, fake, mod, mod, mod, fake, ws_bytes,
                                0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_denoise_image(cfg, w, cache, *args, 0, 8, 1000.0, fake, fake, mod, mod, mod, fake, ws_bytes,
                                0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_denoise_image(bad, w, cache, *args, fake, 8, 1000.0, fake, fake, mod, mod, mod, fake, ws_bytes,
                                0) == B.QI21_ERR_SHAPE
    assert B.qi21_status_string(B.QI21_ERR_DEVICE_TIMEOUT).startswith("device wait")


def test_workspace_covers_the_selected_kernel_family(B):
    """BF16 with the tensor cores switched off runs the CUDA-core GEMMs, whose
    fp32 outputs need extra workspace; a workspace sized for the tensor-core
    family must then be refused before any launch."""
    from prefix_kv_cached_b200.runner import make_config
    cfg = make_config(C.SMALL, B.QI21_DTYPE_BF16)
    tc_bytes = B.qi21_workspace_bytes(cfg, 2, 198, 300)
    B.qi21_set_tensor_cores(0)
    try:
        cc_bytes = B.qi21_workspace_bytes(cfg, 2, 198, 300)
        assert cc_bytes >= tc_bytes + 4 * 2 * 498 * 768
        fake = 0x10000
        w = B.qi21_weights(*([fake] * 15))
        cache = B.qi21_kv_cache_init(fake, cfg, 2, 198, 300)
        cache.state = B.QI21_CACHE_EXTRACTED
        assert B.qi21_cached_step(cfg, w, cache, fake, fake, fake, fake, fake, fake, tc_bytes, 0) == \
            B.QI21_ERR_WORKSPACE_TOO_SMALL
    finally:
        B.qi21_set_tensor_cores(1)
    assert B.qi21_workspace_bytes(cfg, 2, 198, 300) == tc_bytes


def test_packing_tables_bit_exact_vs_oracle(B):
    from tests.test_oracle_pins import _random_layouts
    layouts = _random_layouts(30, seed=11) + [[(0, 2, 0), (1, 2, 2), (0, 1, 0), (1, 2, 2)]]
    for segs in layouts:
        got = B.qi21_build_packing(segs)
        slot_of, img_row, n_slots, n_img = O.slot_expansion(segs)
        assert got["slot_of"].tolist() == slot_of.tolist()
        assert got["img_row"].tolist() == img_row.tolist()
        assert (got["P"], got["n_slots"], got["n_img"]) == (len(slot_of), n_slots, n_img)


def test_packing_errors_and_validation(B):
    for segs in ([(0, 3, 0), (1, 3, 3), (1, 2, 2)],      # 9 cells: not whole slots
                 [(1, 2, 2), (0, 3, 0)]):                 # target is not an image
        with pytest.raises(B.Qi21Error) as e:
            B.qi21_build_packing(segs)
        assert e.value.status == B.QI21_ERR_METADATA
    fake = 0x10000
    assert B.qi21_pack_prefix(1, 7, 6, 4, 4, fake, fake, fake, fake, 0, fake, 0) == B.QI21_ERR_INVALID_ARG  # d % 4
    assert B.qi21_pack_prefix(1, 7, 8, 4, 4, fake, fake, fake, fake, 2, fake, 0) == B.QI21_ERR_INVALID_ARG  # mode
    assert B.qi21_pack_prefix(1, 7, 8, 4, 4, fake + 4, fake, fake, fake, 0, fake, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_pack_prefix(1, 7, 8, 4, 4, fake, fake, 0, fake, 0, fake, 0) == B.QI21_ERR_INVALID_ARG
    cfg = _cfg(B)
    w = B.qi21_weights(*([fake] * 15))
    assert B.qi21_img_in_tokens(cfg, w, fake, 0, fake, 0) == B.QI21_ERR_INVALID_ARG
    assert B.qi21_img_in_tokens(cfg, w, fake + 4, 4, fake, 0) == B.QI21_ERR_INVALID_ARG


def test_shared_prefix_cache_layout(B):
    cfg = _cfg(B)
    fake = 0x10000
    # [L][2][Pp + B*N][d], Pp = P rounded up to the 128-key attention tile
    for P, N, Bn in ((8, 4, 3), (128, 4, 1), (129, 7, 2)):
        pp = -(-P // 128) * 128
        assert B.qi21_kv_cache_bytes_shared(cfg, Bn, P, N) == 4 * cfg.n_layers * 2 * (pp + Bn * N) * cfg.d_model
    cache = B.qi21_kv_cache_init_shared(fake, cfg, 3, 8, 4)
    assert (cache.shared_prefix, cache.batch, cache.state) == (1, 3, B.QI21_CACHE_EMPTY)
    assert B.qi21_kv_cache_init(fake, cfg, 3, 8, 4).shared_prefix == 0
    ws_bytes = B.qi21_workspace_bytes(cfg, 3, 8, 4)
    w = B.qi21_weights(*([fake] * 15))
    assert B.qi21_cached_step(cfg, w, cache, fake, fake, fake, fake, fake, fake, ws_bytes, 0) == \
        B.QI21_ERR_CACHE_STATE


def test_packed_weights_size_and_validation(B):
    for name in ("small", "full"):
        sh = C.make_workload(name).shape
        for dt, eb in ((B.QI21_DTYPE_F32, 4), (B.QI21_DTYPE_BF16, 2)):
            from prefix_kv_cached_b200.runner import make_config
            cfg = make_config(sh, dt)
            want = 0
            for wname, shp in C.weight_specs(sh):
                nbytes = int(np.prod(shp)) * (4 if wname in ("q_norm", "k_norm") else eb)
                want += (nbytes + 255) // 256 * 256
            assert B.qi21_packed_weights_bytes(cfg) == want
    cfg = _cfg(B)
    fake = 0x10000
    cw = B.qi21_weights_canonical(*([fake] * 15))
    need = B.qi21_packed_weights_bytes(cfg)
    assert B.qi21_pack_weights(cfg, cw, fake, need - 1)[0] == B.QI21_ERR_WORKSPACE_TOO_SMALL
    assert B.qi21_pack_weights(cfg, cw, fake + 8, need)[0] == B.QI21_ERR_INVALID_ARG
    cw.w_down = fake + 4
    assert B.qi21_pack_weights(cfg, cw, fake, need)[0] == B.QI21_ERR_INVALID_ARG


def test_bf16_shape_without_tensor_core_kernels_is_refused(B):
    """BF16 never falls back to the CUDA-core kernels on its own: a head_dim the
    tensor-core attention does not cover is refused before any launch."""
    from prefix_kv_cached_b200.runner import make_config
    shape = C.ModelShape(256, 8, 32, 1, 768, 64, 256)
    cfg = make_config(shape, B.QI21_DTYPE_BF16)
    assert B.qi21_kernel_family(cfg) == B.QI21_FAMILY_NONE
    fake = 0x10000
    w = B.qi21_weights(*([fake] * 15))
    cache = B.qi21_kv_cache(fake, 1, 8, 8, 1, 256, B.QI21_DTYPE_BF16, B.QI21_CACHE_EXTRACTED, 0)
    st = B.qi21_cached_step(cfg, w, cache, fake, fake, fake, fake, fake, fake, 1 << 30, 0)
    assert st == B.QI21_ERR_UNSUPPORTED
    B.qi21_set_tensor_cores(0)
    try:
        assert B.qi21_kernel_family(cfg) == B.QI21_FAMILY_CUDA_CORES
    finally:
        B.qi21_set_tensor_cores(1)


def test_lab_rope_omega_matches_oracle(B):
    assert np.array_equal(B.qi21_rope_omega_lab(), O.rope_omega_lab())


def test_noalloc_applies_the_modulation_shape_checks(B):
    """qi21_modulation_noalloc refuses what qi21_modulation refuses (here a BF16
    head_dim the tensor-core kernels do not cover), before any launch."""
    from prefix_kv_cached_b200.runner import make_config
    cfg = make_config(C.ModelShape(256, 8, 32, 1, 768, 64, 256), B.QI21_DTYPE_BF16)
    fake = 0x10000
    w = B.qi21_weights(*([fake] * 15))
    assert B.qi21_modulation(cfg, w, 500.0, fake, fake, fake, 1 << 30, 0) == B.QI21_ERR_UNSUPPORTED
    assert B.qi21_modulation_noalloc(cfg, w, 500.0, fake, fake, 0) == B.QI21_ERR_UNSUPPORTED
    bad = make_config(C.SMALL, B.QI21_DTYPE_F32)
    bad.n_heads = 3
    assert B.qi21_modulation_noalloc(bad, w, 500.0, fake, fake, 0) == B.QI21_ERR_SHAPE


def test_runner_checks_caller_weights_on_its_device(B):
    """The runner takes the caller's weights as they are (no drawing, no
    conversion): tensors of the storage dtype on its device; anything else is
    refused. Host-only: a runner on the CPU device builds its metadata, RoPE
    table and cache descriptor without touching a GPU."""
    import torch
    from prefix_kv_cached_b200.runner import Qi21Runner
    w = C.make_workload("toy")
    wts = C.host_weights(w, "float32")
    r = Qi21Runner(w, B.QI21_DTYPE_F32, device="cpu", host_weights=wts)
    assert (r.P, r.N) == (7, 4) and r.weights["w_q"].dtype == torch.float32
    tw = {k: torch.from_numpy(v).float() for k, v in wts.items()}
    Qi21Runner(w, B.QI21_DTYPE_F32, device="cpu", weights=tw)
    bad = dict(tw, w_q=tw["w_q"].double())
    with pytest.raises(ValueError):
        Qi21Runner(w, B.QI21_DTYPE_F32, device="cpu", weights=bad)
    with pytest.raises(ValueError):
        Qi21Runner(w, B.QI21_DTYPE_F32, device="cpu", weights=tw, host_weights=wts)
