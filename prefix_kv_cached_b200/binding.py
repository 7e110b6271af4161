"""ctypes binding of libqi21.so: the C ABI of include/qi21.h under the same names.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Device buffers are passed as integer addresses (for torch tensors,
``t.data_ptr()``), streams as ``torch.cuda.current_stream().cuda_stream``.
Importing this module loads the in-tree library and fails loudly if it is
missing; nothing here falls back to another implementation.
"""
from __future__ import annotations

import ctypes as ct
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# QI21_LIB selects another build of the library (the --debug build of build.py)
LIB_PATH = os.environ.get("QI21_LIB") or os.path.join(_HERE, "libqi21.so")

QI21_OK = 0
QI21_ERR_INVALID_ARG = 1
QI21_ERR_SHAPE = 2
QI21_ERR_METADATA = 3
QI21_ERR_CACHE_STATE = 4
QI21_ERR_UNSUPPORTED = 5
QI21_ERR_CUDA = 6
QI21_ERR_DEVICE_TIMEOUT = 7
QI21_ERR_WORKSPACE_TOO_SMALL = 8
QI21_ERR_DEVICE_CHECK = 9

QI21_DTYPE_F32 = 0
QI21_DTYPE_BF16 = 1
QI21_SEG_TEXT = 0
QI21_SEG_IMAGE = 1
QI21_CACHE_EMPTY = 0
QI21_CACHE_EXTRACTED = 1
QI21_FAMILY_NONE = -1
QI21_FAMILY_CUDA_CORES = 0
QI21_FAMILY_TENSOR_CORES = 1
QI21_T_PER_SIGMA = 1000.0


class qi21_config(ct.Structure):
    _fields_ = [("d_model", ct.c_int32), ("n_heads", ct.c_int32), ("head_dim", ct.c_int32),
                ("n_layers", ct.c_int32), ("mlp_hidden", ct.c_int32), ("latent_ch", ct.c_int32),
                ("time_dim", ct.c_int32), ("dtype", ct.c_int32), ("use_shift", ct.c_int32),
                ("ln_eps", ct.c_float), ("qk_eps", ct.c_float)]


class qi21_segment(ct.Structure):
    _fields_ = [("kind", ct.c_int32), ("n_text", ct.c_int32), ("h", ct.c_int32), ("w", ct.c_int32)]


class qi21_weights(ct.Structure):
    _fields_ = [(n, ct.c_void_p) for n in ("w_img_in", "w_out", "w_t1", "w_t2", "w_mod", "w_fin", "w_q", "w_k",
                                           "w_v", "w_o", "w_gate", "w_up", "w_down", "q_norm", "k_norm")]


class qi21_weights_canonical(ct.Structure):
    """Same fields as qi21_weights, row-major [in][out] matrices."""
    _fields_ = [(n, ct.c_void_p) for n in ("w_img_in", "w_out", "w_t1", "w_t2", "w_mod", "w_fin", "w_q", "w_k",
                                           "w_v", "w_o", "w_gate", "w_up", "w_down", "q_norm", "k_norm")]


class qi21_kv_cache(ct.Structure):
    _fields_ = [("base", ct.c_void_p), ("batch", ct.c_int32), ("n_prefix", ct.c_int32),
                ("n_target", ct.c_int32), ("n_layers", ct.c_int32), ("d_model", ct.c_int32),
                ("dtype", ct.c_int32), ("state", ct.c_int32), ("shared_prefix", ct.c_int32)]


class qi21_kernel_time(ct.Structure):
    _fields_ = [("name", ct.c_char_p), ("launches", ct.c_int64), ("total_ms", ct.c_double)]


_P = ct.c_void_p
_I32 = ct.c_int32
_SIGS = {
    "qi21_build_metadata": (_I32, [ct.POINTER(qi21_segment), _I32, _I32, _I32, _P, _P, _P, _P,
                                   ct.POINTER(_I32), ct.POINTER(_I32), ct.POINTER(_I32)]),
    "qi21_rope_omega_axial": (_I32, [_I32, ct.c_double, _P]),
    "qi21_rope_omega_lab": (_I32, [ct.c_double, _P]),
    "qi21_rope_table": (_I32, [_I32, _P, _I32, _P, _P]),
    "qi21_timestep_embedding": (_I32, [ct.c_double, _I32, _P]),
    "qi21_kv_cache_bytes": (ct.c_size_t, [ct.POINTER(qi21_config), _I32, _I32, _I32]),
    "qi21_workspace_bytes": (ct.c_size_t, [ct.POINTER(qi21_config), _I32, _I32, _I32]),
    "qi21_kv_cache_init": (_I32, [ct.POINTER(qi21_kv_cache), _P, ct.POINTER(qi21_config), _I32, _I32, _I32]),
    "qi21_packed_weights_bytes": (ct.c_size_t, [ct.POINTER(qi21_config)]),
    "qi21_pack_weights": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights_canonical), _P, ct.c_size_t,
                                 ct.POINTER(qi21_weights), _P]),
    "qi21_kv_cache_bytes_shared": (ct.c_size_t, [ct.POINTER(qi21_config), _I32, _I32, _I32]),
    "qi21_kv_cache_init_shared": (_I32, [ct.POINTER(qi21_kv_cache), _P, ct.POINTER(qi21_config), _I32, _I32,
                                         _I32]),
    "qi21_modulation": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), ct.c_double, _P, _P, _P,
                               ct.c_size_t, _P]),
    "qi21_modulation_sigma": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), ct.c_double, _P, _P, _P,
                                     ct.c_size_t, _P]),
    "qi21_modulation_noalloc": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), ct.c_double, _P, _P,
                                       _P]),
    "qi21_prefix_extract": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), ct.POINTER(qi21_kv_cache),
                                   _P, _P, _P, _P, _P, ct.c_size_t, _P]),
    "qi21_cached_step": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), ct.POINTER(qi21_kv_cache),
                                _P, _P, _P, _P, _P, _P, ct.c_size_t, _P]),
    "qi21_full_recompute_step": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), _I32, _I32, _I32,
                                        _P, _P, _P, _P, _P, _P, _P, _P, _P, ct.c_size_t, _P]),
    "qi21_euler_update": (_I32, [_P, _P, ct.c_double, ct.c_double, _P, ct.c_int64, _P]),
    "qi21_build_packing": (_I32, [ct.POINTER(qi21_segment), _I32, _I32, _P, _P, ct.POINTER(_I32),
                                  ct.POINTER(_I32), ct.POINTER(_I32)]),
    "qi21_pack_prefix": (_I32, [_I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _I32, _P, _P]),
    "qi21_img_in_tokens": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), _P, _I32, _P, _P]),
    "qi21_modulation_at": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), _P, _I32, ct.c_double, _P,
                                  _P, _P, ct.c_size_t, _P]),
    "qi21_euler_update_at": (_I32, [_P, _P, _P, _I32, _P, ct.c_int64, _P]),
    "qi21_denoise_image": (_I32, [ct.POINTER(qi21_config), ct.POINTER(qi21_weights), ct.POINTER(qi21_kv_cache),
                                  _P, _P, _P, _P, _P, _I32, ct.c_double, _P, _P, _P, _P, _P, _P, ct.c_size_t, _P]),
    "qi21_check_device_error": (_I32, [_P, ct.c_size_t, _P]),
    "qi21_status_string": (ct.c_char_p, [_I32]),
    "qi21_selftest_wait_timeout": (_I32, [_P, ct.c_size_t, ct.c_int64, _P]),
    "qi21_profile_enable": (None, [_I32]),
    "qi21_profile_read": (_I32, [ct.POINTER(qi21_kernel_time), _I32]),
    "qi21_profile_reset": (None, []),
    "qi21_version": (ct.c_char_p, []),
    "qi21_last_launch_count": (_I32, []),
    "qi21_set_tensor_cores": (None, [_I32]),
    "qi21_kernel_family": (_I32, [ct.POINTER(qi21_config)]),
}

EXPORTED = tuple(_SIGS)

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m prefix_kv_cached_b200.build`")
lib = ct.CDLL(LIB_PATH)
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class Qi21Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} -> {status} ({lib.qi21_status_string(status).decode()})")
        self.status = status


def check(fn: str, status: int) -> int:
    if status != QI21_OK:
        raise Qi21Error(fn, status)
    return status


def _addr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(type(x))


# ----------------------------------------------------------------- same-name wrappers

def qi21_build_metadata(segments, frame_mode=0):
    """Host metadata; returns dict(image_ids, target_mask, coords, kv_limit, S, P, N) as numpy arrays."""
    import numpy as np
    segs = (qi21_segment * len(segments))(*[qi21_segment(int(k), int(a) if k == QI21_SEG_TEXT else 0,
                                                         int(a) if k == QI21_SEG_IMAGE else 0,
                                                         int(b) if k == QI21_SEG_IMAGE else 0)
                                            for (k, a, b) in segments])
    S, P, N = _I32(), _I32(), _I32()
    check("qi21_build_metadata", lib.qi21_build_metadata(segs, len(segments), frame_mode, 0, None, None, None,
                                                         None, ct.byref(S), ct.byref(P), ct.byref(N)))
    ids = np.zeros(S.value, np.int32)
    mask = np.zeros(S.value, np.uint8)
    coords = np.zeros((S.value, 3), np.int32)
    lim = np.zeros(S.value, np.int32)
    check("qi21_build_metadata", lib.qi21_build_metadata(segs, len(segments), frame_mode, S.value, _addr(ids),
                                                         _addr(mask), _addr(coords), _addr(lim), ct.byref(S),
                                                         ct.byref(P), ct.byref(N)))
    return {"image_ids": ids, "target_mask": mask, "coords": coords, "kv_limit": lim,
            "S": S.value, "P": P.value, "N": N.value}


def qi21_rope_omega_axial(head_dim, base=10000.0):
    import numpy as np
    om = np.zeros((head_dim // 2, 3), np.float64)
    check("qi21_rope_omega_axial", lib.qi21_rope_omega_axial(head_dim, base, _addr(om)))
    return om


def qi21_rope_omega_lab(base=10000.0):
    import numpy as np
    om = np.zeros((2, 3), np.float64)
    check("qi21_rope_omega_lab", lib.qi21_rope_omega_lab(base, _addr(om)))
    return om


def qi21_rope_table(head_dim, coords, omega):
    import numpy as np
    coords = np.ascontiguousarray(coords, dtype=np.int32)
    omega = np.ascontiguousarray(omega, dtype=np.float64)
    out = np.zeros((coords.shape[0], head_dim // 2, 2), np.float32)
    check("qi21_rope_table", lib.qi21_rope_table(head_dim, _addr(coords), coords.shape[0], _addr(omega), _addr(out)))
    return out


def qi21_timestep_embedding(t, time_dim):
    import numpy as np
    out = np.zeros(time_dim, np.float32)
    check("qi21_timestep_embedding", lib.qi21_timestep_embedding(float(t), time_dim, _addr(out)))
    return out


def qi21_kv_cache_bytes(cfg, batch, n_prefix, n_target):
    return lib.qi21_kv_cache_bytes(ct.byref(cfg), batch, n_prefix, n_target)


def qi21_workspace_bytes(cfg, batch, n_prefix, n_target):
    return lib.qi21_workspace_bytes(ct.byref(cfg), batch, n_prefix, n_target)


def qi21_kv_cache_init(base, cfg, batch, n_prefix, n_target):
    cache = qi21_kv_cache()
    check("qi21_kv_cache_init", lib.qi21_kv_cache_init(ct.byref(cache), _addr(base), ct.byref(cfg), batch,
                                                       n_prefix, n_target))
    return cache


def qi21_packed_weights_bytes(cfg):
    return lib.qi21_packed_weights_bytes(ct.byref(cfg))


def qi21_pack_weights(cfg, canonical, packed, packed_bytes, stream=0):
    """Returns (status, qi21_weights pointing into `packed`)."""
    w = qi21_weights()
    st = lib.qi21_pack_weights(ct.byref(cfg), ct.byref(canonical), _addr(packed), packed_bytes, ct.byref(w), stream)
    return st, w


def qi21_kv_cache_bytes_shared(cfg, batch, n_prefix, n_target):
    return lib.qi21_kv_cache_bytes_shared(ct.byref(cfg), batch, n_prefix, n_target)


def qi21_kv_cache_init_shared(base, cfg, batch, n_prefix, n_target):
    cache = qi21_kv_cache()
    check("qi21_kv_cache_init_shared", lib.qi21_kv_cache_init_shared(ct.byref(cache), _addr(base), ct.byref(cfg),
                                                                     batch, n_prefix, n_target))
    return cache


def qi21_modulation(cfg, weights, t, mod_row, scale_final, ws, ws_bytes, stream=0):
    return lib.qi21_modulation(ct.byref(cfg), ct.byref(weights), float(t), _addr(mod_row), _addr(scale_final),
                               _addr(ws), ws_bytes, stream)


def qi21_modulation_sigma(cfg, weights, sigma, mod_row, scale_final, ws, ws_bytes, stream=0):
    return lib.qi21_modulation_sigma(ct.byref(cfg), ct.byref(weights), float(sigma), _addr(mod_row),
                                     _addr(scale_final), _addr(ws), ws_bytes, stream)


def qi21_modulation_noalloc(cfg, weights, t, mod_row, scale_final, stream=0):
    return lib.qi21_modulation_noalloc(ct.byref(cfg), ct.byref(weights), float(t), _addr(mod_row),
                                       _addr(scale_final), stream)


def qi21_prefix_extract(cfg, weights, cache, prefix_hidden, cos_sin_prefix, kv_limit_prefix, mod_row_prefix,
                        ws, ws_bytes, stream=0):
    return lib.qi21_prefix_extract(ct.byref(cfg), ct.byref(weights), ct.byref(cache), _addr(prefix_hidden),
                                   _addr(cos_sin_prefix), _addr(kv_limit_prefix), _addr(mod_row_prefix),
                                   _addr(ws), ws_bytes, stream)


def qi21_cached_step(cfg, weights, cache, x_k, cos_sin_target, mod_row_target, scale_final, v_out, ws, ws_bytes,
                     stream=0):
    return lib.qi21_cached_step(ct.byref(cfg), ct.byref(weights), ct.byref(cache), _addr(x_k),
                                _addr(cos_sin_target), _addr(mod_row_target), _addr(scale_final), _addr(v_out),
                                _addr(ws), ws_bytes, stream)


def qi21_full_recompute_step(cfg, weights, batch, n_prefix, n_target, prefix_hidden, x_k, cos_sin_all,
                             kv_limit_all, mod_row_prefix, mod_row_target, scale_final, v_out, ws, ws_bytes,
                             stream=0):
    return lib.qi21_full_recompute_step(ct.byref(cfg), ct.byref(weights), batch, n_prefix, n_target,
                                        _addr(prefix_hidden), _addr(x_k), _addr(cos_sin_all), _addr(kv_limit_all),
                                        _addr(mod_row_prefix), _addr(mod_row_target), _addr(scale_final),
                                        _addr(v_out), _addr(ws), ws_bytes, stream)


def qi21_euler_update(x_k, v, sigma_k, sigma_k1, x_out, n, stream=0):
    return lib.qi21_euler_update(_addr(x_k), _addr(v), float(sigma_k), float(sigma_k1), _addr(x_out), int(n), stream)


QI21_PACK_SUBSTITUTE = 0
QI21_PACK_ADD = 1


def qi21_build_packing(segments):
    """Host index tables of the 4x slot expansion: dict(slot_of, img_row int32[P], P, n_slots, n_img)."""
    import numpy as np
    arr = (qi21_segment * len(segments))(*[qi21_segment(int(k), int(a) if k == QI21_SEG_TEXT else 0,
                                                       int(a) if k == QI21_SEG_IMAGE else 0,
                                                       int(b) if k == QI21_SEG_IMAGE else 0)
                                           for (k, a, b) in segments])
    P, ns, ni = _I32(), _I32(), _I32()
    check("qi21_build_packing", lib.qi21_build_packing(arr, len(segments), 0, None, None, ct.byref(P),
                                                       ct.byref(ns), ct.byref(ni)))
    slot_of = np.zeros(P.value, dtype=np.int32)
    img_row = np.zeros(P.value, dtype=np.int32)
    check("qi21_build_packing", lib.qi21_build_packing(arr, len(segments), P.value, slot_of.ctypes.data,
                                                       img_row.ctypes.data, ct.byref(P), ct.byref(ns),
                                                       ct.byref(ni)))
    return {"slot_of": slot_of, "img_row": img_row, "P": P.value, "n_slots": ns.value, "n_img": ni.value}


def qi21_pack_prefix(batch, P, d, n_slots, n_img, ctx, img_tokens, slot_of, img_row, mode, out, stream=0):
    return lib.qi21_pack_prefix(int(batch), int(P), int(d), int(n_slots), int(n_img), _addr(ctx),
                                _addr(img_tokens), _addr(slot_of), _addr(img_row), int(mode), _addr(out), stream)


def qi21_img_in_tokens(cfg, weights, latents, rows, out, stream=0):
    return lib.qi21_img_in_tokens(ct.byref(cfg), ct.byref(weights), _addr(latents), int(rows), _addr(out), stream)


def qi21_modulation_at(cfg, weights, sigmas, step, t_per_sigma, mod_row, scale_final, ws, ws_bytes, stream=0):
    return lib.qi21_modulation_at(ct.byref(cfg), ct.byref(weights), _addr(sigmas), int(step), float(t_per_sigma),
                                  _addr(mod_row), _addr(scale_final), _addr(ws), ws_bytes, stream)


def qi21_euler_update_at(x_k, v, sigmas, step, x_out, n, stream=0):
    return lib.qi21_euler_update_at(_addr(x_k), _addr(v), _addr(sigmas), int(step), _addr(x_out), int(n), stream)


def qi21_denoise_image(cfg, weights, cache, prefix_hidden, cos_sin_prefix, kv_limit_prefix, cos_sin_target,
                       sigmas, n_steps, t_per_sigma, x, v, mod_row_prefix, mod_row_target, scale_final, ws,
                       ws_bytes, stream=0):
    return lib.qi21_denoise_image(ct.byref(cfg), ct.byref(weights), ct.byref(cache), _addr(prefix_hidden),
                                  _addr(cos_sin_prefix), _addr(kv_limit_prefix), _addr(cos_sin_target),
                                  _addr(sigmas), int(n_steps), float(t_per_sigma), _addr(x), _addr(v),
                                  _addr(mod_row_prefix), _addr(mod_row_target), _addr(scale_final), _addr(ws),
                                  ws_bytes, stream)


def qi21_check_device_error(ws, ws_bytes, stream=0):
    return lib.qi21_check_device_error(_addr(ws), ws_bytes, stream)


def qi21_selftest_wait_timeout(ws, ws_bytes, limit_ns, stream=0):
    return lib.qi21_selftest_wait_timeout(_addr(ws), ws_bytes, int(limit_ns), stream)


def qi21_status_string(s):
    return lib.qi21_status_string(s).decode()


def qi21_profile_enable(on):
    lib.qi21_profile_enable(1 if on else 0)


def qi21_profile_reset():
    lib.qi21_profile_reset()


def qi21_profile_read(max_entries=64):
    buf = (qi21_kernel_time * max_entries)()
    n = lib.qi21_profile_read(buf, max_entries)
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(n)}


def qi21_version():
    return lib.qi21_version().decode()


def qi21_last_launch_count():
    return int(lib.qi21_last_launch_count())


def qi21_set_tensor_cores(on):
    lib.qi21_set_tensor_cores(1 if on else 0)


def qi21_kernel_family(cfg):
    return int(lib.qi21_kernel_family(ct.byref(cfg)))
