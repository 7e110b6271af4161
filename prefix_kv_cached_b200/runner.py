"""Device-side driver of one model instance over the C ABI.

Owns the torch-allocated device buffers (K/V cache, workspace, metadata
tables, modulation rows) and calls the library's entry points; it computes
nothing itself. The caller supplies the weights, either as host arrays (copied
to the device once) or as device tensors it already holds, and a description
of the model and the sequence: an object with ``shape`` (the fields of
``qi21_config`` plus ``rope``: "axial" or "lab"), ``segments`` (kind, n_text | h,
w), ``batch``, ``n_prefix`` and ``n_target``.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import binding as B

_TORCH_DTYPE = {B.QI21_DTYPE_F32: torch.float32, B.QI21_DTYPE_BF16: torch.bfloat16}

# qi21_weights field order
WEIGHT_NAMES = ("w_img_in", "w_out", "w_t1", "w_t2", "w_mod", "w_fin", "w_q", "w_k", "w_v", "w_o", "w_gate",
                "w_up", "w_down", "q_norm", "k_norm")
NORM_WEIGHTS = ("q_norm", "k_norm")      # float32 in both storage modes


def make_config(shape, dtype: int) -> B.qi21_config:
    return B.qi21_config(shape.d_model, shape.n_heads, shape.head_dim, shape.n_layers, shape.mlp_hidden,
                         shape.latent_ch, shape.time_dim, dtype, shape.use_shift, shape.ln_eps, shape.qk_eps)


class Qi21Runner:
    def __init__(self, workload, dtype: int = B.QI21_DTYPE_F32, device: str = "cuda",
                 host_weights: Optional[Dict[str, np.ndarray]] = None,
                 weights: Optional[Dict[str, torch.Tensor]] = None, frame_mode: int = 0,
                 shared_prefix: bool = False, share_weights_with: Optional["Qi21Runner"] = None):
        """Weights: exactly one of host_weights (arrays holding the stored values,
        copied to the device in the storage dtype), weights (device tensors in the
        storage dtype, norm weights float32) or share_weights_with (another
        runner's device weights). shared_prefix: the batch items are requests
        sharing one prefix (one extract from prefix_hidden [1][P][d], every
        request's attention reading the one copy)."""
        if sum(x is not None for x in (host_weights, weights, share_weights_with)) != 1:
            raise ValueError("give exactly one of host_weights, weights, share_weights_with")
        self.w = workload
        self.shape = workload.shape
        self.dtype = dtype
        self.tdtype = _TORCH_DTYPE[dtype]
        self.device = torch.device(device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.cfg = make_config(self.shape, dtype)
        sh = self.shape
        self.meta = B.qi21_build_metadata(list(workload.segments), frame_mode)
        self.S, self.P, self.N = self.meta["S"], self.meta["P"], self.meta["N"]
        assert (self.P, self.N) == (workload.n_prefix, workload.n_target)
        self.Bn = workload.batch
        omega = B.qi21_rope_omega_lab() if sh.rope == "lab" else B.qi21_rope_omega_axial(sh.head_dim)
        cs = B.qi21_rope_table(sh.head_dim, self.meta["coords"], omega)
        self.cos_sin_all = torch.from_numpy(cs).to(self.device)
        self.cos_sin_prefix = self.cos_sin_all[: self.P].contiguous()
        self.cos_sin_target = self.cos_sin_all[self.P:].contiguous()
        lim = torch.from_numpy(self.meta["kv_limit"].astype(np.int32)).to(self.device)
        self.kv_limit_all = lim
        self.kv_limit_prefix = lim[: self.P].contiguous()
        self.weights: Dict[str, torch.Tensor] = {}
        self.shared_prefix = shared_prefix
        for name in WEIGHT_NAMES:
            sdt = torch.float32 if name in NORM_WEIGHTS else self.tdtype
            if share_weights_with is not None:
                t = share_weights_with.weights[name]
            elif weights is not None:
                t = weights[name]
            else:
                t = torch.from_numpy(np.ascontiguousarray(host_weights[name])).to(device=self.device, dtype=sdt)
            if t.dtype != sdt or t.device != self.device or not t.is_contiguous():
                raise ValueError(f"weight {name}: expected a contiguous {sdt} tensor on {self.device}")
            self.weights[name] = t
        self.wstruct = B.qi21_weights(*[self.weights[n].data_ptr() for n in WEIGHT_NAMES])
        if shared_prefix:
            kvb = B.qi21_kv_cache_bytes_shared(self.cfg, self.Bn, self.P, self.N)
            self.cache_buf = torch.zeros(kvb, dtype=torch.uint8, device=self.device)
            self.cache = B.qi21_kv_cache_init_shared(self.cache_buf, self.cfg, self.Bn, self.P, self.N)
        else:
            kvb = B.qi21_kv_cache_bytes(self.cfg, self.Bn, self.P, self.N)
            self.cache_buf = torch.zeros(kvb, dtype=torch.uint8, device=self.device)
            self.cache = B.qi21_kv_cache_init(self.cache_buf, self.cfg, self.Bn, self.P, self.N)
        self.ws_bytes = B.qi21_workspace_bytes(self.cfg, self.Bn, self.P, self.N)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=self.device)
        nch = 6 if sh.use_shift else 4
        self.mod_prefix = torch.zeros(nch * sh.d_model, dtype=torch.float32, device=self.device)
        self.mod_target = torch.zeros_like(self.mod_prefix)
        self.scale_final = torch.zeros(sh.d_model, dtype=torch.float32, device=self.device)
        self._sf0 = torch.zeros_like(self.scale_final)

    @property
    def stream(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream

    # ------------------------------------------------------------------ calls
    def modulation(self, t: float, mod_row: torch.Tensor, scale_final: torch.Tensor):
        B.check("qi21_modulation", B.qi21_modulation(self.cfg, self.wstruct, t, mod_row, scale_final, self.ws,
                                                     self.ws_bytes, self.stream))

    def set_prefix_row(self):
        """Prefix modulation row at t = 0 (3B page: prefix tokens read t = 0)."""
        self.modulation(0.0, self.mod_prefix, self._sf0)

    def set_target_row(self, sigma: float):
        """Target modulation row and final scale at noise level sigma (the library
        forms t = QI21_T_PER_SIGMA * sigma)."""
        B.check("qi21_modulation_sigma", B.qi21_modulation_sigma(self.cfg, self.wstruct, float(sigma),
                                                                 self.mod_target, self.scale_final, self.ws,
                                                                 self.ws_bytes, self.stream))

    def prefix_extract(self, prefix_hidden: torch.Tensor, mod_prefix: Optional[torch.Tensor] = None):
        B.check("qi21_prefix_extract", B.qi21_prefix_extract(
            self.cfg, self.wstruct, self.cache, prefix_hidden, self.cos_sin_prefix, self.kv_limit_prefix,
            self.mod_prefix if mod_prefix is None else mod_prefix, self.ws, self.ws_bytes, self.stream))

    def cached_step(self, x: torch.Tensor, v_out: torch.Tensor):
        B.check("qi21_cached_step", B.qi21_cached_step(
            self.cfg, self.wstruct, self.cache, x, self.cos_sin_target, self.mod_target, self.scale_final, v_out,
            self.ws, self.ws_bytes, self.stream))

    def full_recompute(self, prefix_hidden: torch.Tensor, x: torch.Tensor, v_out: torch.Tensor,
                       mod_prefix: Optional[torch.Tensor] = None):
        B.check("qi21_full_recompute_step", B.qi21_full_recompute_step(
            self.cfg, self.wstruct, self.Bn, self.P, self.N, prefix_hidden, x, self.cos_sin_all, self.kv_limit_all,
            self.mod_prefix if mod_prefix is None else mod_prefix, self.mod_target, self.scale_final, v_out,
            self.ws, self.ws_bytes, self.stream))

    def euler(self, x: torch.Tensor, v: torch.Tensor, s0: float, s1: float, x_out: torch.Tensor):
        B.check("qi21_euler_update", B.qi21_euler_update(x, v, s0, s1, x_out, x.numel(), self.stream))

    # ------------------------------------------------------------------ whole image

    def denoise_image(self, prefix_hidden: torch.Tensor, x: torch.Tensor, sigmas_dev: torch.Tensor,
                      v: Optional[torch.Tensor] = None) -> torch.Tensor:
        """One call of qi21_denoise_image: extract, then len(sigmas_dev) - 1 cached
        steps with Euler, all enqueued on the current stream; x is updated in
        place (x_0 in, final latent out). sigmas_dev: float64 device tensor."""
        assert sigmas_dev.dtype == torch.float64 and sigmas_dev.is_cuda and sigmas_dev.numel() >= 2
        v = torch.empty_like(x) if v is None else v
        B.check("qi21_denoise_image", B.qi21_denoise_image(
            self.cfg, self.wstruct, self.cache, prefix_hidden, self.cos_sin_prefix, self.kv_limit_prefix,
            self.cos_sin_target, sigmas_dev, sigmas_dev.numel() - 1, B.QI21_T_PER_SIGMA, x, v, self.mod_prefix,
            self.mod_target, self.scale_final, self.ws, self.ws_bytes, self.stream))
        return x

    def capture_image(self, prefix_hidden: torch.Tensor, x: torch.Tensor, sigmas_dev: torch.Tensor):
        """Capture the whole-image call into a CUDA graph (after one eager call
        that sets kernel attributes). Replaying the returned graph re-runs the
        image on the current contents of prefix_hidden, x and sigmas_dev."""
        v = torch.empty_like(x)
        x_warm = x.clone()
        self.denoise_image(prefix_hidden, x_warm, sigmas_dev, v)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
                self.denoise_image(prefix_hidden, x, sigmas_dev, v)
        torch.cuda.current_stream(self.device).wait_stream(s)
        return g

    def check_device(self):
        B.check("qi21_check_device_error", B.qi21_check_device_error(self.ws, self.ws_bytes, self.stream))

    def cache_kv(self):
        """Views of the cache as K, V [L][B][P+N][H][Dh] (for tests); with a shared
        prefix, [L][Pp + B*N][H][Dh] (prefix rows [0, P), request b at Pp + b*N)."""
        sh = self.shape
        if self.shared_prefix:
            pp = -(-self.P // 128) * 128
            t = self.cache_buf.view(self.tdtype).view(sh.n_layers, 2, pp + self.Bn * self.N, sh.n_heads,
                                                      sh.head_dim)
            return t[:, 0], t[:, 1]
        t = self.cache_buf.view(self.tdtype).view(sh.n_layers, 2, self.Bn, self.P + self.N, sh.n_heads,
                                                  sh.head_dim)
        return t[:, 0], t[:, 1]

    def denoise(self, prefix_hidden: torch.Tensor, x0: torch.Tensor, sigmas=None):
        """Whole image: t = 0 prefix row, extract once, then cached steps + Euler."""
        sigmas = self.w.sigmas if sigmas is None else sigmas
        self.set_prefix_row()
        self.prefix_extract(prefix_hidden)
        x = x0.clone()
        v = torch.empty_like(x)
        for k in range(len(sigmas) - 1):
            self.set_target_row(sigmas[k])
            self.cached_step(x, v)
            self.euler(x, v, sigmas[k], sigmas[k + 1], x)
        return x
