"""Shared set-up of the parity tests: the same seeded inputs for the fp64
oracle and for the CUDA path (through the C ABI), and the per-layer cache
comparisons.

What the parity tests compare, element by element, on both sides:
* the prefix K/V of every layer that the extract writes into cache rows [0, P)
  (layers >= 1 observe the block-causal masked attention of the layers below);
* after each cached step, the target K/V of every layer that the step writes
  into cache rows [P, P+N) (layers >= 1 observe the cached attention of the
  layers below);
* v_theta and the latent after the Euler update.
``tests/test_parity_strength.py`` checks on the CPU that, with the parity
workloads' inputs, replacing the oracle's attention by zeros moves every one of
these tensors by at least ten times the tolerance it is compared with.
"""
import numpy as np

from oracle import qi21_oracle as O
from qi21_synth import configs as C

F32_TOL = 1e-4      # max relative error, fp32 storage against the fp64 oracle
BF16_TOL = 2e-2     # relative L2, bf16 storage against the fp64 oracle


def oracle_model(w: C.Workload, store_dtype: str):
    sh = w.shape
    wts = C.host_weights(w, store_dtype)
    omega = O.rope_omega_lab() if sh.rope == "lab" else O.rope_omega_axial(sh.head_dim)
    return O.Model(sh.n_heads, sh.n_layers, sh.n_chunks, sh.ln_eps, sh.qk_eps, omega, wts), wts


def max_rel(a, b):
    """max |a - b| / max |b| over the tensor."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def oracle_item(model, seq, pre, x0, sigmas, n_steps):
    """fp64 oracle of one batch item: the t = 0 prefix row, the extract, then
    n_steps cached steps with Euler. Returns dict(ck, cv [L][P][H][Dh],
    v, x, tk, tv: lists over steps; tk/tv [L][N][H][Dh])."""
    m0, _ = O.modulation(0.0, model.wts, model.n_chunks)
    ck, cv = O.prefix_extract(model, seq, pre, m0)
    x = x0
    out = {"ck": ck, "cv": cv, "m0": m0, "v": [], "x": [], "tk": [], "tv": []}
    for k in range(n_steps):
        mt, sf = O.modulation(1000.0 * sigmas[k], model.wts, model.n_chunks)
        v, tk, tv = O.cached_step(model, seq, ck, cv, x, mt, sf)
        x = O.euler_step(x, v, sigmas[k], sigmas[k + 1])
        out["v"].append(v)
        out["x"].append(x)
        out["tk"].append(tk)
        out["tv"].append(tv)
    return out


def cache_rows(r, prefix=True, target=True):
    """The runner's K/V cache as float64 numpy arrays (prefix K, prefix V
    [L][B][P][H][Dh]; target K, target V [L][B][N][H][Dh]; None where not
    asked for), for either layout (with a shared prefix, the one prefix copy is
    repeated over the items)."""
    K, V = r.cache_kv()
    P, N, Bn = r.P, r.N, r.Bn
    f = lambda t: t.double().cpu().numpy()   # noqa: E731
    pk = pv = tk = tv = None
    if r.shared_prefix:
        pp = -(-P // 128) * 128
        if prefix:
            pk = np.repeat(f(K[:, None, :P]), Bn, axis=1)
            pv = np.repeat(f(V[:, None, :P]), Bn, axis=1)
        if target:
            tk = f(K[:, pp:pp + Bn * N].reshape(K.shape[0], Bn, N, *K.shape[2:]))
            tv = f(V[:, pp:pp + Bn * N].reshape(V.shape[0], Bn, N, *V.shape[2:]))
    else:
        if prefix:
            pk, pv = f(K[:, :, :P]), f(V[:, :, :P])
        if target:
            tk, tv = f(K[:, :, P:]), f(V[:, :, P:])
    return pk, pv, tk, tv


def gpu_steps(r, pre_t, x0_t, sigmas, n_steps):
    """The same sequence on the GPU through the runner (modulation by the
    library). Returns dict(pk, pv [L][B][P][H][Dh], v, x, tk, tv: lists over
    steps; tk/tv [L][B][N][H][Dh])."""
    import torch
    r.set_prefix_row()
    r.prefix_extract(pre_t)
    x = x0_t.clone()
    v = torch.empty_like(x)
    out = {"v": [], "x": [], "tk": [], "tv": []}
    for k in range(n_steps):
        r.set_target_row(sigmas[k])
        r.cached_step(x, v)
        out["v"].append(v.double().cpu().numpy())
        _, _, tk, tv = cache_rows(r, prefix=False)
        out["tk"].append(tk)
        out["tv"].append(tv)
        r.euler(x, v, sigmas[k], sigmas[k + 1], x)
        out["x"].append(x.double().cpu().numpy())
    torch.cuda.synchronize()
    r.check_device()
    out["pk"], out["pv"], _, _ = cache_rows(r, target=False)
    return out


def assert_item_matches(got, want, b, n_steps, metric, tol, what=""):
    """Compare item b of gpu_steps() with oracle_item(): the prefix K/V of
    every layer, then per step the target K/V of every layer, v and x."""
    assert metric(got["pk"][:, b], want["ck"]) < tol, f"{what} prefix K item {b}"
    assert metric(got["pv"][:, b], want["cv"]) < tol, f"{what} prefix V item {b}"
    for k in range(n_steps):
        assert metric(got["tk"][k][:, b], want["tk"][k]) < tol, f"{what} target K step {k} item {b}"
        assert metric(got["tv"][k][:, b], want["tv"][k]) < tol, f"{what} target V step {k} item {b}"
        assert metric(got["v"][k][b], want["v"][k]) < tol, f"{what} v step {k} item {b}"
        assert metric(got["x"][k][b], want["x"][k]) < tol, f"{what} x step {k} item {b}"
