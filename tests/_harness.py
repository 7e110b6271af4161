"""Shared set-up of the parity tests: the same seeded inputs for the fp64
oracle and for the CUDA path (through the C ABI)."""
import numpy as np

from oracle import qi21_oracle as O
from qi21_synth import configs as C


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
