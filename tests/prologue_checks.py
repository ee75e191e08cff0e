"""Per-element tolerances of the QK-norm + RoPE prologue against the float64 oracle (shared by the GPU parity
test and the CPU check of the bounds). Derivation in tests/test_prologue_parity.py's header."""
import numpy as np
import torch

BF16_REL = 2.0 ** -8
FWD_ABS = 1e-4
BWD_SCALED = 1e-4


def oracle_kwargs(w, offsets):
    return dict(base=w.rope_base, eps=w.eps, pairing=w.pairing, offsets=0 if offsets is None else offsets)


def check_fwd(y_gpu, y_ref, what):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = BF16_REL * np.abs(y_ref) + FWD_ABS
    bad = err > bound
    assert not bad.any(), \
        f"{what}: {bad.sum()} elements off, worst {err.max():.3e} (bound there {bound.flat[err.argmax()]:.3e})"


def check_bwd(dx_gpu, dx_ref, x, dy, eps, what):
    dx_gpu = np.asarray(dx_gpu, dtype=np.float64)
    x, dy = (t.double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t, dtype=np.float64)
             for t in (x, dy))
    r = 1.0 / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)
    scale = r * np.abs(dy).max(axis=-1, keepdims=True)
    err = np.abs(dx_gpu - dx_ref)
    bound = BF16_REL * np.abs(dx_ref) + BWD_SCALED * scale
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {err.max():.3e}"
