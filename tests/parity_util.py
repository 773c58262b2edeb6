"""Helpers shared by the GPU parity tests: random packed weights, tolerances."""
import numpy as np
import torch

# Output tolerances: relative L2 over all outputs and max absolute error.
TOL = {"f32": dict(rel_l2=1e-5, max_abs=2e-2), "f16": dict(rel_l2=2e-3, max_abs=2e-2)}


def rel_l2(y, ref):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(y - ref) / (den if den > 0 else 1.0))


def assert_close(y, ref, act):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    assert y.shape == ref.shape
    assert np.all(np.isfinite(y))
    r = rel_l2(y, ref)
    m = float(np.max(np.abs(y - ref))) if y.size else 0.0
    t = TOL[act]
    assert r <= t["rel_l2"], f"rel L2 {r:.3e} > {t['rel_l2']}"
    assert m <= t["max_abs"], f"max abs {m:.3e} > {t['max_abs']}"
    return r, m


def random_packed(rng, N, K, bs, has_zp, scale_dtype, scale_lo=0.001, scale_hi=0.005):
    """Arbitrary nibbles and zero points (not only RTN outputs)."""
    nb = K // bs
    packed = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = rng.uniform(scale_lo, scale_hi, (N, nb)).astype(scale_dtype)
    zp = None
    if has_zp:
        zp = rng.integers(0, 256, (N, (nb + 1) // 2), dtype=np.uint8)
        if nb % 2:
            zp[:, -1] &= 0x0F
    return packed, scales, zp


def to_dev(a, dev):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def np_of(t):
    return t.detach().cpu().numpy()
