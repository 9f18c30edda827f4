"""Tolerance helpers shared by the GPU parity tests.

Encoder and adapter outputs: per-row cosine similarity >= 0.999 and maximum
per-row relative L2 error <= 2e-2 (BF16 with fp32 accumulation); log-mel:
maximum absolute error <= 1e-3 (fp32 on both sides); token counts and window
partitions: bit-exact.
"""
import numpy as np

COS_MIN = 0.999
REL_L2_MAX = 2e-2
MEL_ABS_MAX = 1e-3


def row_metrics(gpu, ref):
    g = np.asarray(gpu, np.float64).reshape(-1, np.shape(gpu)[-1])
    r = np.asarray(ref, np.float64).reshape(-1, np.shape(ref)[-1])
    assert g.shape == r.shape, (g.shape, r.shape)
    dot = (g * r).sum(1)
    ng = np.linalg.norm(g, axis=1)
    nr = np.linalg.norm(r, axis=1)
    cos = dot / np.maximum(ng * nr, 1e-300)
    rel = np.linalg.norm(g - r, axis=1) / np.maximum(nr, 1e-300)
    return float(cos.min()), float(rel.max())


def assert_encoder_parity(gpu, ref, what=""):
    cmin, rmax = row_metrics(gpu, ref)
    assert np.isfinite(np.asarray(gpu)).all(), f"{what}: non-finite output"
    print(f"[parity] {what}: rows {np.shape(gpu)[0] if np.ndim(gpu) == 2 else int(np.prod(np.shape(gpu)[:-1]))}, "
          f"min row cosine {cmin:.6f}, max row rel L2 {rmax:.3e}")
    assert cmin >= COS_MIN and rmax <= REL_L2_MAX, f"{what}: min row cosine {cmin:.6f}, max rel L2 {rmax:.3e}"
    return cmin, rmax
