"""Shared helpers for the GPU parity tests (tolerances, upload, comparison)."""
import numpy as np

# Acceptance: fp32-accumulated outputs against the fp64 oracle, per matrix and
# per row: relative L2 error <= 1e-3 and max absolute error <= 1e-2.
REL_L2 = 1e-3
MAX_ABS = 1e-2


def to_dev(a: np.ndarray):
    import torch
    if a.dtype == np.uint32:
        return torch.from_numpy(a.view(np.int32).copy()).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def check_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    err = got - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    mx = np.max(np.abs(err))
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e}"
    assert mx <= MAX_ABS, f"{what}: max-abs {mx:.3e}"
    if got.ndim == 2:
        for r in range(got.shape[0]):
            rr = np.linalg.norm(err[r]) / max(np.linalg.norm(ref[r]), 1e-30)
            assert rr <= REL_L2, f"{what}: row {r} rel-L2 {rr:.3e}"
    return rel, mx
