"""Shared helpers of the GPU tests: run the CUDA path on seeded inputs and
compare it with the FP64 oracle under the benchmark spec's tolerance."""
import numpy as np

REL_L2_TOL = 1e-3   # ||o_gpu - o_ref||_2 / ||o_ref||_2 over the whole output
MAX_ABS_TOL = 5e-3  # max |o_gpu - o_ref|


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def parity(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.isfinite(got).all(), "non-finite values in the GPU output"
    diff = got - want
    ref = np.linalg.norm(want)
    rel = np.linalg.norm(diff) / ref if ref > 0 else np.linalg.norm(diff)
    mx = np.abs(diff).max() if diff.size else 0.0
    return rel, mx


def assert_parity(got, want, rel_tol=REL_L2_TOL, abs_tol=MAX_ABS_TOL, what=""):
    rel, mx = parity(got, want)
    assert rel <= rel_tol and mx <= abs_tol, f"{what}: rel-L2 {rel:.3e} (tol {rel_tol}), max-abs {mx:.3e} (tol {abs_tol})"
    return rel, mx
