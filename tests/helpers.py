"""Shared pieces of the GPU parity tests: moving seeded synthetic arrays onto the
device and the acceptance metrics.

Tolerance (bf16 path): cosine >= 0.9999 and max |err| <= 3e-2 * RMS(reference)
on each compared output, and the same on the branch delta y - x of a block,
where the residual would otherwise dominate. Stages whose output is a bf16
rounding of an fp32 computation are also held to about one bf16 ulp.
"""
from __future__ import annotations

import numpy as np

COS_MIN = 0.9999
REL_MAX = 3e-2


def to_dev(a, dtype="bf16"):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda()


def to_np(t) -> np.ndarray:
    import torch

    return t.detach().to(torch.float64).cpu().numpy()


def metrics(got, ref):
    got = np.asarray(got, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    num = float(np.dot(got, ref))
    den = float(np.linalg.norm(got) * np.linalg.norm(ref))
    cos = num / den if den > 0 else (1.0 if np.array_equal(got, ref) else 0.0)
    rms = float(np.sqrt(np.mean(ref * ref)))
    maxerr = float(np.max(np.abs(got - ref))) if got.size else 0.0
    return cos, maxerr, rms


def assert_close(got, ref, what: str, cos_min: float = COS_MIN, rel_max: float = REL_MAX):
    cos, maxerr, rms = metrics(got, ref)
    assert cos >= cos_min and maxerr <= rel_max * rms, (
        f"{what}: cosine {cos:.7f} (min {cos_min}), max|err| {maxerr:.4g} "
        f"vs {rel_max} * RMS {rms:.4g}")
    return cos, maxerr, rms


def assert_bf16_rounding(got, ref, what: str, abs_floor: float = 1e-5):
    """got is ref rounded to bf16 up to about one ulp (plus fp32 noise)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bound = 2.0 ** -7 * np.abs(ref) + abs_floor
    bad = np.argwhere(err > bound)
    assert bad.size == 0, (
        f"{what}: {len(bad)} values beyond one bf16 ulp, first at {bad[0].tolist()}: "
        f"got {got[tuple(bad[0])]!r} ref {ref[tuple(bad[0])]!r}")


def block_tensors(w: dict):
    return {k: to_dev(v, "f32" if k == "b_ada" else "bf16") for k, v in w.items()}


def time_tensors(w: dict):
    return {k: to_dev(v, "f32") for k, v in w.items()}
