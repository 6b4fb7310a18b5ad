"""Shared pieces of the GPU parity tests: moving seeded synthetic arrays onto the
device and the acceptance metrics.

Tolerance (bf16 path): cosine >= 0.9999 and max |err| <= 3e-2 * RMS(reference)
on each compared output. Because the residual dominates a block's output, the
branch delta y - x is also checked by cosine: >= 0.9999 over the whole tensor
and >= 0.999 on every row. Stages whose output is a bf16 rounding of an fp32
computation are also held to about one bf16 ulp.
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


def assert_delta_close(got, ref, what: str, cos_min: float = COS_MIN, row_cos_min: float = 0.999):
    """Cosine of the branch delta, whole and per row (rows = tokens)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    cos, _, _ = metrics(got, ref)
    num = np.sum(got * ref, axis=1)
    den = np.linalg.norm(got, axis=1) * np.linalg.norm(ref, axis=1)
    row = np.where(den > 0, num / np.where(den > 0, den, 1.0), 1.0)
    worst = int(np.argmin(row))
    assert cos >= cos_min and row[worst] >= row_cos_min, (
        f"{what}: cosine {cos:.7f} (min {cos_min}), worst row {worst} cosine {row[worst]:.6f} "
        f"(min {row_cos_min})")
    return cos, float(row[worst])


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


def assert_attention_bound(got, ref, v_absmax: float, what: str):
    """Attention with P and O rounded to bf16: per element
    |err| <= 2^-8 |O| (output rounding) + 2^-8 max|v| (rounding of each p_i,
    weighted by |v_i| and normalised by sum p), taken twice for margin; plus
    the cosine floor."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    cos, maxerr, rms = metrics(got, ref)
    assert cos >= COS_MIN, f"{what}: cosine {cos:.7f}"
    bound = 2.0 ** -7 * (np.abs(ref) + v_absmax)
    bad = np.argwhere(np.abs(got - ref) > bound)
    assert bad.size == 0, (f"{what}: {len(bad)} elements beyond the bf16 bound; first "
                           f"{bad[0].tolist()} got {got[tuple(bad[0])]!r} ref {ref[tuple(bad[0])]!r}")
