"""Tolerances and helpers shared by the GPU parity tests.

Tolerances (fixed before any tuning, never adjusted per run):
* relative L2 error over all checked outputs, in fp64:
  <= 1e-5 for the fp32 path, <= 2e-2 for the bf16 path;
* per-element bound:
  fp32: |e_i| <= 1e-4 * RMS(y_ref)
  bf16: |e_i| <= 2^-8 |y_ref,i| + 5e-2 * RMS(y_ref)
  (2^-8 covers the bf16 rounding of the stored output, 2^-9 relative, with
  room for the fp32-accumulated transform error that is spread over the row).
"""
import numpy as np
import torch

REL_L2 = {"f32": 1e-5, "bf16": 2e-2}


def errors(y, y_ref):
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    diff = y - y_ref
    ref_norm = np.linalg.norm(y_ref)
    rel = float(np.linalg.norm(diff) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(diff))
    rms = float(np.sqrt(np.mean(y_ref * y_ref))) if y_ref.size else 0.0
    return rel, diff, rms


def assert_close(y, y_ref, dtype, what=""):
    """Check rel-L2 and the per-element bound; returns (rel_l2, max_abs)."""
    rel, diff, rms = errors(y, y_ref)
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    assert rel <= REL_L2[dtype], f"{what}: rel-L2 {rel:.3e} > {REL_L2[dtype]:.0e}"
    y_ref = np.asarray(y_ref, dtype=np.float64)
    if dtype == "f32":
        bound = 1e-4 * rms + np.zeros_like(y_ref)
    else:
        bound = 2.0 ** -8 * np.abs(y_ref) + 5e-2 * rms
    bad = np.abs(diff) > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements over the per-element bound; "
                           f"worst excess {float((np.abs(diff) - bound).max()):.3e}, rms {rms:.3e}")
    return rel, float(np.abs(diff).max()) if diff.size else 0.0


def to_dev(a, dtype, device="cuda"):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device=device, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)


def to_host(t):
    return t.float().cpu().numpy().astype(np.float64)
