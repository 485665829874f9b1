"""Tolerances and helpers shared by the GPU parity tests.

Tolerances (fixed before any tuning, never adjusted per run):
* relative L2 error over all checked outputs, in fp64:
  <= 1e-5 for the fp32 path, <= 2e-2 for the bf16 path;
* per-element bound:
  fp32: |e_i| <= 1e-4 * RMS(y_ref) * s_i
  bf16: |e_i| <= 2^-8 |y_ref,i| + 5e-2 * RMS(y_ref) * s_i
  (2^-8 covers the bf16 rounding of the stored output, 2^-9 relative, with
  room for the fp32-accumulated transform error that is spread over the row).
  s_i = 1 for the ungated form.  In the gated form y = v (x conv k) the
  transform error of element i is multiplied by v_i, so s_i = max(1, |v_i| /
  RMS(v)): the bound on the convolution itself is the same as ungated.
  RMS(y_ref) is the scale of element i's own row where the caller gives one
  (row_scale_1d / row_scale_2d: (||k_h||_2 + |D_h|) RMS(x_row), the expected
  RMS of that row's output), since the transform error of a row is relative
  to that row's magnitude and channels can differ in scale by 10x or more;
  otherwise the RMS over all checked outputs.
"""
import numpy as np
import torch

REL_L2 = {"f32": 1e-5, "bf16": 2e-2}
RECORD = []  # (what, dtype, rel_l2, max_abs, rms, n) of every check, for the parity report


def errors(y, y_ref):
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    diff = y - y_ref
    ref_norm = np.linalg.norm(y_ref)
    rel = float(np.linalg.norm(diff) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(diff))
    rms = float(np.sqrt(np.mean(y_ref * y_ref))) if y_ref.size else 0.0
    return rel, diff, rms


def row_scale_1d(wl, b_idx=None, h_idx=None):
    """(||k_h||_2 + |D_h|) RMS(x_{b,h}) for every row, or at the given (b, h) samples."""
    x = wl.u.astype(np.float64)
    if wl.gated:
        x = x * wl.w.astype(np.float64)
    knorm = np.sqrt(np.sum(wl.k.astype(np.float64) ** 2, axis=1))
    if wl.D is not None:
        knorm = knorm + np.abs(wl.D.astype(np.float64))
    sc = np.sqrt(np.mean(x * x, axis=2)) * knorm[None, :]  # [B, H]
    if b_idx is None:
        return np.broadcast_to(sc[:, :, None], wl.u.shape)
    return sc[b_idx, h_idx]


def row_scale_2d(wl, b_idx=None, c_idx=None):
    u = wl.u.astype(np.float64)
    knorm = np.sqrt(np.sum(wl.k.astype(np.float64) ** 2, axis=(1, 2)))
    sc = np.sqrt(np.mean(u * u, axis=(2, 3))) * knorm[None, :]
    if b_idx is None:
        return np.broadcast_to(sc[:, :, None, None], wl.u.shape)
    return sc[b_idx, c_idx]


def assert_close(y, y_ref, dtype, what="", gate=None, scale=None):
    """Check rel-L2 and the per-element bound; returns (rel_l2, max_abs).
    gate: the v values at the checked outputs (gated form), else None.
    scale: per-element row scale (see row_scale_1d), else the global RMS."""
    rel, diff, rms = errors(y, y_ref)
    if scale is not None:
        rms = np.asarray(scale, dtype=np.float64).reshape(np.shape(y_ref))
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    assert rel <= REL_L2[dtype], f"{what}: rel-L2 {rel:.3e} > {REL_L2[dtype]:.0e}"
    y_ref = np.asarray(y_ref, dtype=np.float64)
    s = np.ones_like(y_ref)
    if gate is not None:
        g = np.abs(np.asarray(gate, dtype=np.float64)).reshape(y_ref.shape)
        s = np.maximum(1.0, g / max(float(np.sqrt(np.mean(g * g))), 1e-30))
    if dtype == "f32":
        bound = 1e-4 * rms * s
    else:
        bound = 2.0 ** -8 * np.abs(y_ref) + 5e-2 * rms * s
    RECORD.append((what, dtype, rel, float(np.abs(diff).max()) if diff.size else 0.0,
                   float(np.sqrt(np.mean(y_ref * y_ref))) if y_ref.size else 0.0, int(y_ref.size)))
    bad = np.abs(diff) > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements over the per-element bound; "
                           f"worst excess {float((np.abs(diff) - bound).max()):.3e}")
    return rel, float(np.abs(diff).max()) if diff.size else 0.0


def to_dev(a, dtype, device="cuda"):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device=device, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)


def to_host(t):
    return t.float().cpu().numpy().astype(np.float64)
