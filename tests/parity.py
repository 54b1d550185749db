"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (fp32-accumulated bf16 attention, fixed for this method):
  O   : max |O - O_ref| <= 2e-2 and mean |O - O_ref| <= 2e-3
  lse : max |lse - lse_ref| <= 1e-3
  HSTU additionally: ||O - O_ref||_2 / ||O_ref||_2 <= 1e-2 and max |O - O_ref| <= 2e-2 * max |O_ref|,
  because its outputs are ~1e-3 in magnitude and the absolute bounds alone would accept O = 0.
"""
import numpy as np

O_MAX_ABS, O_MEAN_ABS, LSE_MAX_ABS = 2e-2, 2e-3, 1e-3
HSTU_REL_L2, HSTU_REL_MAX = 1e-2, 2e-2


def to_f64(t):
    import torch

    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def check_o(o, o_ref, what=""):
    o, o_ref = to_f64(o), to_f64(o_ref)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite outputs"
    err = np.abs(o - o_ref)
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    worst = np.unravel_index(int(np.argmax(err)), err.shape) if err.size else None
    assert mx <= O_MAX_ABS and mean <= O_MEAN_ABS, \
        f"{what}: O max-abs {mx:.3e} (at {worst}) mean-abs {mean:.3e} exceed {O_MAX_ABS}/{O_MEAN_ABS}"
    return mx, mean


def check_lse(lse, lse_ref, what=""):
    lse, lse_ref = to_f64(lse), to_f64(lse_ref)
    assert lse.shape == lse_ref.shape
    both_inf = np.isneginf(lse) & np.isneginf(lse_ref)
    with np.errstate(invalid="ignore"):  # -inf - -inf (rows with no visible key on both sides) is masked below
        err = np.where(both_inf, 0.0, np.abs(lse - lse_ref))
    mx = float(np.nan_to_num(err, nan=np.inf).max(initial=0.0))
    assert mx <= LSE_MAX_ABS, f"{what}: lse max-abs {mx:.3e} exceeds {LSE_MAX_ABS}"
    return mx


def check_hstu(o, o_ref, what=""):
    o, o_ref = to_f64(o), to_f64(o_ref)
    check_o(o, o_ref, what)
    ref_norm = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o - o_ref)) / max(ref_norm, 1e-300)
    mx = float(np.abs(o - o_ref).max(initial=0.0))
    ref_max = float(np.abs(o_ref).max(initial=0.0))
    assert rel <= HSTU_REL_L2, f"{what}: relative L2 error {rel:.3e} exceeds {HSTU_REL_L2}"
    assert mx <= HSTU_REL_MAX * ref_max, f"{what}: max error {mx:.3e} exceeds {HSTU_REL_MAX} * max|O_ref| = {HSTU_REL_MAX * ref_max:.3e}"
    return rel
