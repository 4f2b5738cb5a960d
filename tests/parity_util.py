"""Comparison helpers for the GPU parity tests (no attention arithmetic here).

Tolerances: fp32 path max-abs <= 1e-5 (out, lse). bf16 path: for out, dq,
dk, dv max-abs <= 2e-2 and relative L2 <= 1e-2 against the fp64 oracle fed
the same bf16-rounded inputs; lse max-abs <= 2e-3 (lse is formed in fp32 from
fp32 scores; its error budget is set by the fp32 row sum over up to a few
thousand terms, ~1e-5 relative, far inside 2e-3). Peaked stress inputs
(unscaled q/k) have gradients well above 1, so there the max-abs bound is
taken relative to the largest reference magnitude: 2e-2 * max(1, max|ref|).
"""
import numpy as np
import torch


def f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def errors(got, ref):
    got, ref = f64(got), f64(ref)
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(ref))
    rel_l2 = float(np.linalg.norm(diff) / den) if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel_l2


def check_bf16(name, got, ref, peaked=False):
    ref = f64(ref)
    max_abs, rel_l2 = errors(got, ref)
    bound = 2e-2 * (max(1.0, float(np.max(np.abs(ref)))) if peaked and ref.size else 1.0)
    assert np.all(np.isfinite(f64(got))), f"{name}: non-finite values"
    assert max_abs <= bound, f"{name}: max-abs {max_abs:.3e} > {bound:.3e} (rel-L2 {rel_l2:.3e})"
    assert rel_l2 <= 1e-2, f"{name}: rel-L2 {rel_l2:.3e} > 1e-2 (max-abs {max_abs:.3e})"
    return max_abs, rel_l2


def check_abs(name, got, ref, tol):
    max_abs, rel_l2 = errors(got, ref)
    assert np.all(np.isfinite(f64(got))), f"{name}: non-finite values"
    assert max_abs <= tol, f"{name}: max-abs {max_abs:.3e} > {tol:.1e}"
    return max_abs, rel_l2
