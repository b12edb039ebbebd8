"""Shared helpers for the GPU parity tests (tolerances, comparisons)."""
import numpy as np
import torch

# Tolerances fixed by the workload spec: fp32 max abs 1e-5 on O and lse;
# bf16 max abs 2e-2 on O and 1e-3 relative on lse (denominator max(|lse_ref|, 1)).
TOL = {
    torch.float32: dict(o_abs=1e-5, lse_abs=1e-5, lse_rel=None),
    torch.bfloat16: dict(o_abs=2e-2, lse_abs=None, lse_rel=1e-3),
}


def errors(out, lse, O_ref, L_ref):
    """Max abs error on O and on lse, and max relative lse error (den max(|ref|, 1))."""
    o = out.detach().float().cpu().numpy().astype(np.float64)
    l = lse.detach().cpu().numpy().astype(np.float64)
    eo = np.abs(o - O_ref)
    el = np.abs(l - L_ref)
    rel = el / np.maximum(np.abs(L_ref), 1.0)
    return float(np.nanmax(eo)) if eo.size else 0.0, float(np.nanmax(el)) if el.size else 0.0, \
        float(np.nanmax(rel)) if rel.size else 0.0, bool(np.isfinite(o).all() and np.isfinite(l).all())


def assert_parity(out, lse, O_ref, L_ref, dtype, what=""):
    eo, el, rel, finite = errors(out, lse, O_ref, L_ref)
    t = TOL[dtype]
    msg = f"{what}: max|dO|={eo:.3e} max|dlse|={el:.3e} rel(lse)={rel:.3e}"
    assert finite, "non-finite output " + msg
    assert eo <= t["o_abs"], msg
    if t["lse_abs"] is not None:
        assert el <= t["lse_abs"], msg
    if t["lse_rel"] is not None:
        assert rel <= t["lse_rel"], msg
    return eo, el, rel


def gather_rows(out, lse, rows):
    """Pick (b, h, t) rows from device outputs -> host tensors [n, D], [n]."""
    idx_b = torch.tensor([r[0] for r in rows], device=out.device)
    idx_h = torch.tensor([r[1] for r in rows], device=out.device)
    idx_t = torch.tensor([r[2] for r in rows], device=out.device)
    return out[idx_b, idx_h, idx_t], lse[idx_b, idx_h, idx_t]
