"""Shared test helpers: the relative-error metric and oracle/device glue."""
import numpy as np

TOL = 2e-3   # max relative error for fp outputs and states


def rel_err(got, ref) -> float:
    """max_i |got_i - ref_i| / max(|ref_i|, rms(ref)) over one tensor."""
    got = np.asarray(got, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    if ref.size == 0:
        return 0.0
    rms = np.sqrt(np.mean(ref * ref))
    denom = np.maximum(np.abs(ref), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(got - ref) / denom))


def to_np(t):
    return t.detach().cpu().numpy()
