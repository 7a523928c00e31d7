"""Parity gates for bf16-output attention against the fp64 oracle.

Two gates, both applied by every parity test:

* the stated bar: max |g - r| <= 2e-2 and max |g - r| / max |r| <= 2e-2
  (relative error taken normwise, because elementwise relative error is
  undefined where the reference output is near zero);
* a tight gate derived from the kernels' arithmetic.  Decode keeps the
  softmax weights and both products in fp32 and rounds only the output to
  bf16 (relative error <= 2^-8, bf16's unit roundoff, when rounding to
  nearest), so |g - r| <= 2^-8 |r| + 2^-10 max|r|.  Prefill also rounds the
  weights p to bf16 before the P.V product (relative error <= 2^-8 on each
  weight, which moves a weighted mean of the value rows by at most
  2^-8 max|v| if every rounding went the same way); its floor is set at half
  that, 2^-9 max|v|: the roundings of different keys are independent and
  largely cancel, and the kernels stay inside this tighter gate.

The tight decode floor is below the effect of dropping or adding one cached
token at the lengths tested, which ``test_oracle_pins`` checks on the oracle.
"""
from __future__ import annotations

import numpy as np

BAR_ABS = 2e-2
BAR_REL = 2e-2


def compare(got, ref, *, floor: float | None = None, kind: str = "decode", vmax: float | None = None):
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    err = np.abs(g - r)
    rmax = float(np.max(np.abs(r))) if r.size else 0.0
    if floor is None:
        if kind == "decode":
            floor = 2.0 ** -10 * rmax
        else:
            assert vmax is not None
            floor = 2.0 ** -9 * vmax
    bound = 2.0 ** -8 * np.abs(r) + floor
    stats = {
        "max_abs": float(err.max()) if err.size else 0.0,
        "rel_normwise": float(err.max() / rmax) if rmax > 0 else float(err.max() if err.size else 0.0),
        "rms": float(np.sqrt(np.mean(err ** 2))) if err.size else 0.0,
        "ref_max": rmax,
        "nan": int(np.isnan(g).sum()),
        "tight_violations": int(np.sum(~(err <= bound))),
    }
    return stats


def assert_close(got, ref, *, abs_bar: bool = True, **kw):
    """All gates.  abs_bar=False drops only the 2e-2 absolute bar, for stress cases whose outputs
    reach magnitudes (|out| >= 4) where rounding the output to bf16 alone can be off by 2^-6;
    the normwise relative bar and the tight gate still apply there."""
    s = compare(got, ref, **kw)
    assert s["nan"] == 0, s
    if abs_bar:
        assert s["max_abs"] <= BAR_ABS, s
    assert s["rel_normwise"] <= BAR_REL, s
    assert s["tight_violations"] == 0, s
    return s
