"""Error statistics of a computed result against the oracle's -- TEST
INFRASTRUCTURE ONLY (used by ``tests/`` and by the parity sample that
``bench.py`` reports beside its timing).

The parity rule is max |got - want| / max |want| over the whole output; the
other statistics (mean, rms, percentiles of the per-element error, all
divided by the same max |want|) are reported, not gated.
"""
from __future__ import annotations

import numpy as np


class ErrorStats:
    """Running statistics of |got - want| over blocks of one output:
    the max error, max |want| (the normalisation), the sum of |error| and
    of error^2, and a histogram of |error| in bins of 2^(1/8) (exact
    percentiles to within a bin, independent of the normalisation)."""

    BINS_PER_OCTAVE = 8
    LOW = -160  # 2^-160: everything below (exact zeros included) goes there

    def __init__(self):
        self.max_err = 0.0
        self.scale = 0.0
        self.count = 0
        self.sum_abs = 0.0
        self.sum_sq = 0.0
        self.hist = np.zeros(8 * 200, dtype=np.int64)

    def add(self, got, want):
        got = np.asarray(got, dtype=np.float64)
        want = np.asarray(want, dtype=np.float64)
        e = np.abs(got - want).ravel()
        if e.size == 0:
            return
        if not np.all(np.isfinite(got)):
            self.max_err = float("inf")
        self.max_err = max(self.max_err, float(e.max()))
        self.scale = max(self.scale, float(np.abs(want).max()))
        self.count += e.size
        self.sum_abs += float(e.sum())
        self.sum_sq += float(np.dot(e, e))
        with np.errstate(divide="ignore"):
            k = np.floor(np.log2(np.maximum(e, 2.0 ** self.LOW)) * self.BINS_PER_OCTAVE)
        k = np.clip(k - self.LOW * self.BINS_PER_OCTAVE, 0, self.hist.size - 1).astype(np.int64)
        self.hist += np.bincount(k, minlength=self.hist.size)

    def percentile_abs(self, q):
        """Upper edge of the bin holding the q-quantile of |error|."""
        if self.count == 0:
            return 0.0
        c = np.cumsum(self.hist)
        i = int(np.searchsorted(c, q * self.count))
        return 2.0 ** ((i + 1) / self.BINS_PER_OCTAVE + self.LOW)

    @property
    def norm_err(self) -> float:
        return self.max_err / self.scale if self.scale > 0 else self.max_err

    def summary(self) -> dict:
        s = self.scale if self.scale > 0 else 1.0
        return {"max_norm_err": self.norm_err,
                "mean_norm_err": self.sum_abs / max(1, self.count) / s,
                "rms_norm_err": (self.sum_sq / max(1, self.count)) ** 0.5 / s,
                "p99_norm_err": self.percentile_abs(0.99) / s,
                "p999_norm_err": self.percentile_abs(0.999) / s,
                "elements": self.count, "max_abs_ref": self.scale}
