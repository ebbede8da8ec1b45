"""Reporting helpers for a realised routing histogram (no part of the layer's arithmetic)."""

from __future__ import annotations

import math
from typing import Dict

import numpy as np


def histogram_stats(counts) -> Dict[str, float]:
    """Max/mean count, empty and active experts, and effective experts.

    Effective experts is read as the perplexity exp(H) of the normalised
    histogram: the compact skew summary named by Decoding the Skew (abstract),
    which gives no formula for it.  Reported only; never part of a parity check.
    """
    counts = np.asarray(counts, dtype=np.float64)
    tot = counts.sum()
    nz = counts[counts > 0] / tot if tot > 0 else np.zeros(0)
    H = float(-(nz * np.log(nz)).sum()) if nz.size else 0.0
    return {
        "max_count": float(counts.max()) if counts.size else 0.0,
        "mean_count": float(counts.mean()) if counts.size else 0.0,
        "empty_experts": int((counts == 0).sum()),
        "active_experts": int((counts > 0).sum()),
        "effective_experts": math.exp(H),
    }
