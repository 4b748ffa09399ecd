"""fp64 oracle for the allocation diagnostics of Sketch Attention.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: SequenceO1 (arXiv 2609.08443).
* §5.1 and Fig. 3: for every token of a sampled history, the largest weight the token receives in A
  (its "maximum normalized weight"), and the histogram of those maxima, recorded as a descriptive
  diagnostic of the two normalisations.
* §2.4: Slot Attention's normalisation is the closest in spirit to SA's prototype-wise softmax. Slot
  Attention (Locatello et al., 2020) turns its weights into a weighted mean of the inputs. The
  renormalised sketch below is that weighted mean, each prototype's sum A V divided by the mass
  sum_i A_{j,i} it received.

Readings taken here: the diagnostic is built for the prototype-wise normalisation (Eq. (8)), where
the maximum is over the k prototypes of each token. Padding tokens carry -1, and the histogram skips
negative values. The histogram has `bins` equal bins over [0, 1], with 1.0 in the last. A prototype
with zero mass gets a zero renormalised row.
"""
from __future__ import annotations

import numpy as np

from .sa import NORM_PROTO, _q_for, _segments, sa_problem


def token_max_weight(q, k, v, cu_seqlens, seqused=None, scale=1.0):
    """max_j A_{j,i} for every history row i and head (PROTO, Eq. (8)); -1 on padding rows.
    Returns [T, H]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, H = k.shape[0], k.shape[1]
    out = np.full((T, H), -1.0)
    for b, (lo, n) in enumerate(_segments(cu_seqlens, seqused)):
        for h in range(H):
            if n == 0:
                continue
            _, _, _, A = sa_problem(_q_for(q, b, h), k[lo:lo + n, h], v[lo:lo + n, h], scale, NORM_PROTO)
            out[lo:lo + n, h] = A.max(axis=0)
    return out


def weight_histogram(values, bins):
    """Counts of the non-negative values in `bins` equal bins over [0, 1] (1.0 in the last)."""
    vals = np.asarray(values, dtype=np.float64).reshape(-1)
    vals = vals[vals >= 0]
    counts = np.zeros(bins, dtype=np.int64)
    for x in vals:
        counts[min(int(x * bins), bins - 1)] += 1
    return counts


def renormalized_sketch(sketch, mass):
    """sketch_j / mass_j per (user, head, prototype): the weighted mean of the values the prototype
    aggregated; zero rows where the mass is zero."""
    sketch = np.asarray(sketch, dtype=np.float64)
    mass = np.asarray(mass, dtype=np.float64)
    out = np.zeros_like(sketch)
    nz = mass > 0
    out[nz] = sketch[nz] / mass[nz][..., None]
    return out
