"""Row-split runs of the oracle on every host core (test infrastructure: the benchmark's CPU
baseline).  A spawn pool's workers each hold the workload once and run the unchanged oracle,
oracle.gemv_f64, on a disjoint range of output rows of every call; the split happens outside the
oracle, which stays single-threaded and plain."""
from __future__ import annotations

import numpy as np

_WL = None


def init(layers, xs):
    """Pool initializer: keep the layers and the fp64 activations of every call."""
    global _WL
    _WL = (layers, xs)
    from . import oracle
    oracle.build()


def run(task):
    """One (call, row range): y rows lo..hi of call k.  Returns the number of rows done."""
    from . import oracle
    k, li, lo, hi = task
    layers, xs = _WL
    oracle.gemv_f64(layers[li], xs[k], rows=np.arange(lo, hi, dtype=np.int32))
    return hi - lo
