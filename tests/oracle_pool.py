"""A spawn-started process pool for oracle work that is too slow in one process (test
infrastructure: it only calls the oracle).

The long-context cascade (16384 tokens, up to 32 heads of d_h = 128) needs the oracle's column
sums of every kept head at every layer to compare the device's token importance element by
element.  Each task is one (layer, head): the head's query, key and value rows of the layer go in,
its probability column sums, sum |O| and refetch-flag agreement come out.  Workers are started with
the spawn method (never forked from a process that has used CUDA) and run single-threaded BLAS.
"""
from __future__ import annotations

import multiprocessing as mp

import numpy as np


def _init_worker():
    from threadpoolctl import threadpool_limits
    threadpool_limits(1)


def head_layer_task(args):
    """Oracle progressive attention of one head over all of its query rows, in row blocks.

    args = (q [n, d] float32, k [n, d] float32 (key gain applied), v [n, d] float32, theta,
    sm_scale, dev_flags [n] bool).  Where the device's refetch decision differs from the oracle's
    the row must be a near-tie (|max p - theta| <= 1e-5 theta); such rows are recomputed with the
    device's decision so the comparison stays like for like.
    Returns (column sums [n], sum |O|, near-tie flag count, off-tie flag count)."""
    from oracle import spatten_ref as R

    q, k32, v32, theta, sm, dev_flags = args
    kq, vq = R.quantize_head(k32), R.quantize_head(v32)
    q = np.asarray(q, np.float64)
    n = q.shape[0]
    col = np.zeros(n)
    habs = 0.0
    near = off = 0
    for r0 in range(0, n, 512):
        rows = slice(r0, min(n, r0 + 512))
        r = R.progressive_attention(q[rows], kq, vq, theta, sm)
        diff = dev_flags[rows] != r["flags"]
        if diff.any():
            off += int(np.count_nonzero(np.abs(r["pmax_msb"][diff] - theta) > 1e-5 * theta))
            near += int(diff.sum())
            r = R.progressive_attention(q[rows], kq, vq, theta, sm, flags_override=dev_flags[rows])
        col += R.token_importance_increment(r["P"])
        habs += R.head_importance_increment(r["O"])
    return col, habs, near, off


def spawn_pool(workers: int):
    return mp.get_context("spawn").Pool(workers, initializer=_init_worker)
