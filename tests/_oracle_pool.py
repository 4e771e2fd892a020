"""The oracle's Y rows computed in spawned worker processes, for parity checks of
every row of a large layer (test infrastructure; the arithmetic is the oracle's,
row by row, unchanged)."""
import multiprocessing as mp

import numpy as np


def _rows_job(args):
    import oracle
    qX, s, st, qW, sw, G, rows = args
    return oracle.linear_rows(qX, s, st, qW, sw, G, rows=rows)


def linear_rows_all(qX, s, st, qW, sw, G, workers=None):
    """(Y, bound) of oracle.linear_rows over every row of qX."""
    M = qX.shape[0]
    workers = workers or max(1, min(mp.cpu_count(), 32))
    chunks = [c for c in np.array_split(np.arange(M), 2 * workers) if len(c)]
    with mp.get_context("spawn").Pool(workers) as pool:
        parts = pool.map(_rows_job, [(qX, s, st, qW, sw, G, [int(r) for r in c]) for c in chunks])
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])
