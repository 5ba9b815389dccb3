"""Oracle work for full-size attention checks, run in a process pool.

The pool is started with the `spawn` method, so its workers import only this
module and the oracle (no CUDA context is inherited).  Holds none of the
method's arithmetic: it calls the oracle's row/column-restricted forms."""
import numpy as np


def head_lse_and_token_scores(args):
    """(Q, K, idx_d) of one (batch, q-head) -> (lse of every row, t of every column)."""
    Q, K, idx_d = args
    from oracle import attention as OA
    S = Q.shape[0]
    L = OA.lse_rows(Q, K, idx_d, np.arange(S))
    return L, OA.token_scores(Q, K, idx_d, L, np.arange(S))


def spawn_pool(n):
    import multiprocessing as mp
    return mp.get_context("spawn").Pool(n)
