"""Vector search on a TurboQuant-packed database (oracle side; test
infrastructure).

The pages evaluate TurboQuant as a nearest-neighbour index: database vectors
are quantized online, queries stay in full precision, and the search ranks
the database by the estimated inner product ("内存厂商的噩梦来了", section
6.4, the vector-search evaluation and its near-zero index-build time).  The
estimate is the asymmetric one of the attention scores,

    est_j = n_j ( <q', c[idx_j]> + [prod] ||r_j|| sqrt(pi/2)/d <S q', sign_j> ),

q' the rotated query (oracle.attention).  Reading taken here (the pages give
no interface): for each query, the k records with the largest estimate,
ordered by estimate, highest first, ties by record index, lowest first.
"""

import numpy as np

from . import attention as _att


def scores(qz, queries: np.ndarray, db: dict, dtype=np.float64) -> np.ndarray:
    """est_j for every (query, record): [n_q, N].  ``db`` holds the packed
    arrays of N records (codes [N, nb], norms [N], qjl, rnorms)."""
    q = np.asarray(queries, dtype)
    return np.stack([_att._scores_one(qz, q[i], db, dtype=dtype) for i in range(q.shape[0])])


def topk(est: np.ndarray, k: int):
    """(values, indices) of the k largest entries of each row, highest first,
    ties by index, lowest first."""
    n_q, N = est.shape
    k = min(k, N)
    idx = np.empty((n_q, k), np.int64)
    for i in range(n_q):
        order = np.lexsort((np.arange(N), -est[i]))
        idx[i] = order[:k]
    return np.take_along_axis(est, idx, axis=1), idx


def search_topk(qz, queries: np.ndarray, db: dict, k: int):
    """The k best records per query by estimated inner product."""
    return topk(scores(qz, queries, db), k)
