"""Equal-size spherical k-means (the FlashHead index builder) in float64 — TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this module; the
product path never does, and it imports nothing from the product package.

Sources (FlashHead pages, "Module 1: equal-size spherical K-Means", Eq.4 and Eq.5, and the
implementation details under "Experimental setup"):
  * the embedding matrix E (v x d) is clustered offline into c clusters of exactly b = v / c tokens
    each, so that the cluster-to-token map is a dense c x b tensor;
  * Eq.4: minimise the sum over tokens of the negative cosine similarity between a token's embedding
    and its cluster's (L2-normalised) centre;
  * Eq.5: a centre is the L2-normalised mean of its members' embeddings;
  * the clustering is spherical k-means after Dhillon & Modha (2001), run for up to 1000 iterations.

Readings where the pages are silent (each also listed with the other readings of the pages):
  * Following Dhillon & Modha, rows are projected onto the unit sphere first (x_i = e_i / |e_i|),
    so the cosine of Eq.4 is x_i . c_k and Eq.5 averages the unit rows.  With this reading both
    half-steps below are exact optimisers and the objective can never rise.
  * The equal-size constraint enters the assignment half-step: for fixed centres, the labels are
    the exact optimum of  max sum_i x_i . c_{k(i)}  subject to |{i : k(i) = k}| = b  for every k
    (a transportation problem).  It is solved here as a linear assignment of the v tokens to c*b
    slots, slot j belonging to cluster j // b, with scipy's linear_sum_assignment as the library
    step.  Which of several equally good labelings comes back is not part of the definition; only
    the objective value is unique.
  * Initial centres: the unit rows of c distinct tokens, chosen by a caller-supplied order (the
    seeded generator draws it; the pages do not say how the clustering starts).
  * Iteration stops at a fixed point of the labels or after `iters` rounds.
"""

from __future__ import annotations

import itertools

import numpy as np
from scipy.optimize import linear_sum_assignment


def stored_to_f64(a: np.ndarray) -> np.ndarray:
    """Stored values to float64, exactly: float32 as is, BF16 given as uint16 bit patterns."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if a.dtype in (np.float32, np.float64):
        return a.astype(np.float64)
    raise TypeError(f"unsupported storage dtype {a.dtype}")


def unit_rows(E: np.ndarray) -> np.ndarray:
    """x_i = e_i / |e_i|_2 (spherical k-means works on directions).  Zero rows are rejected."""
    X = stored_to_f64(E)
    n = np.sqrt((X * X).sum(axis=1))
    if np.any(n == 0.0):
        raise ValueError("zero embedding row: its direction is undefined")
    return X / n[:, None]


def objective(X: np.ndarray, C: np.ndarray, labels: np.ndarray) -> float:
    """Eq.4: the sum over tokens of the negative cosine similarity to the token's centre."""
    return -float(np.einsum("ij,ij->", X, C[labels]))


def update_centres(X: np.ndarray, labels: np.ndarray, c: int) -> np.ndarray:
    """Eq.5: each centre is the L2-normalised mean (equivalently, sum) of its members' rows.
    A cluster whose members sum to zero keeps no direction; that is an error here."""
    S = np.zeros((c, X.shape[1]), dtype=np.float64)
    np.add.at(S, labels, X)
    n = np.sqrt((S * S).sum(axis=1))
    if np.any(n == 0.0):
        raise ValueError("a cluster's members sum to zero")
    return S / n[:, None]


def similarities(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """A[i, k] = x_i . c_k (the cosine of Eq.4, as both sides are unit vectors)."""
    return X @ C.T


def assign_equal_size(X: np.ndarray, C: np.ndarray, b: int) -> np.ndarray:
    """Exact equal-size assignment for fixed centres: labels maximising sum_i A[i, k(i)] with exactly
    b tokens per cluster, as a linear assignment of tokens to c*b slots (slot j -> cluster j // b)."""
    v, c = X.shape[0], C.shape[0]
    if v != c * b:
        raise ValueError("v must equal c * b")
    A = similarities(X, C)
    rows, slots = linear_sum_assignment(np.repeat(A, b, axis=1), maximize=True)
    labels = np.empty(v, dtype=np.int64)
    labels[rows] = slots // b
    return labels


def assignment_value(A: np.ndarray, labels: np.ndarray) -> float:
    """sum_i A[i, labels[i]] (the negated objective of Eq.4 for these labels)."""
    return float(A[np.arange(A.shape[0]), labels].sum())


def is_equal_size(labels: np.ndarray, c: int, b: int) -> bool:
    """Every token has one cluster in [0, c) and every cluster exactly b tokens."""
    labels = np.asarray(labels)
    if labels.min(initial=0) < 0 or labels.max(initial=0) >= c:
        return False
    return bool(np.all(np.bincount(labels, minlength=c) == b))


def c2t_from_labels(labels: np.ndarray, c: int, b: int) -> np.ndarray:
    """The dense cluster-to-token map: row k lists cluster k's tokens in ascending id order."""
    if not is_equal_size(labels, c, b):
        raise ValueError("labels are not an equal-size partition")
    order = np.lexsort((np.arange(labels.size), labels))
    return order.reshape(c, b).astype(np.int32)


def brute_force_assignment(A: np.ndarray, b: int) -> float:
    """The best equal-size assignment value by enumerating every partition (tiny inputs only)."""
    v, c = A.shape
    best = -np.inf
    base = np.repeat(np.arange(c), b)
    for perm in set(itertools.permutations(base.tolist())):
        best = max(best, float(A[np.arange(v), list(perm)].sum()))
    return best


def kmeans(E: np.ndarray, c: int, init_tokens: np.ndarray, iters: int):
    """Equal-size spherical k-means: alternate the exact equal-size assignment and Eq.5.

    Returns (labels, C, history), history[t] = Eq.4 objective after iteration t's update.
    """
    X = unit_rows(E)
    v = X.shape[0]
    if v % c:
        raise ValueError("v must be a multiple of c")
    b = v // c
    init_tokens = np.asarray(init_tokens)
    if init_tokens.shape != (c,) or np.unique(init_tokens).size != c:
        raise ValueError("init_tokens must name c distinct tokens")
    C = X[init_tokens].copy()
    labels = None
    history = []
    for _ in range(iters):
        new = assign_equal_size(X, C, b)
        if labels is not None and np.array_equal(new, labels):
            break
        labels = new
        C = update_centres(X, labels, c)
        history.append(objective(X, C, labels))
    return labels, C, history


def eps_cs_gap(A: np.ndarray, labels: np.ndarray, prices: np.ndarray) -> float:
    """Largest violation of complementary slackness for a labeling and cluster prices:
    max_i [ max_k (A[i,k] - prices[k]) - (A[i,labels[i]] - prices[labels[i]]) ].
    A labeling that is equal-size and has gap <= eps is within v * eps of the optimum (weak
    duality of the transportation problem), which is how an auction result is checked."""
    net = A - prices[None, :]
    own = net[np.arange(A.shape[0]), labels]
    return float((net.max(axis=1) - own).max())


def dual_bound(A: np.ndarray, prices: np.ndarray, b: int) -> float:
    """Weak-duality upper bound on any equal-size assignment value: sum_i max_k (A[i,k] - p_k)
    + b * sum_k p_k."""
    return float((A - prices[None, :]).max(axis=1).sum() + b * prices.sum())
