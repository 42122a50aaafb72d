"""Oracle for full-catalog retrieval scoring with top-K selection (test
infrastructure only: the GPU path never imports this module).

Sources:
* The GenRec explainer on techistory.net (scratchpad page 13), the equation
  s = E^T h and its "GenRec方式" toy code: the user representation h is the
  encoder's hidden state at the sequence's last position, and all M catalog
  items are scored at once by one matrix product (no autoregressive loop).
* 'NetflixのGenRec解説――LLMを生成させず推薦rankerとして使う', section
  '全体像：LLMは入力を読み、ranking headが作品を採点する': scores over the
  catalog, sorted in descending order, give the ranking.
* 'HSTUとGenerative Recommenders', section 'DLRMから行動sequenceへ何を変えたのか'
  (ranking and retrieval as one sequential transduction): retrieval predicts
  the next content and may use maximum-inner-product search.

Read as: for user u with vector h_u (row offsets[u+1]-1 of the encoder output;
a user without tokens has h_u = 0), score item m as <E_m, h_u> exactly (the
oracle sums the bf16-rounded inputs in float64), and return the K highest
scores in descending order, equal scores ordered by ascending item id.

Plain numpy.  The GPU computes the scores in fp32 (tensor-core accumulation),
so on inputs whose sums are not exact in fp32 the tests compare validity within
a derived bound rather than exact order; integer-valued inputs make every sum
exact on both sides and the ids are compared exactly.
"""
from __future__ import annotations

import numpy as np


def user_vectors(Y, offsets) -> np.ndarray:
    """h_u = Y[offsets[u+1] - 1] (float64), or 0 for an empty user."""
    Y = np.asarray(Y, np.float64)
    offsets = np.asarray(offsets, np.int64)
    U = len(offsets) - 1
    H = np.zeros((U, Y.shape[1]), np.float64)
    for u in range(U):
        if offsets[u + 1] > offsets[u]:
            H[u] = Y[offsets[u + 1] - 1]
    return H


def scores(E, H) -> np.ndarray:
    """s[u, m] = <E_m, h_u> in float64, [U, M]."""
    return np.asarray(H, np.float64) @ np.asarray(E, np.float64).T


def topk(S, K: int):
    """Per row of S: the K largest entries in descending order, ties by
    ascending column index.  Returns (values [U, K] float64, ids [U, K] int64)."""
    S = np.asarray(S, np.float64)
    U, M = S.shape
    if not 1 <= K <= M:
        raise ValueError("need 1 <= K <= M")
    vals = np.empty((U, K), np.float64)
    ids = np.empty((U, K), np.int64)
    cols = np.arange(M)
    for u in range(U):
        order = np.lexsort((cols, -S[u]))[:K]   # primary: -score, secondary: id
        ids[u] = order
        vals[u] = S[u, order]
    return vals, ids


def retrieve(E, H, K: int):
    """Top-K items of every user: (values, ids)."""
    return topk(scores(E, H), K)
