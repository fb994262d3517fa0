"""Grouping of routed (token, slot) pairs by expert.

The pages run the experts as separate GEMMs ("DeepSeek-V4-Flash-SI",
解码瓶颈: the MoE GEMM over 43 layers x 6 experts); they do not describe the
grouping.  Reading taken:
  * a pair p = t*k + j (token t, slot j) goes to expert idx[t, j];
  * rows of one expert are stored contiguously in ascending pair id;
  * the shared expert (always active, one per layer) is group E and holds one
    row per token, in token order, after all routed rows;
  * counts[g] rows per group, offsets = exclusive prefix sum (length G+1);
  * perm[r] is the id of the source of row r: the pair id p < P for routed rows,
    P + t for the shared row of token t; inv[p] is the row of pair p.
"""
from __future__ import annotations

import numpy as np


def permute(idx: np.ndarray, E: int, has_shared: int = 1):
    """Step a3 (index part): idx int32 [T, k] -> counts, offsets, perm, inv, src_token."""
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    P = T * k
    flat = idx.reshape(-1)
    assert ((flat >= 0) & (flat < E)).all()
    counts = np.zeros(E + 1, np.int64)
    counts[:E] = np.bincount(flat, minlength=E)
    counts[E] = T if has_shared else 0
    offsets = np.zeros(E + 2, np.int64)
    offsets[1:] = np.cumsum(counts)
    routed = np.argsort(flat, kind="stable")             # pair ids grouped by expert
    perm = np.concatenate([routed, P + np.arange(T if has_shared else 0)])
    inv = np.empty(P, np.int64)
    inv[routed] = np.arange(P)
    src = np.where(perm < P, perm // max(k, 1), perm - P)
    return (counts.astype(np.int32), offsets.astype(np.int32), perm.astype(np.int32),
            inv.astype(np.int32), src.astype(np.int64))


def gather_rows(xq: np.ndarray, sx: np.ndarray, src_token: np.ndarray):
    """Step a3 (data part): FP8 rows and their scales in permuted order."""
    return xq[src_token], sx[src_token]
