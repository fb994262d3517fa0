"""Router: sqrtsoftplus scoring, top-k selection, route scale 1.5.

Passage: "DeepSeek-V4-Flash-SI" model card, 架构特性, Mixture of Experts
paragraph: each layer has 256 routed experts plus one shared expert; a gate
picks the top 6 experts per token; layers past the first three score with
sqrtsoftplus; the routing scale is 1.5.

Readings (the pages give only these words):
  * score s = sqrt(softplus(z)) of the gate logit z, softplus(z) = log(1 + e^z);
  * selection is the k largest scores; since sqrt(softplus(.)) is strictly
    increasing this is the k largest logits, ties to the lower expert index;
  * weights are the selected scores normalised to sum to one, times the route
    scale (route_norm = 1); with route_norm = 0 they are the scores times the
    scale.  Whether the scores are normalised is not stated (parity unpinned).
The gate projection producing the logits is outside the expert path.
"""
from __future__ import annotations

import numpy as np


def softplus(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def sqrtsoftplus(z: np.ndarray) -> np.ndarray:
    return np.sqrt(softplus(z))


def route_topk(logits: np.ndarray, k: int, route_scale: float = 1.5, route_norm: int = 1):
    """Step a2: logits float32 [T, E] -> (idx int32 [T, k], w float64 [T, k]).

    idx rows are in selection order (largest logit first)."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    assert 1 <= k <= E
    order = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    s = sqrtsoftplus(np.take_along_axis(logits, idx, axis=1))
    if route_norm:
        w = route_scale * s / s.sum(axis=1, keepdims=True)
    else:
        w = route_scale * s
    return idx, w


def route_hash(token_ids: np.ndarray, tid2eid: np.ndarray, logits: np.ndarray,
               route_scale: float = 1.5, route_norm: int = 1):
    """Hash routing of the first layers ("DeepSeek-V4-Flash-SI" model card,
    架构特性, Mixture of Experts paragraph: the first 3 layers route by hash,
    chosen deterministically from the token ID; the other layers score with
    sqrtsoftplus top-k; routing scale 1.5).

    The page gives no hash function.  Reading: the choice is a table lookup,
    idx[t] = tid2eid[token_ids[t]], in a table of k expert ids per vocabulary
    entry that the checkpoint carries (the table itself is an input, not a
    step of the method); the gate still scores every expert, and the weights
    are the sqrtsoftplus scores of the chosen experts, normalised to sum to
    one (route_norm = 1) and multiplied by the route scale -- the same weight
    rule as the scored layers, applied at the looked-up indices.

    token_ids int [T] in [0, vocab); tid2eid int [vocab, k] with ids in
    [0, E); logits float32 [T, E].  Returns (idx int32 [T, k] in table
    order, w float64 [T, k])."""
    token_ids = np.asarray(token_ids, dtype=np.int64)
    tid2eid = np.asarray(tid2eid, dtype=np.int64)
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    vocab, k = tid2eid.shape
    assert token_ids.shape == (T,) and ((token_ids >= 0) & (token_ids < vocab)).all()
    assert ((tid2eid >= 0) & (tid2eid < E)).all()
    idx = tid2eid[token_ids].astype(np.int32)
    s = sqrtsoftplus(np.take_along_axis(logits, idx.astype(np.int64), axis=1))
    if route_norm:
        w = route_scale * s / s.sum(axis=1, keepdims=True)
    else:
        w = route_scale * s
    return idx, w
