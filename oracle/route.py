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
