"""Low-resolution draft attention map (oracle).

DraftAttention2 abstract; reading note, Method overview bullet 1 and Figure 2
caption: the average-pooled and the max-pooled queries and keys each give a
region-level attention map, and the two maps are mixed with weight lambda;
lambda = 0 leaves the average-pooled map alone, which is the v1 guidance
(DraftAttention abstract: a down-sampled attention map).

Readings adopted: the logits use attention's own scale 1/sqrt(d); each map is a
row-wise softmax over all key regions of the same head; the mixture is convex,
D = (1 - lambda) * softmax(avgQ avgK^T / sqrt d) + lambda * softmax(maxQ maxK^T / sqrt d).
The map is computed in fp64 and handed to the ranking as fp32.
"""

from __future__ import annotations

import numpy as np


def row_softmax(x):
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=1, keepdims=True)


def draft_map(q_avg, k_avg, q_max, k_max, lam, d):
    """fp64 D [nb, nb] for one (batch, head); lam is taken at fp32 precision."""
    lam = float(np.float32(lam))
    a = (q_avg @ k_avg.T) / np.sqrt(d)
    b = (q_max @ k_max.T) / np.sqrt(d)
    return (1.0 - lam) * row_softmax(a) + lam * row_softmax(b)


def draft_scores(q_avg, k_avg, q_max, k_max, lam, d):
    """The fp32 scores the ranking sees."""
    return draft_map(q_avg, k_avg, q_max, k_max, lam, d).astype(np.float32)
