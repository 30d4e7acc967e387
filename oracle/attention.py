"""Decode attention over the dequantised paged cache, partial states and their merge.

ORACLE -- test infrastructure only (see ``oracle/formats.py`` for the rule on who may use it).

What the method computes (brainszone.ai "Minima-KV ..." summary, pt section "Como os
resultados parciais são combinados"; fr section "Comment les résultats partiels sont
assemblés"): per-format kernels produce partial attention states that a globally
normalised online-softmax merge combines, so that the result equals attention over all
pages.  The exact result therefore has a plain definition, written out here in float64:

  for query i of q_len (the new tokens are the last q_len positions of the context),
  query head hq, KV head h = hq // (Hq // Hkv):
     visible tokens t <= L - q_len + i
     s_t = sm_scale * sum_d q[i, hq, d] * K[t, h, d]
     o   = sum_t softmax(s)_t V[t, h, :]

K and V are the dequantised cache values (FP8: code value * page scale; TQ3:
(q - 3.5) * group scale); q is the bf16 query value.  Positional encoding is not part of this
step (keys are stored already rotated).  The default sm_scale is 1/sqrt(D).
"""
from __future__ import annotations

import numpy as np


def attention(K, V, q, sm_scale, q_len=None):
    """Single-pass attention in float64.

    K, V: [L, Hkv, D] dequantised cache of one sequence; q: [q_len, Hq, D].
    Returns o: [q_len, Hq, D].
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    L, Hkv, D = K.shape
    q_len = q.shape[0] if q_len is None else q_len
    Hq = q.shape[1]
    g = Hq // Hkv
    if L == 0:
        raise ValueError("attention over an empty context is undefined")
    o = np.empty((q_len, Hq, D))
    for i in range(q_len):
        last = L - q_len + i                  # inclusive
        for h in range(Hkv):
            Kh = K[:last + 1, h, :]
            Vh = V[:last + 1, h, :]
            qs = q[i, h * g:(h + 1) * g, :]            # [g, D]
            s = sm_scale * (qs @ Kh.T)                 # [g, t]
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            o[i, h * g:(h + 1) * g] = (p @ Vh) / p.sum(axis=1, keepdims=True)
    return o


def partial_state(K, V, q, sm_scale, tokens, q_len=None, L=None):
    """(m, l, acc) of one part: the token indices ``tokens`` of the context.

    m = max visible logit, l = sum exp(s - m), acc = sum exp(s - m) V; a part with no visible
    token gives (-inf, 0, 0).  Shapes: m, l [q_len, Hq]; acc [q_len, Hq, D].
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    L = K.shape[0] if L is None else L
    q_len = q.shape[0] if q_len is None else q_len
    Hkv, D = K.shape[1], K.shape[2]
    Hq = q.shape[1]
    g = Hq // Hkv
    tokens = np.asarray(tokens, dtype=np.int64)
    m = np.full((q_len, Hq), -np.inf)
    lsum = np.zeros((q_len, Hq))
    acc = np.zeros((q_len, Hq, D))
    for i in range(q_len):
        vis = tokens[tokens <= L - q_len + i]
        if vis.size == 0:
            continue
        for hq in range(Hq):
            h = hq // g
            s = sm_scale * (K[vis, h, :] @ q[i, hq])
            mm = s.max()
            p = np.exp(s - mm)
            m[i, hq] = mm
            lsum[i, hq] = p.sum()
            acc[i, hq] = p @ V[vis, h, :]
    return m, lsum, acc


def merge(parts):
    """Globally normalised merge: M = max m_k, Lsum = sum l_k e^(m_k - M),
    O = sum acc_k e^(m_k - M) / Lsum.  Parts with m = -inf contribute nothing."""
    ms = np.stack([p[0] for p in parts])
    M = ms.max(axis=0)
    if np.any(np.isneginf(M)):
        raise ValueError("no visible token in any part")
    w = [np.where(np.isneginf(p[0]), 0.0, np.exp(p[0] - M)) for p in parts]
    Lsum = sum(wk * p[1] for wk, p in zip(w, parts))
    O = sum(wk[..., None] * p[2] for wk, p in zip(w, parts))
    return O / Lsum[..., None]


def materialise_and_attend(pool, seq, q, sm_scale):
    """The pages' "materialising profile": expand every page of the sequence into dense
    float64 K and V, then plain softmax(q K^T) V.  Used only to cross-check on small cases."""
    K, V = pool.dequant_seq(seq)
    return attention(K, V, q, sm_scale)
