"""Decode attention straight from the quantized cache (oracle).

R, *Problem*: attention reads the KV cache only through query-key inner products, so
the estimator's error is what reaches the softmax.  R, *Comparison*: TurboQuant also
quantizes the tokens generated during decoding.  LK, X thread 8/16: decode attention
is memory-bandwidth bound.  The step computed here is textbook softmax attention
with the keys' inner products replaced by the quantizer's estimates and the values
replaced by their dequantized reconstructions:

    logit_i = scale * est(q, k_i),  p = exp(logit - max) / sum,  o = sum_i p_i v_hat_i

Readings: scale = 1/sqrt(d); no mask, no sinks (one query token); query head h_q
reads KV head h_q // (Hq / Hkv) (grouped-query attention); the step attends over
seq_lens[b] tokens, the newest one included.
"""
from __future__ import annotations

import numpy as np

__all__ = ["softmax_attend", "decode_attention", "exact_attention"]


def softmax_attend(logits: np.ndarray, vhat: np.ndarray) -> np.ndarray:
    """o[g] = softmax(logits[g]) @ vhat for logits [G, N], vhat [N, d]."""
    logits = np.asarray(logits, dtype=np.float64)
    m = np.max(logits, axis=1, keepdims=True)
    p = np.exp(logits - m)
    p /= np.sum(p, axis=1, keepdims=True)
    return p @ np.asarray(vhat, dtype=np.float64)


def decode_attention(q, seq_lens, Hkv: int, key_scores, value_rows, scale: float):
    """Decode attention for q [B, Hq, d].

    ``key_scores(b, h, qs)`` returns est(q, k_i) of the queries qs [G, d] against the
    first seq_lens[b] keys of KV head h as [G, N]; ``value_rows(b, h, n)`` returns the
    dequantized values [n, d].  Output [B, Hq, d] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    for b in range(B):
        n = int(seq_lens[b])
        for h in range(Hkv):
            qs = q[b, h * G:(h + 1) * G]
            logits = scale * key_scores(b, h, qs)[:, :n]
            out[b, h * G:(h + 1) * G] = softmax_attend(logits, value_rows(b, h, n))
    return out


def exact_attention(q, K, V, seq_lens, scale: float):
    """Unquantized reference: K, V [B, Hkv, N, d] float64."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    return decode_attention(q, seq_lens, Hkv,
                            lambda b, h, qs: qs @ np.asarray(K[b, h], dtype=np.float64).T,
                            lambda b, h, n: np.asarray(V[b, h, :n], dtype=np.float64), scale)
