"""Serving-side forms of the attention step over a quantized cache (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

R, *Comparison*: TurboQuant also quantizes the tokens generated during decoding, so a
decode step appends the new token's key and value to the quantized cache and attends
over it.  LK, X thread and Show HN post: prefill over the compressed cache at long
context.  R, closing discussion: the rotation and the codebook lookup belong inside the
attention kernel.  Three forms follow from these, written out plainly:

* append-then-attend: quantize the step's new key/value into slot seq_len of its row,
  then decode attention over seq_len + 1 tokens;
* a paged cache: token t of sequence b lives in physical slot
  block_table[b][t // P] * P + t % P of a record pool (P tokens per page);
* causal prefill over the cache: query i at absolute position pos_i attends to the
  tokens 0..pos_i.

Readings (listed in the design notes): pages are whole blocks of P records of every
record array; a page id indexes the pool, not the sequence; the prefill mask is the
textbook causal mask on absolute positions, with the same scale 1/sqrt(d) and GQA head
mapping as the decode step.
"""
from __future__ import annotations

import numpy as np

from .attention import softmax_attend

__all__ = ["page_slots", "prefill_attention"]


def page_slots(block_table, page_size: int, b: int, n: int) -> np.ndarray:
    """Physical slots of tokens 0..n-1 of sequence b under a block table [B][max_pages]."""
    t = np.arange(n)
    pages = np.asarray(block_table, dtype=np.int64)[b, t // page_size]
    return pages * page_size + t % page_size


def prefill_attention(q, q_pos, Hkv: int, key_scores, value_rows, scale: float):
    """Causal attention for a block of queries q [B, Hq, T, d] at absolute positions
    q_pos [B, T] over the cached tokens 0..max(q_pos[b]) of each sequence.

    ``key_scores(b, h, qs)`` returns est(q, k_j) of the queries qs [R, d] against the
    first n_b = max(q_pos[b]) + 1 keys of KV head h as [R, n_b]; ``value_rows(b, h, n)``
    the reconstructed values [n, d].  Output [B, Hq, T, d] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, T, d = q.shape
    G = Hq // Hkv
    pos = np.asarray(q_pos, dtype=np.int64)
    out = np.zeros((B, Hq, T, d))
    for b in range(B):
        n = int(pos[b].max()) + 1
        for h in range(Hkv):
            qs = q[b, h * G:(h + 1) * G].reshape(G * T, d)
            logits = scale * key_scores(b, h, qs)[:, :n]
            # row g*T + i belongs to query i: it sees tokens 0..pos[b, i]
            visible = np.arange(n)[None, :] <= np.tile(pos[b], G)[:, None]
            logits = np.where(visible, logits, -np.inf)
            o = softmax_attend(logits, value_rows(b, h, n))
            out[b, h * G:(h + 1) * G] = o.reshape(G, T, d)
    return out
