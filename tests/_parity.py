"""Helpers shared by the GPU parity tests: seeded inputs, band-aware code comparison.

Tolerances (applied in the tests):
  * codes and sign bits: bit-exact, except a coordinate whose oracle rotated value lies
    within 1e-5 (unit scale) of a decision boundary, or a sign whose projection
    |(S r)_i| <= 1e-5 ||S_i|| (and any sign of a record that already had an exempt code);
  * norms: 1e-5 relative (the tensor-core path takes ||Pi x|| in fp32);
  * scores: |s - s_ref| <= 1e-3 ||q|| ||x||;
  * attention: per (batch, head) row, max_j |o_j - o_ref_j| <= 1e-3 max_j |o_ref_j|.
"""
from __future__ import annotations

import numpy as np

BAND = 1e-5


def as_u32(t) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint32)


def code_mismatches(gpu_words, ref_words, d, bits, y_ref, boundaries, skip_rows=()):
    """Return (#mismatched coordinates outside the band, #exempt, rows with exemptions).

    A mismatch is exempt only when the two codes are neighbours and the oracle's rotated
    value lies within BAND of the boundary between them.  Rows in ``skip_rows`` (zero
    vectors, whose every coordinate sits on the middle boundary) are not compared here.
    """
    from oracle.quantizer import unpack_codes
    g = np.asarray(gpu_words, dtype=np.uint32)
    r = np.asarray(ref_words, dtype=np.uint32)
    rows = np.nonzero(np.any(g != r, axis=1))[0]
    bad = exempt = 0
    exempt_rows = set()
    t = np.asarray(boundaries, dtype=np.float64)
    for i in rows:
        if int(i) in skip_rows:
            continue
        cg = unpack_codes(g[i:i + 1], d, bits)[0]
        cr = unpack_codes(r[i:i + 1], d, bits)[0]
        for j in np.nonzero(cg != cr)[0]:
            lo = int(min(cg[j], cr[j]))
            near = abs(int(cg[j]) - int(cr[j])) == 1 and abs(y_ref[i, j] - t[lo]) <= BAND
            if near:
                exempt += 1
                exempt_rows.add(int(i))
            else:
                bad += 1
    return bad, exempt, exempt_rows


def sign_mismatches(gpu_words, ref_words, m, proj_ref, S, skip_rows=()):
    from oracle.quantizer import unpack_signs
    g = np.asarray(gpu_words, dtype=np.uint32)
    r = np.asarray(ref_words, dtype=np.uint32)
    rownorm = np.linalg.norm(np.asarray(S, dtype=np.float64), axis=1)
    bad = exempt = 0
    for i in np.nonzero(np.any(g != r, axis=1))[0]:
        if int(i) in skip_rows:
            exempt += 1
            continue
        sg = unpack_signs(g[i:i + 1], m)[0]
        sr = unpack_signs(r[i:i + 1], m)[0]
        for k in np.nonzero(sg != sr)[0]:
            if abs(proj_ref[i, k]) <= BAND * rownorm[k]:
                exempt += 1
            else:
                bad += 1
    return bad, exempt


def rel_rows(o, o_ref):
    """Per-row max |o - o_ref| / max |o_ref| (rows = all leading axes)."""
    o = np.asarray(o, dtype=np.float64).reshape(-1, o.shape[-1])
    r = np.asarray(o_ref, dtype=np.float64).reshape(-1, o_ref.shape[-1])
    return np.max(np.abs(o - r), axis=1) / np.maximum(np.max(np.abs(r), axis=1), 1e-30)
