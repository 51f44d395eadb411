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


def _rows_of(words):
    return np.nonzero(np.any(words, axis=1))[0]


def adopt_mse(gpu_words, ref, bits, boundaries, skip_rows=()):
    """Band-check the GPU's MSE-stage codes against the oracle's ``ref`` (a dict from
    ``quantize_mse`` / ``quantize_prod``) and return ``(idx, exempt)``: the oracle's code
    indices with every band-exempt coordinate replaced by the GPU's code.

    The oracle then rescores with the GPU's codes, so a legitimate flip inside the 1e-5
    band cannot move a score or an attention row beyond the stated tolerance.  Any
    mismatch outside the band fails the calling test.
    """
    from oracle.quantizer import unpack_codes
    g = np.asarray(gpu_words, dtype=np.uint32)
    d = ref["y"].shape[1]
    bad, exempt, rows = code_mismatches(g, ref["codes"], d, bits, ref["y"], boundaries, skip_rows)
    assert bad == 0, f"{bad} code mismatches outside the band ({exempt} exempt)"
    idx = np.array(ref["idx"], copy=True)
    rows = sorted(rows)
    if rows:
        idx[rows] = unpack_codes(g[rows], d, bits)
    return idx, exempt


def adopt_prod(gpu_codes, gpu_signs, gpu_rnorms, ref, bits, centroids, boundaries, S):
    """Band-check a GPU TurboQuant-prod record set and return the records the oracle
    rescores with: ``chat`` and ``rnorms`` recomputed by the oracle's arithmetic from the
    adopted codes (r = y - c[idx]), and the GPU's sign bits after every mismatch against
    sign(S r) was found inside the band |(S r)_i| <= 1e-5 ||S_i||."""
    from oracle.quantizer import unpack_signs
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    y = ref["y"]
    if bits > 1:
        idx, _ = adopt_mse(gpu_codes, ref, bits - 1, boundaries)
        chat = np.asarray(centroids, dtype=np.float64)[idx]
    else:
        idx = np.zeros(y.shape, dtype=np.int64)
        chat = np.zeros_like(y)
    r = y - chat
    gamma = np.sqrt(np.sum(r * r, axis=1))
    proj = r @ S.T
    sg = unpack_signs(np.asarray(gpu_signs, dtype=np.uint32), m)
    sr = (proj >= 0).astype(np.int64)
    diff = sg != sr
    rownorm = np.linalg.norm(S, axis=1)
    outside = diff & (np.abs(proj) > BAND * rownorm[None, :])
    assert not np.any(outside), f"{int(outside.sum())} sign mismatches outside the band"
    rn = np.asarray(gpu_rnorms, dtype=np.float64)
    assert np.all(np.abs(rn - gamma) <= 1e-5 * np.maximum(gamma, 1e-6) + 1e-6), "residual norms"
    return {"idx": idx, "chat": chat, "s": sg, "rnorms": gamma}


def adopt_spectral(gpu_codes, gpu_rnorms, ref, desc, x):
    """Band-check a GPU spectral record set coordinate by coordinate and return the records
    the oracle rescores with.

    A differing top or tail code must be a neighbour of the oracle's, with the oracle's z_j
    within 1e-5 ||x|| of the boundary between them (spectral records carry no norm, so the
    band is taken at the vector's own scale).  The QJL residual is recomputed from the
    adopted top codes; a differing sign bit must have |(S r)_i| <= 1e-5 ||S_i|| ||x||.
    """
    from oracle.spectral import unpack_spectral
    x = np.asarray(x, dtype=np.float64)
    xn = np.linalg.norm(x, axis=1)
    idx_g, s_g = unpack_spectral(np.asarray(gpu_codes, dtype=np.uint32), desc)
    idx = np.array(ref["idx"], copy=True)
    z = ref["z"]
    n, d = z.shape
    bad = exempt = 0
    for i, j in zip(*np.nonzero(idx_g != idx)):
        b = int(desc["bits"][j])
        lo = int(min(idx_g[i, j], idx[i, j]))
        t = desc["books"][b][1][lo] * desc["sigma"][j]
        if abs(int(idx_g[i, j]) - int(idx[i, j])) == 1 and abs(z[i, j] - t) <= BAND * xn[i]:
            exempt += 1
            idx[i, j] = idx_g[i, j]
        else:
            bad += 1
    assert bad == 0, f"{bad} spectral code mismatches outside the band ({exempt} exempt)"
    chat = np.zeros((n, d))
    for j in range(d):
        b = int(desc["bits"][j])
        if b:
            chat[:, j] = desc["sigma"][j] * desc["books"][b][0][idx[:, j]]
    out = {"idx": idx, "chat": chat, "exempt": exempt}
    if desc["qjl"]:
        k = desc["k_top"]
        S = np.asarray(desc["S_top"], dtype=np.float64)
        r = z[:, :k] - chat[:, :k]
        gamma = np.sqrt(np.sum(r * r, axis=1))
        proj = r @ S.T
        sr = (proj >= 0).astype(np.int64)
        diff = s_g != sr
        outside = diff & (np.abs(proj) > BAND * np.linalg.norm(S, axis=1)[None, :] * xn[:, None])
        assert not np.any(outside), f"{int(outside.sum())} spectral sign mismatches outside the band"
        rn = np.asarray(gpu_rnorms, dtype=np.float64)
        # the top coordinates are O(sigma_0) ~ 10: gamma carries absolute rounding ~1e-6 ||x||
        assert np.all(np.abs(rn - gamma) <= 1e-5 * xn), "spectral residual norms"
        out["s"], out["rnorms"] = s_g, gamma
    return out
