"""Plain fp64 CPU oracle for Jet-Long bifocal-RoPE attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the package's
``smoke()`` check and the ``cpu_baseline`` / reference arm of ``bench.py`` may
import this module.  It shares no code, table or constant with the CUDA library;
the two meet only through the seeded inputs the tests hand to both.

Everything here is the definition written out, in float64, with explicit per
(query i, key j) positions and masks.  Sources (page "Jet-Long: Efficient
Long-Context Extension with Dynamic Bifocal RoPE", full text):

* §3, display equation of S(q, k): the bifocal score rule.  A key within the
  protected local window (q - k <= w0) is scored with both vectors rotated to
  their true positions; an older key is scored with both rotated to the remapped
  positions f(q), f(k).
* §3.1, Eq. (2): G = max(1, ceil(L / w_pretrained)); and f(x) = floor(x / G).
* §3.2: the KV cache holds RoPE(x_k, k) at true positions; the correction
  rotation by Delta k = f(k) - k turns a cached key into RoPE(x_k, f(k)).
* §3.3: inclusion-exclusion merge of three attention passes (kept here only as
  an independent cross-check in ``merge_three_pass``; the oracle proper scores
  each pair directly).
* §2.1: RoPE rotates channel pairs at geometrically spaced frequencies, so that
  a dot product depends only on the relative position.
* §4.7 and Table 6 (ablation of the remote map): frequency interpolation in
  place of position aliasing, in ``interp_freq`` and the ``*_interp``
  functions; the readings it needs are stated above ``interp_scale``.
* Appendix H ("Hardware, precision, and software"): BF16 Q/K/V, FP32 softmax
  and log-sum-exp statistics; the oracle works in float64 on the BF16 values.

Readings where the pages are silent (each also listed in the design notes):
positions are 0-based; local iff 0 <= i - j <= w0 (inclusive, consistent with
the remark in §4.6 that w0 = 0 keeps self-attention in the local branch); one G
per prefill call from the full length L; the decode query sits at position L-1
with L counting the new token (Appendix E: 98,304 -> 98,305 moves G from 3 to
4); rotate-half channel pairing (i, i + D/2) with frequency theta^(-2i/D);
softmax scale 1/sqrt(D) and no temperature; GQA head h reads KV head
h // (Hq / Hkv); log-sum-exp in natural log.

Every function is pinned by tests that do not retype it (see tests/).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "group_size",
    "remap",
    "inv_freq",
    "rope",
    "rope_cache",
    "correction_rotate",
    "prefill",
    "prefill_rows",
    "prefill_literal",
    "decode",
    "prefill_chunk",
    "merge_three_pass",
    "interp_scale",
    "interp_freq",
    "rope_at_freq",
    "prefill_interp_rows",
    "prefill_interp",
    "prefill_interp_literal",
    "correction_rotate_interp",
    "prefill_chunk_interp",
    "decode_interp",
]


# --------------------------------------------------------------------------
# Schedule (§3.1)
# --------------------------------------------------------------------------
def group_size(L: int, w_pretrained: int) -> int:
    """Dynamic group size of §3.1, Eq. (2): G = max(1, ceil(L / w_pretrained)).

    Integer arithmetic only: ceil(a / b) for positive ints is -((-a) // b).
    """
    L = int(L)
    w = int(w_pretrained)
    if L < 1 or w < 1:
        raise ValueError("L and w_pretrained must be >= 1")
    return max(1, -((-L) // w))


def remap(x, G: int):
    """Remote position map of §3.1: f(x) = floor(x / G) (identity when G == 1)."""
    return np.floor_divide(np.asarray(x, dtype=np.int64), int(G))


# --------------------------------------------------------------------------
# RoPE (§2.1) and the true-position cache + correction (§3.2)
# --------------------------------------------------------------------------
def inv_freq(D: int, theta: float) -> np.ndarray:
    """Frequencies theta^(-2i/D) for i < D/2, in float64."""
    i = np.arange(D // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * i / np.float64(D))


def rope(x, pos, theta: float) -> np.ndarray:
    """RoPE(x, p): rotate each channel pair (i, i + D/2) by angle p * theta^(-2i/D).

    x: [..., D] (any float dtype; computed in float64).  pos: integer array that
    broadcasts against x[..., 0].  Returns float64 [..., D].
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    h = D // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq(D, theta)
    c = np.cos(ang)
    s = np.sin(ang)
    a = x[..., :h]
    b = x[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def rope_cache(k, pos0: int, theta: float) -> np.ndarray:
    """§3.2: k_cache[k] = RoPE(x_k, k) for the true positions pos0 .. pos0+n-1.

    k: [B, n, Hkv, D] pre-RoPE keys.  Returns float64 [B, n, Hkv, D].
    """
    k = np.asarray(k, dtype=np.float64)
    n = k.shape[1]
    pos = (np.arange(n, dtype=np.int64) + int(pos0))[None, :, None]
    return rope(k, pos, theta)


def correction_rotate(c, kpos, G: int, theta: float) -> np.ndarray:
    """§3.2 correction: rotate a cached key c = RoPE(x, k) by Delta k = f(k) - k."""
    kpos = np.asarray(kpos, dtype=np.int64)
    delta = remap(kpos, G) - kpos
    return rope(c, delta, theta)


# --------------------------------------------------------------------------
# Bifocal attention (§3 score rule), prefill
# --------------------------------------------------------------------------
def _check_shapes(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, L, H, D]")
    B, L, Hq, D = q.shape
    if k.shape[:2] != (B, L) or v.shape != k.shape or k.shape[3] != D:
        raise ValueError("k, v must be [B, L, Hkv, D] matching q")
    Hkv = k.shape[2]
    if Hq % Hkv != 0 or D % 2 != 0:
        raise ValueError("Hq must be a multiple of Hkv and D even")
    return B, L, Hq, Hkv, D


def prefill_rows(q, k, v, w_pretrained: int, w0: int, theta: float, rows,
                 q_holds_rows: bool = False):
    """Bifocal causal attention for the listed query rows (all heads, all batches).

    For query i and key j <= i (§3 score rule, §3.1 schedule, one G for the
    whole prompt of length L):

      s_ij = RoPE(x_q[i], i) . RoPE(x_k[j], j) / sqrt(D)          if i - j <= w0
      s_ij = RoPE(x_q[i], f(i)) . RoPE(x_k[j], f(j)) / sqrt(D)    otherwise

    lse_i = log sum_j exp(s_ij);  o_i = sum_j exp(s_ij - lse_i) v_j.

    Both candidate scores are computed for every pair and the rule picks one
    per (i, j) with an explicit mask; keys are scored in one vectorised product
    per row, which is the same arithmetic as a per-pair loop.

    The prompt length L (and with it G) is k.shape[1].  With
    ``q_holds_rows`` q is [B, len(rows), Hq, D] and holds only the listed
    rows' queries, in the order of ``rows``.

    Returns (o [B, len(rows), Hq, D] float64, lse [B, Hq, len(rows)] float64).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    rows = np.asarray(rows, dtype=np.int64)
    if q_holds_rows:
        if q.ndim != 4 or q.shape[1] != rows.size:
            raise ValueError("q must be [B, len(rows), Hq, D]")
        B, L, Hq, Hkv, D = _check_shapes(np.broadcast_to(q[:, :1], (q.shape[0], k.shape[1]) + q.shape[2:]), k, v)
    else:
        B, L, Hq, Hkv, D = _check_shapes(q, k, v)
    if rows.size and (rows.min() < 0 or rows.max() >= L):
        raise ValueError("row out of range")
    grp = Hq // Hkv
    G = group_size(L, w_pretrained)
    scale = 1.0 / math.sqrt(D)
    jmax = int(rows.max()) + 1 if rows.size else 0
    jpos = np.arange(jmax, dtype=np.int64)
    o = np.zeros((B, rows.size, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq, rows.size), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            xk = k[b, :jmax, g, :].astype(np.float64)
            vv = v[b, :jmax, g, :].astype(np.float64)
            k_true = rope(xk, jpos, theta)             # RoPE(x_k, j)
            k_remote = rope(xk, remap(jpos, G), theta)  # RoPE(x_k, f(j))
            heads = np.arange(g * grp, (g + 1) * grp)
            for r, i in enumerate(rows):
                qi = r if q_holds_rows else i
                xq = q[b, qi, heads, :].astype(np.float64)          # [grp, D]
                q_true = rope(xq, np.int64(i), theta)                 # RoPE(x_q, i)
                q_remote = rope(xq, remap(np.int64(i), G), theta)     # RoPE(x_q, f(i))
                n = i + 1                                             # causal: j <= i
                s_local = k_true[:n] @ q_true.T                       # [n, grp]
                s_remote = k_remote[:n] @ q_remote.T
                dist = (i - jpos[:n])[:, None]
                s = np.where(dist <= w0, s_local, s_remote) * scale
                m = s.max(axis=0)
                e = np.exp(s - m)
                tot = e.sum(axis=0)
                lse[b, heads, r] = m + np.log(tot)
                o[b, r, heads, :] = (e / tot).T @ vv[:n]
    return o, lse


def prefill(q, k, v, w_pretrained: int, w0: int, theta: float):
    """Bifocal causal attention over every query row: (o [B,L,Hq,D], lse [B,Hq,L])."""
    L = np.asarray(q).shape[1]
    return prefill_rows(q, k, v, w_pretrained, w0, theta, np.arange(L))


def prefill_literal(q, k, v, w_pretrained: int, w0: int, theta: float):
    """Pure-Python per-pair version for tiny inputs.

    Re-rotates the query and the key for every (i, j) pair with a 2x2 rotation
    per channel pair written out by hand, picks the position pair by the §3
    rule, and runs a two-pass softmax.  No vectorisation, no precomputed
    rotated vectors: it shares no intermediate with ``prefill_rows``.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, L, Hq, Hkv, D = _check_shapes(q, k, v)
    grp = Hq // Hkv
    G = group_size(L, w_pretrained)
    h2 = D // 2
    freqs = [float(theta) ** (-2.0 * t / D) for t in range(h2)]

    def rot(x, p):
        out = [0.0] * D
        for t in range(h2):
            a = p * freqs[t]
            ca, sa = math.cos(a), math.sin(a)
            out[t] = x[t] * ca - x[t + h2] * sa
            out[t + h2] = x[t] * sa + x[t + h2] * ca
        return out

    o = np.zeros((B, L, Hq, D))
    lse = np.zeros((B, Hq, L))
    for b in range(B):
        for h in range(Hq):
            g = h // grp
            for i in range(L):
                scores = []
                for j in range(i + 1):
                    if i - j <= w0:
                        pi, pj = i, j
                    else:
                        pi, pj = i // G, j // G
                    qa = rot(list(q[b, i, h]), pi)
                    kb = rot(list(k[b, j, g]), pj)
                    scores.append(sum(x * y for x, y in zip(qa, kb)) / math.sqrt(D))
                m = max(scores)
                tot = sum(math.exp(s - m) for s in scores)
                lse[b, h, i] = m + math.log(tot)
                for j, s in enumerate(scores):
                    w = math.exp(s - m) / tot
                    o[b, i, h] += w * v[b, j, g]
    return o, lse


# --------------------------------------------------------------------------
# Decode on the true-position cache (§3.2)
# --------------------------------------------------------------------------
def decode(q, k_cache, v_cache, L: int, w_pretrained: int, w0: int, theta: float):
    """One generation step at query position p = L - 1 on a true-position cache.

    q: [B, Hq, D] pre-RoPE query of the new token.  k_cache: [B, >=L, Hkv, D]
    holding RoPE(x_k, k) (§3.2, never rewritten); v_cache likewise (values are
    not rotated).  G is recomputed from this L (§3.1).  For key j <= p:

      local  (p - j <= w0): s = RoPE(x_q, p) . k_cache[j]
      remote (p - j >  w0): s = RoPE(x_q, f(p)) . R(Delta j) k_cache[j],
                            Delta j = f(j) - j   (§3.2 correction rotation)

    scaled by 1/sqrt(D).  Returns (o [B, Hq, D], lse [B, Hq]) in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    kc = np.asarray(k_cache)
    vc = np.asarray(v_cache)
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    if kc.shape[1] < L or vc.shape[:3] != kc.shape[:3]:
        raise ValueError("cache shorter than L")
    grp = Hq // Hkv
    G = group_size(L, w_pretrained)
    p = L - 1
    scale = 1.0 / math.sqrt(D)
    jpos = np.arange(L, dtype=np.int64)
    local = (p - jpos) <= w0
    o = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for g in range(Hkv):
            c = kc[b, :L, g, :].astype(np.float64)
            vv = vc[b, :L, g, :].astype(np.float64)
            c_corr = correction_rotate(c, jpos, G, theta)
            heads = np.arange(g * grp, (g + 1) * grp)
            q_true = rope(q[b, heads], np.int64(p), theta)
            q_remote = rope(q[b, heads], remap(np.int64(p), G), theta)
            s_local = c @ q_true.T
            s_remote = c_corr @ q_remote.T
            s = np.where(local[:, None], s_local, s_remote) * scale
            m = s.max(axis=0)
            e = np.exp(s - m)
            tot = e.sum(axis=0)
            lse[b, heads] = m + np.log(tot)
            o[b, heads, :] = (e / tot).T @ vv
    return o, lse


# --------------------------------------------------------------------------
# Chunked prefill on the true-position cache (§3.1 schedule, §3.2 cache)
# --------------------------------------------------------------------------
def prefill_chunk(q, k_cache, v_cache, P0: int, w_pretrained: int, w0: int, theta: float,
                  rows=None):
    """A chunk of n new tokens at positions P0 .. P0+n-1 appended to a prompt.

    q: [B, n, Hq, D] pre-RoPE queries of the chunk.  k_cache / v_cache:
    [B, >=P0+n, Hkv, D], rows [0, P0+n) valid, keys at true positions (the
    chunk's own keys already appended, §3.2).  One G for the call, from the
    length after the chunk, L = P0 + n (§3.1: G follows the current sequence
    length; one G per prefill call).  Query i sits at p = P0 + i and sees keys
    j <= p, scored like a decode step with that G:

      local  (p - j <= w0): s = RoPE(x_q, p) . k_cache[j]
      remote (p - j >  w0): s = RoPE(x_q, f(p)) . R(f(j) - j) k_cache[j]

    scaled by 1/sqrt(D).  Returns (o [B, n, Hq, D], lse [B, Hq, n]), float64.
    With P0 = 0 and n = L this is the whole-prompt prefill.  ``rows`` (chunk
    indices) restricts the work to those queries; the others stay zero.
    """
    q = np.asarray(q, dtype=np.float64)
    kc = np.asarray(k_cache)
    vc = np.asarray(v_cache)
    B, n, Hq, D = q.shape
    Hkv = kc.shape[2]
    L = P0 + n
    if kc.shape[1] < L or vc.shape[:3] != kc.shape[:3]:
        raise ValueError("cache shorter than P0 + n")
    grp = Hq // Hkv
    G = group_size(L, w_pretrained)
    scale = 1.0 / math.sqrt(D)
    o = np.zeros((B, n, Hq, D))
    lse = np.zeros((B, Hq, n))
    jpos_all = np.arange(L, dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            c_all = kc[b, :L, g, :].astype(np.float64)
            v_all = vc[b, :L, g, :].astype(np.float64)
            c_corr_all = correction_rotate(c_all, jpos_all, G, theta)
            heads = np.arange(g * grp, (g + 1) * grp)
            for i in (range(n) if rows is None else rows):
                p = P0 + i
                c, cc, vv = c_all[: p + 1], c_corr_all[: p + 1], v_all[: p + 1]
                local = (p - jpos_all[: p + 1]) <= w0
                q_true = rope(q[b, i, heads], np.int64(p), theta)
                q_remote = rope(q[b, i, heads], remap(np.int64(p), G), theta)
                s = np.where(local[:, None], c @ q_true.T, cc @ q_remote.T) * scale
                m = s.max(axis=0)
                e = np.exp(s - m)
                tot = e.sum(axis=0)
                lse[b, heads, i] = m + np.log(tot)
                o[b, i, heads, :] = (e / tot).T @ vv
    return o, lse


# --------------------------------------------------------------------------
# §3.3 inclusion-exclusion merge, as three separate passes (cross-check only)
# --------------------------------------------------------------------------
def merge_three_pass(q, k, v, w_pretrained: int, w0: int, theta: float):
    """O = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C)  (§3.3).

    Reading of A, B, C (the pages do not define them): A = remote-position
    causal attention over all j <= i; B = true-position attention on the band
    0 <= i - j <= w0; C = remote-position attention on the same band.
    W_X = sum_j exp(s_ij) over pass X's keys, so W_A + W_B - W_C sums exactly
    the bifocal scores.  Each pass is a plain masked softmax.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, L, Hq, Hkv, D = _check_shapes(q, k, v)
    grp = Hq // Hkv
    G = group_size(L, w_pretrained)
    pos = np.arange(L, dtype=np.int64)
    dist = pos[:, None] - pos[None, :]
    causal = dist >= 0
    band = causal & (dist <= w0)
    scale = 1.0 / math.sqrt(D)

    def one_pass(qr, kr, vv, mask):
        s = np.where(mask, (qr @ kr.T) * scale, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        w = e.sum(axis=1, keepdims=True)
        return (e / w) @ vv, np.log(w[:, 0]) + m[:, 0]

    o = np.zeros((B, L, Hq, D))
    lse = np.zeros((B, Hq, L))
    for b in range(B):
        for h in range(Hq):
            g = h // grp
            qt = rope(q[b, :, h], pos, theta)
            qf = rope(q[b, :, h], remap(pos, G), theta)
            kt = rope(k[b, :, g], pos, theta)
            kf = rope(k[b, :, g], remap(pos, G), theta)
            oa, la = one_pass(qf, kf, v[b, :, g], causal)
            ob, lb = one_pass(qt, kt, v[b, :, g], band)
            oc, lc = one_pass(qf, kf, v[b, :, g], band)
            M = np.maximum(np.maximum(la, lb), lc)
            wa, wb, wc = np.exp(la - M), np.exp(lb - M), np.exp(lc - M)
            den = wa + wb - wc
            o[b, :, h] = (wa[:, None] * oa + wb[:, None] * ob - wc[:, None] * oc) / den[:, None]
            lse[b, h] = M + np.log(den)
    return o, lse


# --------------------------------------------------------------------------
# §4.7 ablation: frequency interpolation instead of position aliasing
# --------------------------------------------------------------------------
# Table 6 of the page compares the default remote map (positions aliased to
# f(x) = floor(x / G)) with a YaRN-like interpolation of the frequencies inside
# the same bifocal scheme, but gives no formula for it; the readings taken
# here (each also listed in the design notes):
#
# * The local band is untouched: pairs with 0 <= i - j <= w0 are scored at true
#   positions with the pretrained frequencies.  Only the remote map changes.
# * Remote pairs are scored at their TRUE positions with per-frequency
#   interpolated frequencies theta'_t (YaRN's "NTK-by-parts" rule):
#     r_t     = w_pretrained * theta_t / (2 pi)   turns of frequency t within the
#                                                 pretrained window,
#     gamma_t = clip((r_t - alpha) / (beta - alpha), 0, 1),
#     theta'_t = theta_t * ((1 - gamma_t) / s + gamma_t),
#   so slow frequencies (few turns, r_t < alpha) are divided by s and fast ones
#   (r_t > beta) are kept.  alpha = 1, beta = 32 are YaRN's published defaults.
# * s is the dynamic factor the page names for continuous rescaling in §3.1,
#   s = max(1, L / w_pretrained), recomputed from the current length like G.
# * No attention temperature: the softmax scale stays 1/sqrt(D) (the ablation
#   changes only how remote positions are mapped).
# * The cache still holds RoPE(x_k, j) at true positions (§3.2); a cached key
#   is turned into the remote form by the rotation of angle j (theta'_t - theta_t).
def interp_scale(L: int, w_pretrained: int) -> float:
    """Continuous dynamic factor of §3.1: s = max(1, L / w_pretrained)."""
    L = int(L)
    w = int(w_pretrained)
    if L < 1 or w < 1:
        raise ValueError("L and w_pretrained must be >= 1")
    return max(1.0, L / w)


def interp_freq(D: int, theta: float, L: int, w_pretrained: int, alpha: float = 1.0,
                beta: float = 32.0) -> np.ndarray:
    """Interpolated frequencies theta'_t, t < D/2, of the remote branch (float64)."""
    if not beta > alpha:
        raise ValueError("beta must exceed alpha")
    base = inv_freq(D, theta)
    s = interp_scale(L, w_pretrained)
    turns = float(w_pretrained) * base / (2.0 * math.pi)
    gamma = np.clip((turns - alpha) / (beta - alpha), 0.0, 1.0)
    return base * ((1.0 - gamma) / s + gamma)


def rope_at_freq(x, pos, freqs) -> np.ndarray:
    """Rotate each channel pair (t, t + D/2) of x by angle pos * freqs[t]."""
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[-1] // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * np.asarray(freqs, dtype=np.float64)
    c = np.cos(ang)
    s = np.sin(ang)
    a = x[..., :h]
    b = x[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def prefill_interp_rows(q, k, v, w_pretrained: int, w0: int, theta: float, rows,
                        alpha: float = 1.0, beta: float = 32.0, q_holds_rows: bool = False):
    """Frequency-interpolation variant of ``prefill_rows`` for the listed rows.

      s_ij = RoPE(x_q[i], i) . RoPE(x_k[j], j) / sqrt(D)      if i - j <= w0
      s_ij = RoPE'(x_q[i], i) . RoPE'(x_k[j], j) / sqrt(D)    otherwise

    RoPE' rotates with ``interp_freq`` (one s for the prompt, from L =
    k.shape[1]).  With ``q_holds_rows`` q is [B, len(rows), Hq, D] and holds
    only the listed rows' queries.  Returns (o [B, len(rows), Hq, D],
    lse [B, Hq, len(rows)]).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    rows = np.asarray(rows, dtype=np.int64)
    if q_holds_rows:
        if q.ndim != 4 or q.shape[1] != rows.size:
            raise ValueError("q must be [B, len(rows), Hq, D]")
        B, L, Hq, Hkv, D = _check_shapes(np.broadcast_to(q[:, :1], (q.shape[0], k.shape[1]) + q.shape[2:]), k, v)
    else:
        B, L, Hq, Hkv, D = _check_shapes(q, k, v)
    if rows.size and (rows.min() < 0 or rows.max() >= L):
        raise ValueError("row out of range")
    grp = Hq // Hkv
    fr = interp_freq(D, theta, L, w_pretrained, alpha, beta)
    scale = 1.0 / math.sqrt(D)
    jmax = int(rows.max()) + 1 if rows.size else 0
    jpos = np.arange(jmax, dtype=np.int64)
    o = np.zeros((B, rows.size, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq, rows.size), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            xk = k[b, :jmax, g, :].astype(np.float64)
            vv = v[b, :jmax, g, :].astype(np.float64)
            k_true = rope(xk, jpos, theta)
            k_remote = rope_at_freq(xk, jpos, fr)
            heads = np.arange(g * grp, (g + 1) * grp)
            for r, i in enumerate(rows):
                xq = q[b, r if q_holds_rows else i, heads, :].astype(np.float64)
                q_true = rope(xq, np.int64(i), theta)
                q_remote = rope_at_freq(xq, np.int64(i), fr)
                n = i + 1
                dist = (i - jpos[:n])[:, None]
                s = np.where(dist <= w0, k_true[:n] @ q_true.T, k_remote[:n] @ q_remote.T) * scale
                m = s.max(axis=0)
                e = np.exp(s - m)
                tot = e.sum(axis=0)
                lse[b, heads, r] = m + np.log(tot)
                o[b, r, heads, :] = (e / tot).T @ vv[:n]
    return o, lse


def prefill_interp(q, k, v, w_pretrained: int, w0: int, theta: float, alpha: float = 1.0,
                   beta: float = 32.0):
    """Frequency-interpolation variant over every query row: (o, lse)."""
    L = np.asarray(q).shape[1]
    return prefill_interp_rows(q, k, v, w_pretrained, w0, theta, np.arange(L), alpha, beta)


def prefill_interp_literal(q, k, v, w_pretrained: int, w0: int, theta: float,
                           alpha: float = 1.0, beta: float = 32.0):
    """Pure-Python per-pair version of ``prefill_interp`` for tiny inputs.

    Forms both frequency sets with scalar ``math`` calls, re-rotates the query
    and key of every pair by hand, and runs a two-pass softmax; it shares no
    intermediate with the vectorised version.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, L, Hq, Hkv, D = _check_shapes(q, k, v)
    grp = Hq // Hkv
    h2 = D // 2
    s_fac = max(1.0, L / w_pretrained)
    base, interp = [], []
    for t in range(h2):
        f = float(theta) ** (-2.0 * t / D)
        turns = w_pretrained * f / (2.0 * math.pi)
        gam = min(1.0, max(0.0, (turns - alpha) / (beta - alpha)))
        base.append(f)
        interp.append(f * ((1.0 - gam) / s_fac + gam))

    def rot(x, p, freqs):
        out = [0.0] * D
        for t in range(h2):
            a = p * freqs[t]
            ca, sa = math.cos(a), math.sin(a)
            out[t] = x[t] * ca - x[t + h2] * sa
            out[t + h2] = x[t] * sa + x[t + h2] * ca
        return out

    o = np.zeros((B, L, Hq, D))
    lse = np.zeros((B, Hq, L))
    for b in range(B):
        for h in range(Hq):
            g = h // grp
            for i in range(L):
                scores = []
                for j in range(i + 1):
                    freqs = base if i - j <= w0 else interp
                    qa = rot(list(q[b, i, h]), i, freqs)
                    kb = rot(list(k[b, j, g]), j, freqs)
                    scores.append(sum(x * y for x, y in zip(qa, kb)) / math.sqrt(D))
                m = max(scores)
                tot = sum(math.exp(s - m) for s in scores)
                lse[b, h, i] = m + math.log(tot)
                for j, s in enumerate(scores):
                    o[b, i, h] += math.exp(s - m) / tot * v[b, j, g]
    return o, lse


def correction_rotate_interp(c, kpos, freq_interp, theta: float) -> np.ndarray:
    """Turn a cached key c = RoPE(x, j) into RoPE'(x, j): rotate by angle
    j * (theta'_t - theta_t) per channel pair (the §3.2 correction for this map)."""
    D = np.asarray(c).shape[-1]
    return rope_at_freq(c, kpos, np.asarray(freq_interp) - inv_freq(D, theta))


def prefill_chunk_interp(q, k_cache, v_cache, P0: int, w_pretrained: int, w0: int,
                         theta: float, alpha: float = 1.0, beta: float = 32.0, rows=None):
    """Frequency-interpolation variant of ``prefill_chunk``: queries at P0 ..
    P0+n-1 on the true-position cache, one s from L = P0 + n.

      local  (p - j <= w0): s = RoPE(x_q, p) . k_cache[j]
      remote (p - j >  w0): s = RoPE'(x_q, p) . R(j (theta' - theta)) k_cache[j]

    Returns (o [B, n, Hq, D], lse [B, Hq, n]) in float64.  ``rows`` (chunk
    indices) restricts the work to those queries; the others stay zero.
    """
    q = np.asarray(q, dtype=np.float64)
    kc = np.asarray(k_cache)
    vc = np.asarray(v_cache)
    B, n, Hq, D = q.shape
    Hkv = kc.shape[2]
    L = P0 + n
    if kc.shape[1] < L or vc.shape[:3] != kc.shape[:3]:
        raise ValueError("cache shorter than P0 + n")
    grp = Hq // Hkv
    fr = interp_freq(D, theta, L, w_pretrained, alpha, beta)
    scale = 1.0 / math.sqrt(D)
    o = np.zeros((B, n, Hq, D))
    lse = np.zeros((B, Hq, n))
    jpos_all = np.arange(L, dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            c_all = kc[b, :L, g, :].astype(np.float64)
            v_all = vc[b, :L, g, :].astype(np.float64)
            cc_all = correction_rotate_interp(c_all, jpos_all, fr, theta)
            heads = np.arange(g * grp, (g + 1) * grp)
            for i in (range(n) if rows is None else rows):
                p = P0 + i
                local = (p - jpos_all[: p + 1]) <= w0
                q_true = rope(q[b, i, heads], np.int64(p), theta)
                q_remote = rope_at_freq(q[b, i, heads], np.int64(p), fr)
                s = np.where(local[:, None], c_all[: p + 1] @ q_true.T,
                             cc_all[: p + 1] @ q_remote.T) * scale
                m = s.max(axis=0)
                e = np.exp(s - m)
                tot = e.sum(axis=0)
                lse[b, heads, i] = m + np.log(tot)
                o[b, i, heads, :] = (e / tot).T @ v_all[: p + 1]
    return o, lse


def decode_interp(q, k_cache, v_cache, L: int, w_pretrained: int, w0: int, theta: float,
                  alpha: float = 1.0, beta: float = 32.0):
    """One generation step of the frequency-interpolation variant at p = L - 1:
    the one-token chunk.  Returns (o [B, Hq, D], lse [B, Hq])."""
    q = np.asarray(q, dtype=np.float64)
    o, lse = prefill_chunk_interp(q[:, None], k_cache, v_cache, L - 1, w_pretrained, w0, theta,
                                  alpha, beta)
    return o[:, 0], lse[:, :, 0]
