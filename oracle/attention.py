"""fp64 oracle: single-token decode attention over a block-DCT archive.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Three paths that must agree to rounding:

* ``decode_attention_reference`` -- the plain definition: reconstruct every
  archived token (X_hat = M^T C_hat per block), append the raw tail, then
  softmax(scale * q . K_hat^T) @ V_hat. Query head hq reads kv head
  hq // G with G = Hq / Hk (``flashcodec/triton_attention.py``: the program
  for kv head h and group member g serves query head h * G + g).
* ``coeff_decode_attention`` -- the coefficient-domain method, block by block
  in the order the pages give it (``flashcodec/triton_attention.py`` module
  docstring; README "Materialization-free decode attention":
  q . K[p] = (q . S^T) @ A[p], out = (prob @ A) @ S): s = C_k q,
  logits = scale * A s, online-softmax update, w = p A, acc += w C_v; the raw
  tail tokens are folded into the same softmax one at a time.
* ``splitk_decode_attention`` -- the same per-block loop over contiguous block
  chunks (the raw tail belongs to the last chunk), each chunk leaving a
  (max, sum, acc) partial, merged by the flash-decoding combine
  (``flashcodec/triton_attention.py``, split and combine kernels).

Readings where the pages are silent: the softmax scale defaults to D**-0.5
(``codec_decode_attention_triton``); a chunk with no blocks and no tail
contributes (m=-inf, l=0) and the combine skips it instead of producing NaN.
"""

from __future__ import annotations

import numpy as np

from .codec import decompress, synthesis_basis

F64 = np.float64


def _as64(x):
    return None if x is None else np.asarray(x, dtype=F64)


def decode_attention_reference(q, C_hat_k, C_hat_v, tail_k, tail_v, R,
                               scale=None):
    """Decompress-then-attend.

    q (B, Hq, 1, D); C_hat_* (B, Hk, nb, S, D) archived coefficients as
    float64 (code * scale when quantised); tail_* (B, Hk, nr, D) raw tokens.
    Returns out (B, Hq, 1, D) float64.
    """
    q = _as64(q)
    B, Hq, _, D = q.shape
    K = decompress(C_hat_k, R)
    V = decompress(C_hat_v, R)
    if tail_k is not None and tail_k.shape[-2] > 0:
        K = np.concatenate([K, _as64(tail_k)], axis=-2)
        V = np.concatenate([V, _as64(tail_v)], axis=-2)
    Hk = K.shape[1]
    if Hq % Hk:
        raise ValueError("Hq must be a multiple of Hk")
    G = Hq // Hk
    if K.shape[-2] == 0:
        raise ValueError("decode attention needs at least one token")
    sc = D ** -0.5 if scale is None else float(scale)
    Kx = np.repeat(K, G, axis=1)            # (B, Hq, T, D): head hq -> hq // G
    Vx = np.repeat(V, G, axis=1)
    logits = sc * np.einsum("bhd,bhtd->bht", q[:, :, 0, :], Kx)
    logits -= logits.max(axis=-1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=-1, keepdims=True)
    out = np.einsum("bht,bhtd->bhd", p, Vx)
    return out[:, :, None, :]


def _online_blocks(qg, Ck, Cv, A, sc, m, l, acc):
    """Per-block coefficient-domain update for the G query heads of one kv
    head. qg (G, D); Ck, Cv (n, S, D); A (R, S); state m, l (G,), acc (G, D)."""
    for n in range(Ck.shape[0]):
        s = Ck[n] @ qg.T                      # (S, G): s_j = C_k[j] . q
        logits = sc * (A @ s)                 # (R, G)
        m_new = np.maximum(m, logits.max(axis=0))
        p = np.exp(logits - m_new)            # (R, G)
        alpha = np.exp(m - m_new)
        l = l * alpha + p.sum(axis=0)
        w = p.T @ A                           # (G, S): w_j = sum_t p_t A[t, j]
        acc = acc * alpha[:, None] + w @ Cv[n]
        m = m_new
    return m, l, acc


def _online_tail(qg, tk, tv, sc, m, l, acc):
    """Fold raw tail tokens one at a time into the same softmax."""
    for t in range(tk.shape[0]):
        logit = sc * (qg @ tk[t])             # (G,)
        m_new = np.maximum(m, logit)
        p = np.exp(logit - m_new)
        alpha = np.exp(m - m_new)
        l = l * alpha + p
        acc = acc * alpha[:, None] + p[:, None] * tv[t][None, :]
        m = m_new
    return m, l, acc


def _fresh_state(G, D):
    return (np.full(G, -np.inf), np.zeros(G), np.zeros((G, D)))


def coeff_decode_attention(q, C_hat_k, C_hat_v, tail_k, tail_v, R,
                           scale=None):
    """Coefficient-domain decode attention (same arguments as
    ``decode_attention_reference``)."""
    q = _as64(q)
    Ck, Cv = _as64(C_hat_k), _as64(C_hat_v)
    B, Hq, _, D = q.shape
    Hk, S = Ck.shape[1], Ck.shape[3]
    G = Hq // Hk
    A = synthesis_basis(R, S)
    sc = D ** -0.5 if scale is None else float(scale)
    tk = _as64(tail_k)
    tv = _as64(tail_v)
    out = np.empty((B, Hq, 1, D))
    for b in range(B):
        for h in range(Hk):
            qg = q[b, h * G:(h + 1) * G, 0, :]
            m, l, acc = _fresh_state(G, D)
            m, l, acc = _online_blocks(qg, Ck[b, h], Cv[b, h], A, sc, m, l,
                                       acc)
            if tk is not None and tk.shape[-2] > 0:
                m, l, acc = _online_tail(qg, tk[b, h], tv[b, h], sc, m, l,
                                         acc)
            out[b, h * G:(h + 1) * G, 0, :] = acc / l[:, None]
    return out


def split_partials(q, C_hat_k, C_hat_v, tail_k, tail_v, R, num_splits,
                   scale=None):
    """Split-K partials: chunk c covers blocks [c*chunk, min((c+1)*chunk, nb))
    with chunk = ceil(nb / num_splits); the raw tail goes to the last chunk.

    Returns (m (B, Hq, ns), l (B, Hq, ns), acc (B, Hq, ns, D)).
    """
    q = _as64(q)
    Ck, Cv = _as64(C_hat_k), _as64(C_hat_v)
    B, Hq, _, D = q.shape
    Hk, nb, S = Ck.shape[1], Ck.shape[2], Ck.shape[3]
    G = Hq // Hk
    ns = int(num_splits)
    if ns < 1:
        raise ValueError("num_splits >= 1")
    chunk = -(-nb // ns) if nb else 0
    A = synthesis_basis(R, S)
    sc = D ** -0.5 if scale is None else float(scale)
    tk, tv = _as64(tail_k), _as64(tail_v)
    M = np.full((B, Hq, ns), -np.inf)
    L = np.zeros((B, Hq, ns))
    ACC = np.zeros((B, Hq, ns, D))
    for b in range(B):
        for h in range(Hk):
            qg = q[b, h * G:(h + 1) * G, 0, :]
            for c in range(ns):
                lo, hi = c * chunk, min((c + 1) * chunk, nb)
                m, l, acc = _fresh_state(G, D)
                if hi > lo:
                    m, l, acc = _online_blocks(qg, Ck[b, h, lo:hi],
                                               Cv[b, h, lo:hi], A, sc, m, l,
                                               acc)
                if c == ns - 1 and tk is not None and tk.shape[-2] > 0:
                    m, l, acc = _online_tail(qg, tk[b, h], tv[b, h], sc, m,
                                             l, acc)
                sl = slice(h * G, (h + 1) * G)
                M[b, sl, c], L[b, sl, c], ACC[b, sl, c] = m, l, acc
    return M, L, ACC


def combine_partials(M, L, ACC):
    """Merge (max, sum, acc) partials over the last split axis:
    Mx = max_c m_c, Lx = sum_c l_c e^{m_c - Mx}, out = sum_c acc_c
    e^{m_c - Mx} / Lx. Chunks with l_c = 0 are skipped.

    Returns out (B, Hq, 1, D)."""
    M = np.asarray(M, dtype=F64)
    L = np.asarray(L, dtype=F64)
    ACC = np.asarray(ACC, dtype=F64)
    live = L > 0
    Mm = np.where(live, M, -np.inf)
    Mx = Mm.max(axis=-1, keepdims=True)
    wgt = np.where(live, np.exp(Mm - Mx), 0.0)
    Lx = (L * wgt).sum(axis=-1)
    out = (ACC * wgt[..., None]).sum(axis=-2) / Lx[..., None]
    return out[:, :, None, :]


def splitk_decode_attention(q, C_hat_k, C_hat_v, tail_k, tail_v, R,
                            num_splits, scale=None):
    """Split-K partials followed by the combine."""
    return combine_partials(*split_partials(q, C_hat_k, C_hat_v, tail_k,
                                            tail_v, R, num_splits, scale))


def attend_archive(q, C_hat_k, C_hat_v, tail_k, tail_v, R, heads,
                   scale=None):
    """Reference attention for selected (b, hq) pairs only, one at a time,
    so that full-size workloads can be checked on samples.

    ``heads`` is an iterable of (b, hq). Returns a dict (b, hq) -> (D,)."""
    q = _as64(q)
    D = q.shape[-1]
    Hq = q.shape[1]
    Hk = C_hat_k.shape[1]
    G = Hq // Hk
    out = {}
    for b, hq in heads:
        h = hq // G
        sl = (slice(b, b + 1), slice(h, h + 1))
        tk = None if tail_k is None else tail_k[sl]
        tv = None if tail_v is None else tail_v[sl]
        o = decode_attention_reference(q[b:b + 1, hq:hq + 1], C_hat_k[sl],
                                       C_hat_v[sl], tk, tv, R, scale)
        out[(b, hq)] = o[0, 0, 0]
    return out
