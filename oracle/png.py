"""fp64 oracle: the PNG-style lossless tier of the codec and its decode
attention.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources (flashcodec-kv 1.0.0):
* README, "Math", PNG bullet: inside a block the first token x_0 is kept as
  the anchor and every later token is stored as its first difference
  Delta_i = x_i - x_{i-1} (i >= 1); the block is rebuilt by a cumulative sum,
  x_i = x_0 + sum_{j <= i} Delta_j.
* ``flashcodec/cache.py``, ``_CodecStream`` docstring and ``_archive_spec``:
  the archive holds deltas (B, H, capacity, r - 1, D) in fp32 and anchors
  (B, H, capacity, D) in the stream dtype; README "dtype contracts": the
  deltas are always fp32.
* README, "Materialization-free decode attention": the coefficient-domain
  decode also covers this tier (numerically supported, no byte saving).
* README, mode table and "Cache footprint & latency": the tier is lossless
  at keep_ratio = 1.0 and costs 188 % of bf16 KV (100 % of fp32 KV).

Readings where the pages are silent:
* Only the lossless tier (keep_ratio = 1.0) is modelled: the Top-M filter
  used below 1.0 is named on the pages but never defined.
* The stored delta is the exact difference of the two stored token values,
  rounded once to fp32 (nearest even).
* The per-block rows [x_0, Delta_1, ..., Delta_{r-1}] take the place of the
  DCT coefficients, with the synthesis A[t, j] = 1 for j <= t and 0
  otherwise (x_t = sum_j A[t, j] row_j): decode attention then takes the
  same per-block steps as the DCT tier with this A and S = R.
"""

from __future__ import annotations

import numpy as np

from .attention import _fresh_state, _online_blocks, _online_tail, \
    combine_partials
from .codec import round_to_dtype, split_blocks

F64 = np.float64


def png_filter(X: np.ndarray, R: int):
    """Anchors (B, H, nb, D), exact deltas (B, H, nb, R - 1, D) of every
    complete block of X (B, H, T, D), and the raw tail."""
    blocks, tail = split_blocks(X, R)
    anchors = blocks[:, :, :, 0, :].copy()
    deltas = blocks[:, :, :, 1:, :] - blocks[:, :, :, :-1, :]
    return anchors, deltas, tail


def png_store(deltas: np.ndarray) -> np.ndarray:
    """Deltas as the archive stores them: fp32, as float64 values."""
    return round_to_dtype(deltas, "f32")


def png_reconstruct(anchors: np.ndarray, deltas: np.ndarray) -> np.ndarray:
    """x_0 = anchor, x_i = x_{i-1} + Delta_i, block by block:
    (B, H, nb, D), (B, H, nb, R - 1, D) -> (B, H, nb * R, D)."""
    anchors = np.asarray(anchors, dtype=F64)
    deltas = np.asarray(deltas, dtype=F64)
    B, H, nb, Rm1, D = deltas.shape
    out = np.empty((B, H, nb, Rm1 + 1, D))
    out[:, :, :, 0] = anchors
    for i in range(1, Rm1 + 1):
        out[:, :, :, i] = out[:, :, :, i - 1] + deltas[:, :, :, i - 1]
    return out.reshape(B, H, nb * (Rm1 + 1), D)


def png_synthesis(R: int) -> np.ndarray:
    """A (R, R): A[t, j] = 1 for j <= t, else 0."""
    return np.tril(np.ones((R, R), dtype=F64))


def png_rows(anchors: np.ndarray, deltas: np.ndarray) -> np.ndarray:
    """Per-block rows [anchor, Delta_1, ..., Delta_{R-1}]: (B, H, nb, R, D)."""
    return np.concatenate([np.asarray(anchors, dtype=F64)[:, :, :, None, :],
                           np.asarray(deltas, dtype=F64)], axis=3)


def png_storage_bytes(B: int, H: int, nb: int, R: int, D: int,
                      in_dtype: str, tail_len: int = 0) -> int:
    """Live bytes of one stream: fp32 deltas and input-dtype anchors per
    archived block, plus the raw tail at the input precision."""
    esz = {"f32": 4, "bf16": 2}[in_dtype]
    per_block = (R - 1) * D * 4 + D * esz
    return B * H * (nb * per_block + tail_len * D * esz)


def _attend(q, K, V, scale):
    """softmax(scale q . K^T) V per query head; head hq reads kv head hq // G."""
    B, Hq, _, D = q.shape
    G = Hq // K.shape[1]
    sc = D ** -0.5 if scale is None else float(scale)
    Kx = np.repeat(K, G, axis=1)
    Vx = np.repeat(V, G, axis=1)
    logits = sc * np.einsum("bhd,bhtd->bht", q[:, :, 0, :], Kx)
    logits -= logits.max(axis=-1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=-1, keepdims=True)
    return np.einsum("bht,bhtd->bhd", p, Vx)[:, :, None, :]


def png_decode_attention_reference(q, anchors_k, deltas_k, anchors_v,
                                   deltas_v, tail_k, tail_v, R, scale=None):
    """Reconstruct every archived token by the cumulative sum, append the raw
    tail, then plain softmax attention (the definition)."""
    q = np.asarray(q, dtype=F64)
    K = png_reconstruct(anchors_k, deltas_k)
    V = png_reconstruct(anchors_v, deltas_v)
    if tail_k is not None and tail_k.shape[-2] > 0:
        K = np.concatenate([K, np.asarray(tail_k, dtype=F64)], axis=-2)
        V = np.concatenate([V, np.asarray(tail_v, dtype=F64)], axis=-2)
    if q.shape[1] % K.shape[1]:
        raise ValueError("Hq must be a multiple of Hk")
    if K.shape[-2] == 0:
        raise ValueError("decode attention needs at least one token")
    return _attend(q, K, V, scale)


def _heads(q, anchors_k, deltas_k, anchors_v, deltas_v, tail_k, tail_v,
           R, scale, first, last):
    """Per (b, kv head) online-softmax state over blocks [first, last) in the
    row domain, plus the tail when ``last`` is the block count."""
    q = np.asarray(q, dtype=F64)
    Ck = png_rows(anchors_k, deltas_k)
    Cv = png_rows(anchors_v, deltas_v)
    B, Hq, _, D = q.shape
    Hk, nb = Ck.shape[1], Ck.shape[2]
    G = Hq // Hk
    A = png_synthesis(R)
    sc = D ** -0.5 if scale is None else float(scale)
    states = {}
    for b in range(B):
        for h in range(Hk):
            qg = q[b, h * G:(h + 1) * G, 0, :]
            m, l, acc = _fresh_state(G, D)
            m, l, acc = _online_blocks(qg, Ck[b, h, first:last],
                                       Cv[b, h, first:last], A, sc, m, l, acc)
            if last == nb and tail_k is not None and tail_k.shape[-2] > 0:
                m, l, acc = _online_tail(qg, np.asarray(tail_k[b, h], F64),
                                         np.asarray(tail_v[b, h], F64), sc,
                                         m, l, acc)
            states[(b, h)] = (m, l, acc)
    return states, (B, Hq, D, G, Hk)


def png_coeff_decode_attention(q, anchors_k, deltas_k, anchors_v, deltas_v,
                               tail_k, tail_v, R, scale=None):
    """Decode attention on the stored rows, block by block (s = rows_k q,
    logits = scale A s, online softmax, w = p A, acc += w rows_v), the raw
    tail folded into the same softmax."""
    nb = np.asarray(deltas_k).shape[2]
    states, (B, Hq, D, G, Hk) = _heads(q, anchors_k, deltas_k, anchors_v,
                                       deltas_v, tail_k, tail_v, R, scale,
                                       0, nb)
    out = np.empty((B, Hq, 1, D))
    for (b, h), (m, l, acc) in states.items():
        out[b, h * G:(h + 1) * G, 0, :] = acc / l[:, None]
    return out


def png_splitk_decode_attention(q, anchors_k, deltas_k, anchors_v, deltas_v,
                                tail_k, tail_v, R, num_splits, scale=None):
    """The row-domain pass over contiguous block chunks (the tail in the last
    chunk), each leaving (max, sum, acc), merged by the combine."""
    nb = np.asarray(deltas_k).shape[2]
    q = np.asarray(q, dtype=F64)
    B, Hq, _, D = q.shape
    ns = max(1, int(num_splits))
    chunk = -(-nb // ns) if nb else 0
    M = np.full((B, Hq, ns), -np.inf)
    L = np.zeros((B, Hq, ns))
    ACC = np.zeros((B, Hq, ns, D))
    for c in range(ns):
        first = min(c * chunk, nb)
        last = min((c + 1) * chunk, nb) if c < ns - 1 else nb
        has_tail = c == ns - 1
        states, (_, _, _, G, Hk) = _heads(
            q, anchors_k, deltas_k, anchors_v, deltas_v,
            tail_k if has_tail else None, tail_v if has_tail else None,
            R, scale, first, last)
        for (b, h), (m, l, acc) in states.items():
            M[b, h * G:(h + 1) * G, c] = m
            L[b, h * G:(h + 1) * G, c] = l
            ACC[b, h * G:(h + 1) * G, c] = acc
    return combine_partials(M, L, ACC)
