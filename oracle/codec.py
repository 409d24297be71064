"""fp64 oracle: JPEG-style block codec along the sequence axis.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources (flashcodec-kv 1.0.0):
* README, "Math": a block X (r x D) is encoded as C = M X with
  M[j, n] = c_j cos(pi/r (n + 1/2) j), the encoder matrix has orthonormal rows
  (keeping all r rows is lossless per block) and the reconstruction is M^T C.
* README, mode table and the ``quant_bits=8`` paragraph: the lowest K
  frequencies are kept; int8 storage uses one scale per (block, frequency).
* ``flashcodec/cache.py``, ``_CodecStream`` docstring and ``_archive_spec``:
  coefficients are (B, H, capacity, K, D), int8 codes come with fp32 scales of
  shape (B, H, capacity, K, 1); unquantised coefficients keep the stream dtype.
* ``flashcodec/cache.py``, ``_CodecStream.append``: only complete blocks are
  archived; the remainder stays raw.

Readings where the pages are silent:
* c_0 = sqrt(1/R), c_j = sqrt(2/R): the normalisation that makes the rows
  orthonormal, i.e. the standard orthonormal DCT-II.
* scale = max_d |C| / 127, code = clamp(round_half_even(C / scale), -127, 127);
  an all-zero (block, frequency) row gets scale 0 and codes 0.
"""

from __future__ import annotations

import numpy as np

F64 = np.float64


def dct_basis(R: int, S: int) -> np.ndarray:
    """Encoder rows M (S, R): M[j, n] = c_j cos(pi/R (n + 1/2) j).

    README "Math" (JPEG bullet); c_j is the orthonormal DCT-II normalisation.
    """
    if not (1 <= S <= R):
        raise ValueError("need 1 <= S <= R")
    n = np.arange(R, dtype=F64)[None, :]
    j = np.arange(S, dtype=F64)[:, None]
    c = np.where(j == 0, np.sqrt(1.0 / R), np.sqrt(2.0 / R))
    return c * np.cos(np.pi / R * (n + 0.5) * j)


def synthesis_basis(R: int, S: int) -> np.ndarray:
    """A (R, S) = M^T: block tokens are A @ C (README, "Materialization-free
    decode attention": K_block = A @ S with A the synthesis matrix)."""
    return dct_basis(R, S).T.copy()


def split_blocks(X: np.ndarray, R: int):
    """Split (B, H, T, D) into complete blocks (B, H, nb, R, D) and the raw
    tail (B, H, T - nb R, D), nb = floor(T / R) (``_CodecStream.append``)."""
    X = np.asarray(X, dtype=F64)
    B, H, T, D = X.shape
    nb = T // R
    blocks = X[:, :, : nb * R, :].reshape(B, H, nb, R, D)
    tail = X[:, :, nb * R:, :]
    return blocks, tail


def compress(X: np.ndarray, R: int, S: int):
    """C[b, h, n, j, :] = sum_t M[j, t] X[b, h, nR + t, :] for every complete
    block; returns (C (B, H, nb, S, D), raw tail)."""
    blocks, tail = split_blocks(X, R)
    M = dct_basis(R, S)
    C = np.einsum("jt,bhntd->bhnjd", M, blocks)
    return C, tail


def quantize(C: np.ndarray, decision: str = "f64"):
    """int8 codes with one scale per (block, frequency), taken over D.

    Returns ``(codes int8, scale fp64, y)`` where ``y = C / scale`` is the
    pre-rounding value (0 for an all-zero row). ``decision='f64'`` divides in
    float64, the precision the GPU kernel takes the decision in;
    ``decision='f32'`` rounds C and the scale to float32 first and divides in
    float32, an alternative reading used only to bound how far the two
    precisions can disagree.
    The stored scale is ``float32(scale)`` in both cases.
    """
    C = np.asarray(C, dtype=F64)
    amax = np.max(np.abs(C), axis=-1, keepdims=True)
    if decision == "f64":
        scale = amax / 127.0
        safe = np.where(scale > 0, scale, 1.0)
        y = np.where(scale > 0, C / safe, 0.0)
    elif decision == "f32":
        c32 = C.astype(np.float32)
        amax32 = np.max(np.abs(c32), axis=-1, keepdims=True)
        s32 = (amax32 / np.float32(127.0)).astype(np.float32)
        safe = np.where(s32 > 0, s32, np.float32(1.0)).astype(np.float32)
        y32 = np.where(s32 > 0, (c32 / safe).astype(np.float32),
                       np.float32(0.0))
        scale = s32.astype(F64)
        y = y32.astype(F64)
    else:
        raise ValueError(decision)
    codes = np.clip(np.rint(y), -127, 127).astype(np.int8)  # rint: half-even
    return codes, scale, y


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """C_hat = code * scale (scale broadcast over D)."""
    s = np.asarray(scales, dtype=F64)
    if s.ndim == codes.ndim - 1:
        s = s[..., None]
    return codes.astype(F64) * s


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype with round-to-nearest-even
    and return them as float64 ("f32", "bf16" or "f64")."""
    x = np.asarray(x, dtype=F64)
    if dtype == "f64":
        return x.copy()
    if dtype == "f32":
        return x.astype(np.float32).astype(F64)
    if dtype == "bf16":
        # 8 significant bits: m in [0.5, 1) -> 256 m rounded half-even
        m, e = np.frexp(x)
        return np.ldexp(np.rint(m * 256.0), e - 8)
    raise ValueError(dtype)


def decompress(C_hat: np.ndarray, R: int) -> np.ndarray:
    """X_hat = M^T C per block, (B, H, nb, S, D) -> (B, H, nb R, D)."""
    C_hat = np.asarray(C_hat, dtype=F64)
    B, H, nb, S, D = C_hat.shape
    M = dct_basis(R, S)
    X = np.einsum("jt,bhnjd->bhntd", M, C_hat)
    return X.reshape(B, H, nb * R, D)


def storage_bytes_per_block(S: int, D: int, coeff: str) -> int:
    """Bytes one archived block occupies per (batch, head) in the live region
    (``_CodecStream.storage_bytes``: coefficient tensors, plus the fp32
    scales of shape (..., K, 1) when quantised)."""
    if coeff == "i8":
        return S * D * 1 + S * 4
    if coeff == "bf16":
        return S * D * 2
    if coeff == "f32":
        return S * D * 4
    raise ValueError(coeff)


def encode_stream(X: np.ndarray, R: int, S: int, coeff: str,
                  decision: str = "f64"):
    """Archive every complete block of X (B, H, T, D) the way the codec
    stores it.

    Returns a dict: ``C_hat`` (the coefficients the archive holds, as float64:
    code * fp32 scale for "i8", else C rounded to the stream dtype),
    ``codes``/``scales``/``y`` (for "i8"; scales as float32), ``C`` (exact
    coefficients) and ``tail`` (raw tokens).
    """
    C, tail = compress(X, R, S)
    out = {"C": C, "tail": tail}
    if coeff == "i8":
        codes, scale, y = quantize(C, decision=decision)
        s32 = scale[..., 0].astype(np.float32)
        out.update(codes=codes, scales=s32, y=y,
                   C_hat=dequantize(codes, s32))
    else:
        out["C_hat"] = round_to_dtype(C, coeff)
    return out
