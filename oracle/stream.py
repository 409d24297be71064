"""fp64 oracle: one K or V stream of the codec cache (raw tail + archive).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows ``flashcodec/cache.py`` ``_CodecStream``:
* ``append(tokens)`` concatenates the raw tail and the new tokens, archives
  every complete block of the concatenation (``_archive``), and keeps the
  remainder raw (causal safety: only complete blocks are ever archived, and an
  archived block is never written again).
* the archive capacity starts at 16 blocks and doubles until it covers the
  need; growing copies the live prefix verbatim (``_grow``).
* ``storage_bytes`` counts the live archive region plus the raw tail, not the
  idle capacity.
* ``read`` is the reconstructed view: every archived block decompressed
  (X_hat = M^T C_hat) and restored to the stream input dtype, followed by the
  raw tail (``_CodecStream.read`` and ``_decode_pending``).
* ``crop`` removes trailing tokens exactly: archived blocks below the new
  boundary are kept verbatim and the partial block at the boundary comes back
  as raw tail tokens taken from the reconstruction (``_CodecStream.crop``).
* ``select_batch`` gathers the batch axis of the archive and the raw tail
  (``_CodecStream.select_batch``; beam reorder, repeat and selection of rows);
  ``reset`` empties the stream and keeps its capacity (``_CodecStream.reset``).
"""

from __future__ import annotations

import numpy as np

from .codec import compress, quantize, round_to_dtype, dequantize, decompress

INITIAL_BLOCKS = 16


def grown_capacity(capacity: int, need: int) -> int:
    """Capacity after ``_grow(need)``: unchanged if it suffices, else the
    smallest 16 * 2^k >= need."""
    if need <= capacity:
        return capacity
    cap = INITIAL_BLOCKS
    while cap < need:
        cap *= 2
    return cap


class CodecStreamOracle:
    """One (B, H, T, D) stream. ``coeff`` is "i8", "f32" or "bf16";
    ``in_dtype`` is the token dtype ("f32" or "bf16") used for the raw tail
    byte count."""

    def __init__(self, R: int, S: int, coeff: str, in_dtype: str = "f32",
                 decision: str = "f64"):
        self.R, self.S, self.coeff = R, S, coeff
        self.in_dtype = in_dtype
        self.decision = decision
        self.raw = None            # (B, H, t < R, D) float64
        self.n_blocks = 0
        self.capacity = 0
        self.codes = None          # (B, H, cap, S, D) int8
        self.scales = None         # (B, H, cap, S) float32
        self.coeffs = None         # (B, H, cap, S, D) float64 (unquantised)
        self.pre_round = None      # (B, H, cap, S, D) float64 C / scale

    # -- archive -----------------------------------------------------------
    def _grow(self, need, B, H, D):
        cap = grown_capacity(self.capacity, need)
        if cap == self.capacity:
            return
        nb = self.n_blocks

        def regrow(old, shape, dtype):
            new = np.zeros(shape, dtype=dtype)
            if old is not None and nb:
                new[:, :, :nb] = old[:, :, :nb]
            return new

        if self.coeff == "i8":
            self.codes = regrow(self.codes, (B, H, cap, self.S, D), np.int8)
            self.scales = regrow(self.scales, (B, H, cap, self.S),
                                 np.float32)
            self.pre_round = regrow(self.pre_round, (B, H, cap, self.S, D),
                                    np.float64)
        else:
            self.coeffs = regrow(self.coeffs, (B, H, cap, self.S, D),
                                 np.float64)
        self.capacity = cap

    def _archive(self, head):
        B, H, n, D = head.shape
        n_full = n // self.R
        self._grow(self.n_blocks + n_full, B, H, D)
        C, _ = compress(head, self.R, self.S)
        sl = slice(self.n_blocks, self.n_blocks + n_full)
        if self.coeff == "i8":
            codes, scale, y = quantize(C, decision=self.decision)
            self.codes[:, :, sl] = codes
            self.scales[:, :, sl] = scale[..., 0].astype(np.float32)
            self.pre_round[:, :, sl] = y
        else:
            self.coeffs[:, :, sl] = round_to_dtype(C, self.coeff)
        self.n_blocks += n_full

    def append(self, tokens):
        """Append (B, H, m, D) tokens; archive every complete block."""
        tokens = np.asarray(tokens, dtype=np.float64)
        buf = tokens if self.raw is None else np.concatenate(
            [self.raw, tokens], axis=-2)
        total = buf.shape[-2]
        n_full = total // self.R
        if n_full:
            self._archive(buf[:, :, : n_full * self.R])
        rest = buf[:, :, n_full * self.R:]
        self.raw = rest.copy() if rest.shape[-2] else None

    # -- views ---------------------------------------------------------------
    @property
    def tail_len(self) -> int:
        return 0 if self.raw is None else self.raw.shape[-2]

    @property
    def seq_len(self) -> int:
        return self.n_blocks * self.R + self.tail_len

    def C_hat(self) -> np.ndarray:
        """Live archived coefficients as float64 (B, H, n_blocks, S, D)."""
        nb = self.n_blocks
        if self.coeff == "i8":
            return dequantize(self.codes[:, :, :nb], self.scales[:, :, :nb])
        return self.coeffs[:, :, :nb]

    def tail(self, B, H, D) -> np.ndarray:
        if self.raw is None:
            return np.zeros((B, H, 0, D))
        return self.raw

    def storage_bytes(self) -> int:
        """Live archive region + raw tail (``_CodecStream.storage_bytes``)."""
        elem = {"f32": 4, "bf16": 2, "i8": 1}
        total = 0
        if self.n_blocks:
            if self.coeff == "i8":
                live = self.codes[:, :, : self.n_blocks]
                total += live.size * 1 + live[..., 0].size * 4
            else:
                live = self.coeffs[:, :, : self.n_blocks]
                total += live.size * elem[self.coeff]
        if self.raw is not None:
            total += self.raw.size * elem[self.in_dtype]
        return total

    # -- structural operations -----------------------------------------------
    def read(self) -> np.ndarray:
        """Reconstructed (B, H, seq_len, D) view as float64 values of the input
        dtype: the archived blocks decompressed and rounded to ``in_dtype``,
        then the raw tail as stored. ``None`` for an empty stream."""
        parts = []
        if self.n_blocks:
            parts.append(round_to_dtype(decompress(self.C_hat(), self.R),
                                        self.in_dtype))
        if self.raw is not None:
            parts.append(self.raw)
        if not parts:
            return None
        return np.concatenate(parts, axis=-2) if len(parts) > 1 else \
            parts[0].copy()

    def crop(self, tokens_to_remove: int) -> None:
        """Drop the last ``-tokens_to_remove`` tokens (the pages' convention:
        a negative count; a positive one is an error, zero does nothing)."""
        if tokens_to_remove > 0:
            raise ValueError("crop takes a negative count of tokens to remove")
        if tokens_to_remove == 0:
            return
        keep = max(0, self.seq_len - abs(int(tokens_to_remove)))
        keep_blocks, rest = divmod(keep, self.R)
        if keep_blocks < self.n_blocks:
            # the boundary block's first `rest` tokens, as the view holds them
            view = self.read()
            self.n_blocks = keep_blocks
            self.raw = view[:, :, keep_blocks * self.R:keep].copy() \
                if rest else None
        elif rest == 0:
            self.raw = None
        else:
            self.raw = self.raw[:, :, :rest].copy()

    def select_batch(self, idx) -> None:
        """Batch row i of the result is row ``idx[i]`` of the current stream
        (the live archive region and the raw tail); indices may repeat and
        their count may differ from B. The capacity is kept."""
        idx = np.asarray(idx, dtype=np.int64).reshape(-1)
        nb = self.n_blocks

        def gather(a):
            if a is None:
                return None
            out = np.zeros((idx.size,) + a.shape[1:], dtype=a.dtype)
            if nb:
                out[:, :, :nb] = a[idx][:, :, :nb]
            return out

        self.codes = gather(self.codes)
        self.scales = gather(self.scales)
        self.pre_round = gather(self.pre_round)
        self.coeffs = gather(self.coeffs)
        if self.raw is not None:
            self.raw = self.raw[idx].copy()

    def reset(self) -> None:
        """Empty the stream; the archive keeps its capacity."""
        self.raw = None
        self.n_blocks = 0
