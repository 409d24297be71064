"""Pins for the fp64 oracle's codec (basis, compress, quantiser, storage).

Each check ties the oracle to something other than itself: scipy's DCT-II,
closed forms, brute-force bounds, and the storage numbers the flashcodec-kv
README prints.
"""

import json
import os
from decimal import Decimal, ROUND_HALF_UP

import numpy as np
import pytest
import scipy.fft
import torch

import oracle
from oracle import codec
from oracle.stream import CodecStreamOracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("R", [2, 4, 8, 16, 32])
def test_basis_matches_scipy_dct_ii(R):
    """Full basis (S = R) applied to a block equals scipy's orthonormal
    DCT-II along the token axis; truncation keeps its first S rows."""
    rng = np.random.default_rng(R)
    X = rng.standard_normal((R, 7))
    M = codec.dct_basis(R, R)
    ref = scipy.fft.dct(X, type=2, norm="ortho", axis=0)
    np.testing.assert_allclose(M @ X, ref, atol=1e-13, rtol=0)
    for S in range(1, R + 1):
        np.testing.assert_allclose(codec.dct_basis(R, S) @ X, ref[:S],
                                   atol=1e-13, rtol=0)


@pytest.mark.parametrize("R,S", [(8, 2), (8, 8), (16, 4), (16, 16), (5, 3)])
def test_basis_rows_orthonormal(R, S):
    M = codec.dct_basis(R, S)
    np.testing.assert_allclose(M @ M.T, np.eye(S), atol=1e-14)
    if S == R:
        np.testing.assert_allclose(M.T @ M, np.eye(R), atol=1e-14)
    np.testing.assert_array_equal(codec.synthesis_basis(R, S), M.T)


@pytest.mark.parametrize("R", [2, 4, 8, 16, 32])
def test_basis_rows_are_mirror_symmetric(R):
    """M[j, R-1-n] = (-1)^j M[j, n] (cos(pi j - x) = (-1)^j cos x): the
    identity behind the device encoder's and attention kernel's folded sums
    (rows t < R/2 on x_t + x_{R-1-t} for even j, x_t - x_{R-1-t} for odd j).
    Checked against scipy's DCT-II matrix, and the folded coefficients
    against the plain product on random blocks."""
    M = scipy.fft.dct(np.eye(R), type=2, norm="ortho", axis=0)   # (R, R)
    sign = (-1.0) ** np.arange(R)[:, None]
    np.testing.assert_allclose(M[:, ::-1], sign * M, atol=1e-15)
    ours = codec.dct_basis(R, R)
    np.testing.assert_allclose(ours[:, ::-1], sign * ours, atol=1e-15)
    x = np.random.default_rng(R).standard_normal((R, 7))
    h = R // 2
    u, w = x[:h] + x[::-1][:h], x[:h] - x[::-1][:h]
    folded = np.where(np.arange(R)[:, None] % 2 == 0, ours[:, :h] @ u,
                      ours[:, :h] @ w)
    np.testing.assert_allclose(folded, ours @ x, atol=1e-13)


def test_constant_block_has_only_dc():
    R, S, D = 8, 4, 3
    x = np.array([1.5, -2.0, 0.25])
    X = np.broadcast_to(x, (1, 1, R, D)).copy()
    C, tail = codec.compress(X, R, S)
    assert tail.shape == (1, 1, 0, D)
    np.testing.assert_allclose(C[0, 0, 0, 0], np.sqrt(R) * x, atol=1e-14)
    np.testing.assert_allclose(C[0, 0, 0, 1:], 0.0, atol=1e-14)


def test_basis_row_maps_to_unit_vector():
    """A block whose tokens follow basis row j has coefficients e_j."""
    R, S = 16, 16
    M = codec.dct_basis(R, S)
    for j in range(S):
        X = M[j][None, None, :, None]          # (1, 1, R, 1)
        C, _ = codec.compress(X, R, S)
        e = np.zeros(S)
        e[j] = 1.0
        np.testing.assert_allclose(C[0, 0, 0, :, 0], e, atol=1e-14)


@pytest.mark.parametrize("R", [4, 8, 16])
def test_full_basis_round_trip_is_lossless(R):
    rng = np.random.default_rng(7)
    X = rng.standard_normal((2, 3, 5 * R, 16))
    C, tail = codec.compress(X, R, R)
    Xh = codec.decompress(C, R)
    assert np.max(np.abs(Xh - X)) <= 1e-12


def test_reconstruction_error_monotone_in_kept_frequencies():
    R = 8
    rng = np.random.default_rng(3)
    X = np.cumsum(rng.standard_normal((1, 2, 64 * R, 8)), axis=2)
    errs = []
    for S in range(1, R + 1):
        C, _ = codec.compress(X, R, S)
        errs.append(np.sum((codec.decompress(C, R) - X) ** 2))
    assert all(a >= b - 1e-9 for a, b in zip(errs, errs[1:]))
    assert errs[-1] < 1e-20


def test_split_blocks_indexing():
    X = np.arange(2 * 1 * 19 * 1, dtype=float).reshape(2, 1, 19, 1)
    blocks, tail = codec.split_blocks(X, 8)
    assert blocks.shape == (2, 1, 2, 8, 1) and tail.shape == (2, 1, 3, 1)
    assert blocks[1, 0, 1, 0, 0] == 19 + 8 and tail[0, 0, 0, 0] == 16


# ---------------------------------------------------------------- quantiser

def test_quantiser_hand_worked_rows():
    C = np.array([
        [127.0, -63.5, 0.2, 0.0],      # scale 1: half-even sends -63.5 to -64
        [254.0, 1.0, 3.0, -5.0],       # scale 2: 0.5 -> 0, 1.5 -> 2, -2.5 -> -2
        [-2.5, 1.0, 0.5, 0.0],         # scale 2.5/127
        [0.0, 0.0, 0.0, 0.0],          # all-zero row: scale 0, codes 0
    ])
    codes, scale, y = codec.quantize(C)
    np.testing.assert_allclose(scale[:, 0], [1.0, 2.0, 2.5 / 127, 0.0])
    np.testing.assert_array_equal(codes[0], [127, -64, 0, 0])
    np.testing.assert_array_equal(codes[1], [127, 0, 2, -2])
    np.testing.assert_array_equal(codes[2], [-127, 51, 25, 0])
    np.testing.assert_array_equal(codes[3], [0, 0, 0, 0])
    assert codes.dtype == np.int8


def test_quantiser_error_bound_and_extremes():
    rng = np.random.default_rng(11)
    C = rng.standard_normal((500, 64)) * rng.exponential(3.0, (500, 1))
    codes, scale, y = codec.quantize(C)
    rec = codes.astype(float) * scale
    assert np.all(np.abs(C - rec) <= scale / 2 + 1e-12)
    assert np.all(np.abs(codes) <= 127)
    arg = np.argmax(np.abs(C), axis=1)
    np.testing.assert_array_equal(
        np.abs(codes[np.arange(500), arg]).astype(int), 127)
    np.testing.assert_allclose(scale[:, 0], np.max(np.abs(C), axis=1) / 127)


def test_quantiser_fp32_decision_matches_fp64_off_half_integers():
    rng = np.random.default_rng(5)
    C = rng.standard_normal((2000, 128)) * 3
    c64, s64, y64 = codec.quantize(C, decision="f64")
    c32, s32, y32 = codec.quantize(C, decision="f32")
    frac = np.abs(np.abs(y64 - np.floor(y64)) - 0.5)
    near = frac < 1e-5
    diff = c64.astype(int) - c32.astype(int)
    assert np.all(diff[~near] == 0)
    assert np.all(np.abs(diff[near]) <= 1)
    np.testing.assert_allclose(s32, s64.astype(np.float32), rtol=1e-6)


def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(100000) * 10).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(codec.round_to_dtype(x, "bf16"), ref)
    np.testing.assert_array_equal(codec.round_to_dtype(x, "f32"),
                                  x.astype(np.float64))


# ----------------------------------------------------------------- storage

def _half_up(x, digits):
    q = Decimal(1).scaleb(-digits)
    return str(Decimal(repr(x)).quantize(q, rounding=ROUND_HALF_UP))


def test_storage_footprint_table():
    with open(os.path.join(GOLDEN, "storage_footprint.json")) as f:
        gold = json.load(f)
    B, H, D, R = 1, 8, 64, 8
    for row in gold["rows"]:
        seq, keep = row["seq"], row["keep"]
        coeff = "i8" if row["quant_bits"] == 8 else "f32"
        total = 0
        for _ in ("k", "v"):
            st = CodecStreamOracle(R, keep, coeff, in_dtype="f32")
            # storage only depends on shapes: zero tokens keep this cheap
            st.append(np.zeros((B, H, seq, D)))
            total += st.storage_bytes()
        raw = seq * B * H * D * 4 * 2
        assert _half_up(total / 2 ** 20, 1) == row["storage"], row
        assert _half_up(total / raw, 2) == row["ratio"], row


def test_storage_ratio_table():
    with open(os.path.join(GOLDEN, "storage_ratio.json")) as f:
        gold = json.load(f)
    D, R = 64, 8
    for row in gold["rows"]:
        coeff = "i8" if row["quant_bits"] == 8 else "f32"
        per_block = codec.storage_bytes_per_block(row["keep"], D, coeff)
        pct = 100.0 * per_block / (R * D * 4)
        assert _half_up(pct, 1) == row["storage_pct"], row


def test_reconstruction_quality_ordering_unpinned():
    """Loose sanity band for the README's PSNR table (its random walk is not
    defined on the pages, so parity here is unpinned): error falls with the
    kept frequencies, and int8 costs a little on top of truncation."""
    rng = np.random.default_rng(0)
    X = np.cumsum(rng.standard_normal((2, 8, 2048, 64)), axis=2)
    X /= np.max(np.abs(X))

    def psnr(keep, q):
        enc = codec.encode_stream(X, 8, keep, "i8" if q else "f64")
        Xh = codec.decompress(enc["C_hat"], 8)
        return 10 * np.log10(1.0 / np.mean((Xh - X) ** 2))

    order = [psnr(1, False), psnr(2, True), psnr(2, False), psnr(4, True),
             psnr(4, False)]
    assert all(a < b for a, b in zip(order, order[1:])), order
