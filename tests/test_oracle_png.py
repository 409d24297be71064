"""Pins for the oracle's PNG-style lossless tier: anchor + first differences
per block, cumulative-sum reconstruction, storage, and decode attention on
the stored rows (flashcodec-kv README "Math" PNG bullet, "dtype contracts",
"Materialization-free decode attention"; flashcodec/cache.py,
_CodecStream._archive_spec)."""

import json
import os
from decimal import Decimal, ROUND_HALF_UP

import numpy as np
import pytest
import torch

from oracle import png
from oracle.attention import decode_attention_reference

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _half_up(x, places):
    q = Decimal(1).scaleb(-places)
    return str(Decimal(repr(x)).quantize(q, ROUND_HALF_UP))


def _walk(B=2, H=3, T=45, D=16, seed=0, dtype=torch.bfloat16):
    rng = np.random.default_rng(seed)
    x = np.cumsum(rng.standard_normal((B, H, T, D)), axis=2)
    return torch.from_numpy(x).to(dtype).to(torch.float64).numpy()


def test_filter_of_constant_and_ramp_blocks():
    """A constant block has zero deltas; a linear ramp a + b t has every
    delta equal to b; the anchor is the first token."""
    R, D = 8, 5
    t = np.arange(2 * R, dtype=np.float64)[None, None, :, None]
    a = np.array([0.5, -2.0, 3.0, 0.0, 1.25])
    b = np.array([0.25, 1.0, -0.5, 2.0, 0.0])
    ramp = a + b * t                                # (1, 1, 16, 5)
    anchors, deltas, tail = png.png_filter(ramp, R)
    assert anchors.shape == (1, 1, 2, D) and deltas.shape == (1, 1, 2, R - 1, D)
    np.testing.assert_array_equal(anchors[0, 0, 0], a)
    np.testing.assert_array_equal(anchors[0, 0, 1], a + b * R)
    np.testing.assert_array_equal(deltas, np.broadcast_to(b, deltas.shape))
    const = np.broadcast_to(a, (1, 1, 3 * R + 2, D))
    anchors, deltas, tail = png.png_filter(const, R)
    assert not deltas.any() and tail.shape[-2] == 2


def test_synthesis_is_the_cumulative_sum():
    """A[t, j] = 1 for j <= t applied to [anchor, deltas] is numpy's cumsum
    of the rows, and png_reconstruct agrees with it."""
    X = _walk(T=40)
    anchors, deltas, _ = png.png_filter(X, 8)
    rows = png.png_rows(anchors, deltas)
    A = png.png_synthesis(8)
    via_a = np.einsum("tj,bhnjd->bhntd", A, rows)
    np.testing.assert_allclose(via_a, np.cumsum(rows, axis=3), rtol=0,
                               atol=1e-12)
    np.testing.assert_allclose(png.png_reconstruct(anchors, deltas),
                               via_a.reshape(X.shape), rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_lossless_round_trip(dtype):
    """fp32-stored deltas rebuild the stored tokens: exactly for bf16 inputs
    (the difference of two nearby bf16 values fits an fp32), within 1e-6 of
    the signal's magnitude for fp32 inputs (the README's lossless claim)."""
    X = _walk(T=8 * 30, seed=3, dtype=dtype)
    anchors, deltas, _ = png.png_filter(X, 8)
    rec = png.png_reconstruct(anchors, png.png_store(deltas))
    err = np.max(np.abs(rec - X))
    if dtype == torch.bfloat16:
        assert err == 0.0
    else:
        assert err <= 1e-6 * np.max(np.abs(X))


def test_storage_matches_the_pages():
    with open(os.path.join(GOLDEN, "png_storage.json")) as f:
        gold = json.load(f)
    B, H, D, R = 1, 8, 64, 8
    for row in gold["footprint"]["rows"]:
        seq = row["seq"]
        total = 2 * png.png_storage_bytes(B, H, seq // R, R, D, "f32")
        raw = 2 * B * H * seq * D * 4
        assert _half_up(total / 2 ** 20, 1) == row["storage"]
        assert _half_up(total / raw, 2) == row["ratio"]
    for row in gold["percent_of_raw"]["rows"]:
        r, dt = row["block_size"], row["in_dtype"]
        esz = {"bf16": 2, "f32": 4}[dt]
        pct = 100.0 * png.png_storage_bytes(1, 1, 1, r, D, dt) / (r * D * esz)
        assert _half_up(pct, 0) == row["pct"]
    # the raw tail counts at the input precision
    assert png.png_storage_bytes(2, 3, 4, 8, 16, "bf16", tail_len=5) - \
        png.png_storage_bytes(2, 3, 4, 8, 16, "bf16") == 2 * 3 * 5 * 16 * 2


def _case(T=8 * 12 + 5, R=8, G=2, seed=4):
    X, Y = _walk(T=T, seed=seed), _walk(T=T, seed=seed + 1)
    ak, dk, tk = png.png_filter(X, R)
    av, dv, tv = png.png_filter(Y, R)
    q = np.random.default_rng(seed).standard_normal((2, 3 * G, 1, 16))
    return q, (ak, png.png_store(dk), av, png.png_store(dv), tk, tv), X, Y


def test_row_domain_attention_equals_the_definition():
    q, arc, X, Y = _case()
    ref = png.png_decode_attention_reference(q, *arc, 8)
    got = png.png_coeff_decode_attention(q, *arc, 8)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    for ns in (1, 2, 3, 7, 12, 20):
        np.testing.assert_allclose(
            png.png_splitk_decode_attention(q, *arc, 8, ns), ref, rtol=0,
            atol=1e-12)


def test_lossless_tier_attention_is_plain_attention_on_the_tokens():
    """Textbook special case: the lossless tier attends exactly the stored
    tokens, i.e. torch's scaled_dot_product_attention on the raw K/V."""
    q, arc, X, Y = _case(seed=9)
    got = png.png_coeff_decode_attention(q, *arc, 8, scale=0.3)
    G = q.shape[1] // X.shape[1]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(np.repeat(X, G, axis=1)),
        torch.from_numpy(np.repeat(Y, G, axis=1)), scale=0.3).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_closed_forms():
    """One tail token only: the output is that token's value. q = 0: the
    output is the mean of all value tokens."""
    R, D = 8, 16
    v_tok = np.arange(D, dtype=np.float64)[None, None, None, :]
    empty_a = np.zeros((1, 1, 0, D))
    empty_d = np.zeros((1, 1, 0, R - 1, D))
    q = np.ones((1, 2, 1, D))
    out = png.png_coeff_decode_attention(q, empty_a, empty_d, empty_a,
                                         empty_d, v_tok * 0.1, v_tok, R)
    np.testing.assert_allclose(out, np.broadcast_to(v_tok, out.shape),
                               atol=1e-15)
    Y = _walk(B=1, H=1, T=3 * R + 2, D=D, seed=5)
    X = _walk(B=1, H=1, T=3 * R + 2, D=D, seed=6)
    ak, dk, tk = png.png_filter(X, R)
    av, dv, tv = png.png_filter(Y, R)
    out = png.png_coeff_decode_attention(np.zeros((1, 1, 1, D)), ak, dk, av,
                                         dv, tk, tv, R)
    np.testing.assert_allclose(out[0, 0, 0], Y[0, 0].mean(axis=0),
                               rtol=0, atol=1e-12)


def test_png_and_full_dct_tiers_agree_when_lossless():
    """Both tiers are exact at full rank: the row-domain PNG attention equals
    the DCT tier's reference attention with S = R unquantised coefficients
    (two different synthesis matrices, one result)."""
    from oracle import codec
    q, arc, X, Y = _case(seed=11)
    R = 8
    ek = codec.encode_stream(X, R, R, "f64")
    ev = codec.encode_stream(Y, R, R, "f64")
    dct = decode_attention_reference(q, ek["C_hat"], ev["C_hat"], ek["tail"],
                                     ev["tail"], R)
    got = png.png_coeff_decode_attention(q, *arc, R)
    np.testing.assert_allclose(got, dct, rtol=0, atol=1e-12)
