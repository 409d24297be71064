"""Pins for the oracle's decode attention.

The three oracle paths (decompress-then-softmax, coefficient domain, split-K +
combine) are checked against each other by brute force, against torch's
scaled_dot_product_attention (a library routine) where the codec is lossless,
and against closed forms.
"""

import numpy as np
import pytest
import torch

from oracle import codec
from oracle.attention import (decode_attention_reference,
                              coeff_decode_attention, split_partials,
                              combine_partials, splitk_decode_attention,
                              attend_archive)


def _case(B=2, Hk=2, G=2, D=16, nb=5, nr=3, R=8, S=3, coeff="i8", seed=0,
          rho=0.9):
    rng = np.random.default_rng(seed)
    T = nb * R + nr
    eps = rng.standard_normal((B, Hk, T, D))
    X = np.zeros_like(eps)
    Y = np.zeros_like(eps)
    epv = rng.standard_normal((B, Hk, T, D))
    for t in range(T):
        X[:, :, t] = (rho * X[:, :, t - 1] if t else 0) + eps[:, :, t]
        Y[:, :, t] = (rho * Y[:, :, t - 1] if t else 0) + epv[:, :, t]
    q = rng.standard_normal((B, Hk * G, 1, D))
    ek = codec.encode_stream(X, R, S, coeff)
    ev = codec.encode_stream(Y, R, S, coeff)
    return dict(q=q, X=X, Y=Y, Ck=ek["C_hat"], Cv=ev["C_hat"],
                tk=ek["tail"], tv=ev["tail"], R=R, S=S)


@pytest.mark.parametrize("coeff", ["i8", "f64"])
@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("nr", [0, 3])
def test_three_paths_agree(coeff, G, nr):
    c = _case(G=G, nr=nr, coeff=coeff, seed=G + 10 * nr)
    args = (c["q"], c["Ck"], c["Cv"], c["tk"], c["tv"], c["R"])
    ref = decode_attention_reference(*args)
    co = coeff_decode_attention(*args)
    assert np.max(np.abs(co - ref)) <= 1e-12
    nb = c["Ck"].shape[2]
    for ns in (1, 2, 3, 7, nb, nb + 4):
        sk = splitk_decode_attention(*args, num_splits=ns)
        assert np.max(np.abs(sk - ref)) <= 1e-12, ns


def test_lossless_codec_equals_sdpa_on_raw_tokens():
    """S = R and no quantisation: coefficient-domain attention over the
    archive equals plain softmax attention on the raw K/V (torch SDPA)."""
    R, G = 8, 4
    c = _case(Hk=2, G=G, D=32, nb=6, nr=5, R=R, S=R, coeff="f64", seed=3)
    out = coeff_decode_attention(c["q"], c["Ck"], c["Cv"], c["tk"], c["tv"],
                                 R)
    q = torch.from_numpy(c["q"])
    K = torch.from_numpy(c["X"]).repeat_interleave(G, dim=1)
    V = torch.from_numpy(c["Y"]).repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, K, V).numpy()
    assert np.max(np.abs(out - ref)) <= 1e-12
    # same through the GQA flag of the library routine
    ref2 = torch.nn.functional.scaled_dot_product_attention(
        q, torch.from_numpy(c["X"]), torch.from_numpy(c["Y"]),
        enable_gqa=True).numpy()
    assert np.max(np.abs(out - ref2)) <= 1e-12


def test_explicit_softmax_scale():
    c = _case(G=2, nr=2, coeff="f64", seed=9)
    args = (c["q"], c["Ck"], c["Cv"], c["tk"], c["tv"], c["R"])
    for sc in (0.05, 0.3):
        a = decode_attention_reference(*args, scale=sc)
        b = splitk_decode_attention(*args, num_splits=3, scale=sc)
        assert np.max(np.abs(a - b)) <= 1e-12
    # default scale is D**-0.5
    a = decode_attention_reference(*args)
    b = decode_attention_reference(*args, scale=c["q"].shape[-1] ** -0.5)
    np.testing.assert_array_equal(a, b)


def test_single_tail_token_returns_its_value():
    rng = np.random.default_rng(1)
    D = 8
    q = rng.standard_normal((1, 2, 1, D))
    tk = rng.standard_normal((1, 1, 1, D))
    tv = rng.standard_normal((1, 1, 1, D))
    empty = np.zeros((1, 1, 0, 2, D))
    for f in (decode_attention_reference, coeff_decode_attention):
        out = f(q, empty, empty, tk, tv, 8)
        np.testing.assert_allclose(out[0, :, 0], np.repeat(tv[0, :, 0], 2, 0),
                                   atol=1e-15)


def test_zero_query_gives_mean_of_reconstructed_values():
    c = _case(G=2, nr=3, coeff="i8", seed=4)
    q = np.zeros_like(c["q"])
    out = coeff_decode_attention(q, c["Ck"], c["Cv"], c["tk"], c["tv"],
                                 c["R"])
    Vh = np.concatenate([codec.decompress(c["Cv"], c["R"]), c["tv"]], axis=2)
    mean = np.repeat(Vh.mean(axis=2), 2, axis=1)
    np.testing.assert_allclose(out[:, :, 0], mean, atol=1e-13)


def test_dominant_logit_selects_one_token():
    """q aligned with one reconstructed key and scaled up: the output tends
    to that token's reconstructed value."""
    R, S, D = 8, 8, 16
    c = _case(B=1, Hk=1, G=1, D=D, nb=4, nr=0, R=R, S=S, coeff="f64", seed=6,
              rho=0.0)
    Kh = codec.decompress(c["Ck"], R)[0, 0]
    Vh = codec.decompress(c["Cv"], R)[0, 0]
    p = 13
    q = (Kh[p] / np.linalg.norm(Kh[p]) * 400.0)[None, None, None, :]
    out = coeff_decode_attention(q, c["Ck"], c["Cv"], c["tk"], c["tv"], R)
    logits = Kh @ q[0, 0, 0] / np.sqrt(D)
    assert np.argmax(logits) == p
    gap = logits[p] - np.max(np.delete(logits, p))
    assert gap > 60
    np.testing.assert_allclose(out[0, 0, 0], Vh[p], atol=1e-12)


def test_gqa_query_head_reads_kv_head_hq_div_G():
    """Only kv head 0 carries signal: query heads 0..G-1 see it, the others
    see kv head 1 (a zero value stream)."""
    c = _case(B=1, Hk=2, G=3, D=8, nb=3, nr=1, coeff="f64", seed=8)
    Cv = c["Cv"].copy()
    tv = c["tv"].copy()
    Cv[:, 1] = 0.0
    tv[:, 1] = 0.0
    out = coeff_decode_attention(c["q"], c["Ck"], Cv, c["tk"], tv, c["R"])
    assert np.all(np.abs(out[0, :3]).sum(axis=-1) > 0)
    np.testing.assert_array_equal(out[0, 3:], 0.0)


def test_combine_skips_empty_chunks():
    c = _case(G=2, nb=2, nr=0, coeff="i8", seed=12)
    args = (c["q"], c["Ck"], c["Cv"], c["tk"], c["tv"], c["R"])
    M, L, A = split_partials(*args, num_splits=5)
    assert np.all(L[..., 2:] == 0) and np.all(np.isneginf(M[..., 2:]))
    out = combine_partials(M, L, A)
    assert np.all(np.isfinite(out))
    ref = decode_attention_reference(*args)
    assert np.max(np.abs(out - ref)) <= 1e-12


def test_attend_archive_samples_match_full():
    c = _case(B=2, Hk=2, G=2, nb=4, nr=2, coeff="i8", seed=13)
    args = (c["q"], c["Ck"], c["Cv"], c["tk"], c["tv"], c["R"])
    ref = decode_attention_reference(*args)
    heads = [(0, 0), (1, 3), (1, 2)]
    got = attend_archive(*args, heads=heads)
    for b, hq in heads:
        np.testing.assert_allclose(got[(b, hq)], ref[b, hq, 0], atol=1e-14)
