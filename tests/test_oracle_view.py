"""Pins for the oracle's structural stream operations: the reconstructed view
(``read``), exact trailing-token removal (``crop``), batch gather
(``select_batch``) and ``reset`` (flashcodec/cache.py, ``_CodecStream``)."""

import numpy as np
import pytest
import torch

from oracle.attention import decode_attention_reference
from oracle.stream import CodecStreamOracle


def _tokens(B=3, H=2, T=77, D=16, seed=0):
    rng = np.random.default_rng(seed)
    return np.cumsum(rng.standard_normal((B, H, T, D)), axis=2)


def _as_dtype(x, dtype):
    """Round through torch's own cast (independent of the oracle's rounding)."""
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(tdt) \
        .to(torch.float64).numpy()


def _stream(X, R=8, S=2, coeff="i8", in_dtype="f32"):
    st = CodecStreamOracle(R, S, coeff, in_dtype)
    st.append(X)
    return st


# ---------------------------------------------------------------- read view

@pytest.mark.parametrize("in_dtype", ["f32", "bf16"])
def test_read_with_one_frequency_is_the_block_mean(in_dtype):
    """S = 1 keeps only the DC row c_0 = 1/sqrt(R): every token of a block
    reconstructs to the block's mean (a closed form), then the raw tail."""
    R = 8
    X = _as_dtype(_tokens(T=61, seed=1), in_dtype)
    st = _stream(X, R=R, S=1, coeff="f32", in_dtype=in_dtype)
    view = st.read()
    assert view.shape == X.shape
    nb = 61 // R
    mean = X[:, :, :nb * R].reshape(3, 2, nb, R, 16).mean(axis=3)
    want = np.repeat(mean, R, axis=2)
    got = view[:, :, :nb * R]
    # fp32 coefficient storage, then rounding to the view's dtype
    ulp = 2.0 ** -23 if in_dtype == "f32" else 2.0 ** -8
    assert np.all(np.abs(got - want) <= ulp * np.abs(want) + 1e-12)
    np.testing.assert_array_equal(view[:, :, nb * R:], X[:, :, nb * R:])
    # values are representable in the view's dtype
    np.testing.assert_array_equal(view, _as_dtype(view, in_dtype))


def test_read_with_every_frequency_is_lossless():
    """S = R unquantised: the orthonormal basis reconstructs each block (up to
    the fp32 storage of the coefficients)."""
    X = _as_dtype(_tokens(T=50, seed=2), "f32")
    st = _stream(X, R=8, S=8, coeff="f32")
    view = st.read()
    scale = np.max(np.abs(X))
    assert np.max(np.abs(view - X)) <= 8 * 2.0 ** -24 * scale


def test_read_of_streamed_appends_equals_one_shot():
    X = _as_dtype(_tokens(T=83, seed=3), "bf16")
    one = _stream(X, R=16, S=4, in_dtype="bf16")
    inc = CodecStreamOracle(16, 4, "i8", "bf16")
    for t in range(83):
        inc.append(X[:, :, t:t + 1])
    np.testing.assert_array_equal(one.read(), inc.read())


def test_read_of_empty_and_tail_only_streams():
    st = CodecStreamOracle(8, 2, "i8")
    assert st.read() is None
    X = _tokens(T=5)
    st.append(X)
    np.testing.assert_array_equal(st.read(), X)


# ---------------------------------------------------------------------- crop

@pytest.mark.parametrize("remove", [1, 3, 4, 5, 8, 12, 13, 30, 76, 77, 200])
def test_crop_equals_the_truncated_view(remove):
    """The pages' crop is exact: the view after removing k trailing tokens is
    the first T - k rows of the view before (a boundary block comes back raw,
    from the reconstruction), and archived blocks below it stay verbatim."""
    R, T = 8, 77
    X = _as_dtype(_tokens(T=T, seed=4), "bf16")
    st = _stream(X, R=R, S=3, in_dtype="bf16")
    before = st.read()
    codes = st.codes[:, :, :st.n_blocks].copy()
    st.crop(-remove)
    keep = max(0, T - remove)
    assert st.seq_len == keep
    assert st.n_blocks == keep // R and st.tail_len == keep % R
    if keep:
        np.testing.assert_array_equal(st.read(), before[:, :, :keep])
    else:
        assert st.read() is None
    np.testing.assert_array_equal(st.codes[:, :, :st.n_blocks],
                                  codes[:, :, :st.n_blocks])


def test_repeated_crops_compose():
    X = _as_dtype(_tokens(T=90, seed=5), "f32")
    a = _stream(X, R=8, S=2)
    b = _stream(X, R=8, S=2)
    a.crop(-3)
    a.crop(-9)
    a.crop(-2)
    b.crop(-14)
    assert a.n_blocks == b.n_blocks and a.tail_len == b.tail_len
    np.testing.assert_array_equal(a.read(), b.read())


def test_crop_to_a_block_boundary_then_replay_restores_the_archive():
    """Cropping at a block boundary keeps the archive below it verbatim, so
    appending the removed tokens again rebuilds the same codes and scales."""
    R = 16
    X = _as_dtype(_tokens(T=100, seed=6), "bf16")
    full = _stream(X, R=R, S=4, in_dtype="bf16")
    st = _stream(X, R=R, S=4, in_dtype="bf16")
    st.crop(-(100 - 48))
    assert (st.n_blocks, st.tail_len) == (3, 0)
    for t in range(48, 100):
        st.append(X[:, :, t:t + 1])
    nb = full.n_blocks
    np.testing.assert_array_equal(st.codes[:, :, :nb], full.codes[:, :, :nb])
    np.testing.assert_array_equal(st.scales[:, :, :nb],
                                  full.scales[:, :, :nb])
    np.testing.assert_array_equal(st.read(), full.read())


def test_crop_sign_convention():
    st = _stream(_tokens(T=20))
    with pytest.raises(ValueError):
        st.crop(3)
    before = st.read()
    st.crop(0)
    np.testing.assert_array_equal(st.read(), before)


# -------------------------------------------------------------- select_batch

@pytest.mark.parametrize("idx", [[2, 0, 1], [1, 1, 1], [0, 0, 1, 1, 2, 2],
                                 [2], [0, 1, 2]])
def test_select_batch_gathers_the_view(idx):
    X = _as_dtype(_tokens(T=45, seed=7), "bf16")
    st = _stream(X, R=8, S=2, in_dtype="bf16")
    before = st.read()
    st.select_batch(idx)
    np.testing.assert_array_equal(st.read(), before[idx])
    assert st.capacity == 16


def test_select_batch_then_append_equals_a_fresh_stream_of_those_rows():
    """Batch rows are independent streams: gathering rows and appending more
    tokens archives exactly what a stream built from those rows archives."""
    X = _as_dtype(_tokens(T=70, seed=8), "f32")
    idx = [1, 1, 0, 2]
    st = _stream(X[:, :, :37], R=8, S=3)
    st.select_batch(idx)
    for t in range(37, 70):
        st.append(X[idx][:, :, t:t + 1])
    fresh = _stream(X[idx], R=8, S=3)
    nb = fresh.n_blocks
    np.testing.assert_array_equal(st.codes[:, :, :nb], fresh.codes[:, :, :nb])
    np.testing.assert_array_equal(st.scales[:, :, :nb],
                                  fresh.scales[:, :, :nb])
    np.testing.assert_array_equal(st.read(), fresh.read())


def test_attention_after_select_batch_is_the_gathered_attention():
    R, S, G = 8, 2, 2
    X = _as_dtype(_tokens(T=53, seed=9), "f32")
    Y = _as_dtype(_tokens(T=53, seed=10), "f32")
    sk, sv = _stream(X, R, S), _stream(Y, R, S)
    q = np.random.default_rng(1).standard_normal((3, 2 * G, 1, 16))
    out = decode_attention_reference(q, sk.C_hat(), sv.C_hat(), sk.raw,
                                     sv.raw, R)
    idx = [2, 0, 2]
    sk.select_batch(idx)
    sv.select_batch(idx)
    got = decode_attention_reference(q[idx], sk.C_hat(), sv.C_hat(), sk.raw,
                                     sv.raw, R)
    np.testing.assert_array_equal(got, out[idx])


# --------------------------------------------------------------------- reset

def test_reset_keeps_capacity_and_restarts_the_stream():
    X = _tokens(T=300, seed=11)
    st = _stream(X, R=8, S=2)
    cap = st.capacity
    st.reset()
    assert (st.seq_len, st.n_blocks, st.tail_len, st.capacity) == \
        (0, 0, 0, cap)
    assert st.read() is None
    Z = _tokens(T=29, seed=12)
    st.append(Z)
    fresh = _stream(Z, R=8, S=2)
    np.testing.assert_array_equal(st.read(), fresh.read())
