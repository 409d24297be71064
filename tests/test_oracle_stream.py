"""Pins for the oracle's stream (raw tail + capacity-doubling archive)."""

import numpy as np
import pytest

from oracle import codec
from oracle.attention import decode_attention_reference
from oracle.stream import CodecStreamOracle, grown_capacity


def _tokens(B=2, H=3, T=77, D=16, seed=0):
    rng = np.random.default_rng(seed)
    return np.cumsum(rng.standard_normal((B, H, T, D)), axis=2)


@pytest.mark.parametrize("coeff", ["i8", "f32", "bf16"])
def test_token_by_token_equals_one_shot(coeff):
    X = _tokens()
    one = CodecStreamOracle(8, 3, coeff)
    one.append(X)
    inc = CodecStreamOracle(8, 3, coeff)
    for t in range(X.shape[2]):
        inc.append(X[:, :, t:t + 1])
    assert one.n_blocks == inc.n_blocks == 77 // 8
    assert one.tail_len == inc.tail_len == 77 % 8
    np.testing.assert_array_equal(one.C_hat(), inc.C_hat())
    np.testing.assert_array_equal(one.raw, inc.raw)
    if coeff == "i8":
        nb = one.n_blocks
        np.testing.assert_array_equal(one.codes[:, :, :nb],
                                      inc.codes[:, :, :nb])
        np.testing.assert_array_equal(one.scales[:, :, :nb],
                                      inc.scales[:, :, :nb])


def test_random_chunk_appends_equal_one_shot():
    X = _tokens(T=300, seed=1)
    rng = np.random.default_rng(4)
    one = CodecStreamOracle(16, 4, "i8")
    one.append(X)
    inc = CodecStreamOracle(16, 4, "i8")
    t = 0
    while t < X.shape[2]:
        m = int(rng.integers(1, 40))
        inc.append(X[:, :, t:t + m])
        t += m
    np.testing.assert_array_equal(one.C_hat(), inc.C_hat())
    np.testing.assert_array_equal(one.raw, inc.raw)


def test_archived_blocks_never_change():
    """Causal safety: later appends leave every archived code and scale
    bitwise unchanged."""
    X = _tokens(T=200, seed=2)
    st = CodecStreamOracle(8, 2, "i8")
    st.append(X[:, :, :50])
    nb0 = st.n_blocks
    codes0 = st.codes[:, :, :nb0].copy()
    scales0 = st.scales[:, :, :nb0].copy()
    rng = np.random.default_rng(0)
    for t in range(50, 200):
        # perturb the future: archived history must not move
        st.append(X[:, :, t:t + 1] + rng.standard_normal() * 100)
    np.testing.assert_array_equal(st.codes[:, :, :nb0], codes0)
    np.testing.assert_array_equal(st.scales[:, :, :nb0], scales0)


def test_capacity_doubles_from_sixteen():
    assert grown_capacity(0, 1) == 16
    assert grown_capacity(0, 16) == 16
    assert grown_capacity(16, 17) == 32
    assert grown_capacity(32, 100) == 128
    assert grown_capacity(128, 100) == 128
    st = CodecStreamOracle(4, 2, "i8")
    caps = []
    X = _tokens(B=1, H=1, T=4 * 70, D=4)
    for t in range(X.shape[2]):
        st.append(X[:, :, t:t + 1])
        caps.append(st.capacity)
    assert sorted(set(caps)) == [0, 16, 32, 64, 128]
    assert st.capacity == 128 and st.n_blocks == 70


def test_streamed_attention_equals_one_shot_archive():
    X = _tokens(T=90, seed=5)
    Y = _tokens(T=90, seed=6)
    R, S = 8, 2
    sk, sv = CodecStreamOracle(R, S, "i8"), CodecStreamOracle(R, S, "i8")
    for t in range(90):
        sk.append(X[:, :, t:t + 1])
        sv.append(Y[:, :, t:t + 1])
    rng = np.random.default_rng(0)
    q = rng.standard_normal((2, 6, 1, 16))
    B, H, D = 2, 3, 16
    a = decode_attention_reference(q, sk.C_hat(), sv.C_hat(),
                                   sk.tail(B, H, D), sv.tail(B, H, D), R)
    ek = codec.encode_stream(X, R, S, "i8")
    ev = codec.encode_stream(Y, R, S, "i8")
    b = decode_attention_reference(q, ek["C_hat"], ev["C_hat"], ek["tail"],
                                   ev["tail"], R)
    np.testing.assert_array_equal(a, b)
