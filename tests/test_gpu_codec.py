"""GPU parity of the codec kernels against the fp64 oracle (through the C ABI):
prefill compression, single-token append, causal safety, capacity growth."""

import numpy as np
import pytest
import torch

import oracle
import synth
from compressed_decode_attention_blockwise_b200 import (CodecKVCache, FcError,
                                                        _lib)
from _helpers import check_codes, check_coeffs, check_scales, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _compare_stream(stream, X: np.ndarray, heads=None):
    """Device archive of one stream against the oracle's encoding of X
    (B, H, T, D) float64; ``heads`` limits the check to (b, h) pairs."""
    R, S = stream.R, stream.S
    nb = stream.n_blocks
    assert nb == X.shape[2] // R
    pairs = heads or [(b, h) for b in range(X.shape[0])
                      for h in range(X.shape[1])]
    flips = 0
    for b, h in pairs:
        enc = oracle.encode_stream(X[b:b + 1, h:h + 1], R, S, stream.coeff)
        if stream.coeff == "i8":
            codes = stream.coeffs[b, h, :nb].cpu().numpy()
            scales = stream.scales[b, h, :nb].cpu().numpy()
            flips += check_codes(codes, enc["y"][0, 0])
            check_scales(scales, np.abs(enc["C"][0, 0]).max(-1) / 127.0)
        else:
            check_coeffs(f64(stream.coeffs[b, h, :nb]), enc["C"][0, 0],
                         stream.coeff)
        nr = X.shape[2] - nb * R
        np.testing.assert_array_equal(f64(stream.tail[b, h, :nr]),
                                      X[b, h, nb * R:])
    return flips


@pytest.mark.parametrize("name", ["tiny", "gqa", "long", "large"])
def test_prefill_compress_full_size(name):
    w = synth.WORKLOADS[name]
    data = synth.generate(w, q_steps=0)
    cache = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                         token_dtype=synth.torch_dtype(w.in_dtype), device=DEV)
    cache.prefill(data["k"].to(DEV), data["v"].to(DEV))
    torch.cuda.synchronize()
    assert cache.k.tail_len == w.n_tail and cache.k.n_blocks == w.n_blocks
    heads = None
    if w.B * w.Hk > 64:
        rng = np.random.default_rng(0)
        heads = [(int(rng.integers(w.B)), int(rng.integers(w.Hk)))
                 for _ in range(12)] + [(w.B - 1, w.Hk - 1)]
    _compare_stream(cache.k, f64(data["k"]), heads)
    _compare_stream(cache.v, f64(data["v"]), heads)


@pytest.mark.parametrize("coeff", ["i8", "bf16", "f32"])
@pytest.mark.parametrize("R,S,D", [(8, 2, 128), (16, 4, 64), (32, 16, 256),
                                   (5, 3, 32), (1, 1, 64)])
def test_compress_shapes_and_dtypes(coeff, R, S, D):
    w = synth.Workload("t", B=2, Hq=3, Hk=3, D=D, T=R * 11 + R // 2, R=R,
                       S=S, k_coeff=coeff, v_coeff=coeff, seed=R * 7 + S)
    data = synth.generate(w, q_steps=0)
    for tok_dtype in (torch.bfloat16, torch.float32):
        cache = CodecKVCache(w.B, w.Hk, D, R, S, coeff, coeff,
                             token_dtype=tok_dtype, device=DEV)
        k = data["k"].to(tok_dtype)
        cache.prefill(k.to(DEV), k.to(DEV))
        torch.cuda.synchronize()
        _compare_stream(cache.k, f64(k))


def test_zero_block_stores_zero_scale_and_codes():
    B, H, D, R, S = 1, 2, 64, 8, 3
    x = torch.randn(B, H, 4 * R, D, dtype=torch.float32)
    x[:, :, R:2 * R] = 0.0
    cache = CodecKVCache(B, H, D, R, S, "i8", "i8", torch.float32, DEV)
    cache.prefill(x.to(DEV), x.to(DEV))
    torch.cuda.synchronize()
    assert torch.all(cache.k.scales[:, :, 1] == 0)
    assert torch.all(cache.k.coeffs[:, :, 1] == 0)
    _compare_stream(cache.k, f64(x))


@pytest.mark.parametrize("R,S,kc,vc", [(8, 2, "i8", "i8"), (16, 4, "i8", "i8"),
                                       (8, 3, "i8", "bf16")])
def test_append_matches_prefill_bitwise_and_is_causal(R, S, kc, vc):
    # the prefill of these geometries runs the encoder with S and R fixed at
    # compile time, the append its runtime-sized form: the codes must agree
    w = synth.WORKLOADS["stream"].replace(B=2, T=R * 40 + 3, R=R, S=S,
                                          k_coeff=kc, v_coeff=vc, steps=0,
                                          seed=5)
    data = synth.generate(w, q_steps=0)
    k, v = data["k"].to(DEV), data["v"].to(DEV)
    one = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, kc, vc, device=DEV)
    one.prefill(k, v)
    inc = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, kc, vc, device=DEV)
    snap = None
    for t in range(w.T):
        inc.append(k[:, :, t:t + 1], v[:, :, t:t + 1])
        if t == R * 20 + 2:  # 20 archived blocks
            torch.cuda.synchronize()
            snap = [(st.live_coeffs().clone(), st.live_scales())
                    for st in (inc.k, inc.v)]
            snap = [(c, None if sc is None else sc.clone()) for c, sc in snap]
    torch.cuda.synchronize()
    assert inc.k.n_blocks == one.k.n_blocks == 40
    assert inc.k.tail_len == one.k.tail_len == 3
    for a, b in ((inc.k, one.k), (inc.v, one.v)):
        assert torch.equal(a.live_coeffs(), b.live_coeffs())
        if a.live_scales() is None:       # unquantised stream
            assert b.live_scales() is None
        else:
            assert torch.equal(a.live_scales(), b.live_scales())
        assert torch.equal(a.live_tail(), b.live_tail())
    # archived blocks are never rewritten by later appends
    for st, (c0, s0) in zip((inc.k, inc.v), snap):
        nb0 = c0.shape[2]
        assert torch.equal(st.coeffs[:, :, :nb0], c0)
        if s0 is not None:
            assert torch.equal(st.scales[:, :, :nb0], s0)
    # capacity doubled 16 -> 32 -> 64 along the way
    assert inc.k.capacity == 64


def test_prefill_after_partial_tail_matches_oracle_stream():
    """Mixed appends and prefills (random chunk sizes) equal the oracle's
    append semantics."""
    B, H, D, R, S = 1, 2, 64, 8, 2
    rng = np.random.default_rng(3)
    X = torch.from_numpy(np.cumsum(rng.standard_normal((B, H, 300, D)),
                                   axis=2)).to(torch.bfloat16)
    cache = CodecKVCache(B, H, D, R, S, device=DEV)
    ora = oracle.CodecStreamOracle(R, S, "i8", "bf16")
    t = 0
    while t < 300:
        m = int(rng.integers(1, 50))
        chunk = X[:, :, t:t + m]
        if m == 1:
            cache.append(chunk.to(DEV), chunk.to(DEV))
        else:
            cache.prefill(chunk.to(DEV), chunk.to(DEV))
        ora.append(f64(chunk))
        t += m
    torch.cuda.synchronize()
    nb = ora.n_blocks
    assert cache.k.n_blocks == nb and cache.k.tail_len == ora.tail_len
    check_codes(cache.k.live_coeffs().cpu().numpy(), ora.pre_round[:, :, :nb])
    check_scales(cache.k.live_scales().cpu().numpy(), ora.scales[:, :, :nb])
    np.testing.assert_array_equal(f64(cache.k.live_tail()), ora.tail(B, H, D))


def test_capacity_error_then_grow_and_retry():
    B, H, D, R, S = 1, 1, 64, 4, 2
    cache = CodecKVCache(B, H, D, R, S, device=DEV)
    x = torch.randn(B, H, 16 * R, D, dtype=torch.bfloat16, device=DEV)
    cache.prefill(x, x)                      # exactly fills 16 blocks
    assert cache.k.capacity == 16 and cache.k.n_blocks == 16
    tok = torch.randn(B, H, 1, D, dtype=torch.bfloat16, device=DEV)
    for _ in range(R - 1):
        _lib.fc_append_step(tok, tok, cache.k.arc, cache.v.arc,
                            cache.k.tail_desc, cache.v.tail_desc)
    with pytest.raises(FcError) as e:
        _lib.fc_append_step(tok, tok, cache.k.arc, cache.v.arc,
                            cache.k.tail_desc, cache.v.tail_desc)
    assert e.value.status == _lib.FC_ERR_CAPACITY
    assert cache.k.tail_len == R - 1 and cache.k.n_blocks == 16
    before = cache.k.live_coeffs().clone()
    cache.append(tok, tok)                   # grows to 32, copies, archives
    torch.cuda.synchronize()
    assert cache.k.capacity == 32 and cache.k.n_blocks == 17
    assert torch.equal(cache.k.coeffs[:, :, :16], before)
