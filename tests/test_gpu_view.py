"""The stream's structural operations on the GPU, against the fp64 oracle:
the reconstructed view (fc_read_view, memoised across appends), exact crop
(fc_crop) and batch gather (fc_select_batch), plus reset
(flashcodec/cache.py, _CodecStream.read / crop / select_batch / reset).

View tolerance, derived from the arithmetic: the kernel evaluates
x = sum_j M[j, t] * (code_j * scale_j) in fp32 (the basis rounded to fp32, one
rounding per product and FMA), so |x - exact| <= (S + 3) 2^-24
sum_j |M[j, t]| |C_hat_j|. An fp32 view must lie within that bound of the
exact fp64 value. A bf16 view value g is x rounded to nearest, so
|g - exact| <= bound + half a bf16 ulp of g; where the bound is far below a
bf16 ulp this means g is the exact value rounded to bf16 or, next to a
rounding midpoint, its neighbour (near-cancelling rows, whose bound exceeds
their own ulp, may differ by more). At most 0.1% of the positions may differ
from the exact value rounded to bf16.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from compressed_decode_attention_blockwise_b200 import CodecKVCache, _lib
from _helpers import check_out, f64, oracle_on_gpu_archive

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _archive_f64(stream, b=slice(None), h=slice(None), blocks=None):
    """The GPU's live archived coefficients as float64 (B, H, nb, S, D)."""
    sl = slice(0, stream.n_blocks) if blocks is None else blocks
    c = stream.coeffs[b, h, sl]
    if stream.coeff == "i8":
        return oracle.dequantize(c.cpu().numpy(), stream.scales[b, h, sl]
                                 .cpu().numpy())
    return f64(c)


def check_view_rows(got: np.ndarray, C_hat: np.ndarray, R: int, dtype: str):
    """``got`` (B, H, nb*R, D) decoded rows against the exact decompression
    of ``C_hat`` (B, H, nb, S, D) under the tolerance in the module
    docstring. Returns how many bf16 positions differ from the exact value
    rounded to bf16."""
    S = C_hat.shape[-2]
    exact = oracle.decompress(C_hat, R)
    M = oracle.dct_basis(R, S)
    mag = np.einsum("jt,bhnjd->bhntd", np.abs(M), np.abs(C_hat)) \
        .reshape(exact.shape)
    bound = (S + 3) * 2.0 ** -24 * mag + 1e-35
    if dtype == "f32":
        err = np.abs(got - exact)
        assert np.all(err <= bound), "f32 view off by %.3g of the bound" % \
            float(np.max(err / bound))
        return 0
    np.testing.assert_array_equal(got, oracle.round_to_dtype(got, "bf16"))
    half_ulp = np.ldexp(1.0, np.frexp(np.abs(got))[1] - 9)
    err = np.abs(got - exact)
    bad = err > bound + half_ulp
    if bad.any():
        k = tuple(np.argwhere(bad)[0])
        raise AssertionError(
            "bf16 view mismatch at %d positions; first %s: view %r exact %r "
            "bound %.3g" % (int(bad.sum()), k, float(got[k]), float(exact[k]),
                            float(bound[k])))
    n_diff = int((got != oracle.round_to_dtype(exact, "bf16")).sum())
    assert n_diff <= 1e-3 * got.size + 8, n_diff
    return n_diff


def _cache(B, H, D, R, S, coeff, in_dtype, T, seed=0, outlier=0.0, G=1,
           v_coeff=None):
    w = synth.WORKLOADS["gqa"].replace(
        B=B, Hq=H * G, Hk=H, D=D, T=T, R=R, S=S, k_coeff=coeff,
        v_coeff=v_coeff or coeff, in_dtype=in_dtype, outlier_frac=outlier,
        seed=seed)
    data = synth.generate(w, q_steps=0)
    cache = CodecKVCache(B, H, D, R, S, coeff_k=w.k_coeff,
                         coeff_v=w.v_coeff,
                         token_dtype=synth.torch_dtype(in_dtype), device=DEV)
    cache.prefill(data["k"].to(DEV), data["v"].to(DEV))
    return cache, data, w


def _check_stream_view(stream, view, dtype):
    nb, R = stream.n_blocks, stream.R
    assert view.shape[2] == stream.seq_len
    v = f64(view)
    n = check_view_rows(v[:, :, :nb * R], _archive_f64(stream), R, dtype)
    np.testing.assert_array_equal(v[:, :, nb * R:], f64(stream.live_tail()))
    return n


VIEW_CASES = [
    # B, H, D, R, S, coeff, token dtype, T
    (1, 4, 64, 8, 2, "f32", "f32", 256 + 3),        # tiny-like
    (2, 8, 128, 8, 2, "i8", "bf16", 8 * 40 + 5),    # gqa-like
    (1, 8, 128, 16, 4, "i8", "bf16", 16 * 37 + 3),  # long-like
    (2, 8, 128, 8, 3, "bf16", "bf16", 8 * 21 + 7),  # large-like V stream
    (2, 2, 32, 16, 12, "i8", "f32", 16 * 9 + 15),   # S > 8
    (1, 2, 256, 32, 16, "f32", "bf16", 32 * 5 + 1),
    (1, 3, 64, 4, 4, "bf16", "f32", 4 * 50),        # S = R, empty tail
    (1, 4, 128, 8, 3, "i8", "f32", 8 * 33 + 2),     # unrolled rows, S = 3
    (1, 2, 256, 16, 8, "i8", "bf16", 16 * 11 + 9),  # unrolled rows, D = 256
]


@pytest.mark.parametrize("case", VIEW_CASES, ids=lambda c: "-".join(map(str, c)))
def test_read_view_matches_oracle(case):
    B, H, D, R, S, coeff, dt, T = case
    cache, data, w = _cache(B, H, D, R, S, coeff, dt, T, seed=sum(case[:5]),
                            outlier=0.01 if R == 16 else 0.0)
    kv, vv = cache.read()
    torch.cuda.synchronize()
    for stream, view in ((cache.k, kv), (cache.v, vv)):
        _check_stream_view(stream, view, dt)


def test_read_view_is_memoised_across_appends_and_growth():
    """Token-by-token appends with a read after each: every view equals a
    full decode of the current stream, decoded rows of earlier views never
    change, and the buffer grows past its first 16 blocks."""
    R = 8
    cache, data, w = _cache(2, 2, 128, R, 2, "i8", "bf16", 8 * 15 + 3,
                            seed=21)
    extra = synth.generate(w.replace(T=40, seed=22), q_steps=0)
    ek, ev = extra["k"].to(DEV), extra["v"].to(DEV)
    held = []
    for s in range(40):
        cache.append(ek[:, :, s:s + 1], ev[:, :, s:s + 1])
        view = cache.k.read()
        full = torch.empty((2, 2, cache.seq_len + R, 128), dtype=torch.bfloat16,
                           device=DEV)
        _lib.fc_read_view(cache.k.arc, cache.k.tail_desc, 0, full)
        torch.cuda.synchronize()
        assert torch.equal(view, full[:, :, :cache.seq_len])
        held.append((view, view[:, :, :cache.k.n_blocks * R].clone()))
    for view, decoded in held:
        assert torch.equal(view[:, :, :decoded.shape[2]], decoded)
    assert cache.k._rec.shape[2] == 32 * R
    _check_stream_view(cache.k, cache.k.read(), "bf16")


@pytest.mark.parametrize("remove", [2, 5, 6, 13, 40, 165, 500])
def test_crop_is_the_truncated_view_and_decoding_continues(remove):
    B, H, R, T = 2, 2, 8, 8 * 20 + 5
    cache, data, w = _cache(B, H, 128, R, 2, "i8", "bf16", T, seed=remove,
                            G=4)
    before_k, before_v = [x.clone() for x in cache.read()]
    codes = cache.k.live_coeffs().clone()
    cache.crop(-remove)
    keep = max(0, T - remove)
    assert cache.seq_len == keep
    assert (cache.k.n_blocks, cache.k.tail_len) == (keep // R, keep % R)
    assert (cache.v.n_blocks, cache.v.tail_len) == (keep // R, keep % R)
    kb = keep // R
    assert torch.equal(cache.k.live_coeffs(), codes[:, :, :kb])
    if keep:
        kv, vv = cache.read()
        assert torch.equal(kv, before_k[:, :, :keep])
        assert torch.equal(vv, before_v[:, :, :keep])
    else:
        assert cache.read() == (None, None)
    # decoding continues from the cropped stream
    more = synth.generate(w.replace(T=12, seed=remove + 100), q_steps=4)
    mk, mv = more["k"].to(DEV), more["v"].to(DEV)
    for s in range(12):
        cache.append(mk[:, :, s:s + 1], mv[:, :, s:s + 1])
    assert cache.seq_len == keep + 12
    q = more["q"][0].to(DEV)
    out = cache.attention(q)
    torch.cuda.synchronize()
    check_out(f64(out), oracle_on_gpu_archive(cache, q), "after crop")


def test_select_batch_gathers_bitwise_and_attention_follows():
    B, H, R, T = 3, 2, 8, 8 * 30 + 3
    cache, data, w = _cache(B, H, 128, R, 2, "i8", "bf16", T, seed=41, G=4)
    old_k = cache.k.live_coeffs().clone()
    old_s = cache.k.live_scales().clone()
    old_t = cache.v.live_tail().clone()
    old_view = [x.clone() for x in cache.read()]
    idx = [2, 0, 2, 1]
    cache.reorder_cache(torch.tensor(idx))
    torch.cuda.synchronize()
    assert cache.B == 4 and cache.k.n_blocks == 30 and cache.k.tail_len == 3
    assert torch.equal(cache.k.live_coeffs(), old_k[idx])
    assert torch.equal(cache.k.live_scales(), old_s[idx])
    assert torch.equal(cache.v.live_tail(), old_t[idx])
    kv, vv = cache.read()
    assert torch.equal(kv, old_view[0][idx]) and torch.equal(vv, old_view[1][idx])
    more = synth.generate(w.replace(B=4, T=6, seed=42), q_steps=2)
    q = more["q"][0].to(DEV)
    out = cache.attention(q)
    torch.cuda.synchronize()
    check_out(f64(out), oracle_on_gpu_archive(cache, q), "after gather")
    # one fused decode step that completes a block, then shrink and repeat
    mk, mv = more["k"].to(DEV), more["v"].to(DEV)
    for s in range(5):
        out = cache.step(q, mk[:, :, s:s + 1], mv[:, :, s:s + 1])
    torch.cuda.synchronize()
    assert cache.k.n_blocks == 31
    check_out(f64(out), oracle_on_gpu_archive(cache, q), "step after gather")
    view4 = cache.k.read().clone()
    cache.batch_select_indices([3, 0])
    assert torch.equal(cache.k.read(), view4[[3, 0]])
    cache.batch_repeat_interleave(2)
    assert cache.B == 4
    assert torch.equal(cache.k.read(), view4[[3, 3, 0, 0]])
    q4 = more["q"][1].to(DEV)
    out = cache.attention(q4)
    torch.cuda.synchronize()
    check_out(f64(out), oracle_on_gpu_archive(cache, q4), "after repeat")


def test_reset_keeps_capacity_and_refills_like_a_fresh_cache():
    cache, data, w = _cache(2, 2, 128, 8, 2, "i8", "bf16", 8 * 40 + 1,
                            seed=51)
    cap = cache.k.capacity
    cache.reset()
    assert cache.seq_len == 0 and cache.read() == (None, None)
    assert cache.k.capacity == cap
    fresh, data2, w2 = _cache(2, 2, 128, 8, 2, "i8", "bf16", 8 * 9 + 4,
                              seed=52)
    cache.prefill(data2["k"].to(DEV), data2["v"].to(DEV))
    assert torch.equal(cache.k.live_coeffs(), fresh.k.live_coeffs())
    assert torch.equal(cache.k.live_scales(), fresh.k.live_scales())
    assert torch.equal(cache.v.live_tail(), fresh.v.live_tail())
    assert torch.equal(cache.read()[0], fresh.read()[0])


def test_full_size_long_view_sampled_blocks():
    """The long workload's whole K and V views (131075 tokens, 8 heads)
    decoded in one launch each; sampled blocks of every head and the tail
    rows checked against the oracle."""
    w = synth.WORKLOADS["long"]
    data = synth.generate(w, q_steps=0)
    cache = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, device=DEV)
    cache.prefill(data["k"].to(DEV), data["v"].to(DEV))
    kv, vv = cache.read()
    torch.cuda.synchronize()
    nb, R = cache.k.n_blocks, w.R
    rng = np.random.default_rng(7)
    picks = sorted(set([0, 1, nb - 1] + rng.integers(0, nb, 16).tolist()))
    for stream, view in ((cache.k, kv), (cache.v, vv)):
        assert view.shape == (w.B, w.Hk, w.T, w.D)
        for n in picks:
            rows = f64(view[:, :, n * R:(n + 1) * R])
            check_view_rows(rows, _archive_f64(stream, blocks=slice(n, n + 1)),
                            R, "bf16")
        np.testing.assert_array_equal(f64(view[:, :, nb * R:]),
                                      f64(stream.live_tail()))
