"""The PNG lossless tier on the GPU (flashcodec-kv README, "Math", PNG
bullet; "Materialization-free decode attention": the coefficient-domain
decode also covers this tier): the archive holds per block the anchor and
the fp32 first differences, decode attention runs on those rows with the
cumulative-sum synthesis, and the reconstructed view gives the tokens back.
Checked against the fp64 oracle of the tier (oracle/png.py)."""

import numpy as np
import pytest
import torch

import oracle
import synth
from compressed_decode_attention_blockwise_b200 import CodecKVCache, _lib
from _helpers import check_out, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")

CASES = [
    # (B, Hq, Hk, D, R, nb, nr, in_dtype)
    (2, 8, 2, 128, 8, 60, 5, "bf16"),
    (1, 4, 4, 64, 4, 45, 3, "f32"),
    (1, 32, 8, 128, 16, 40, 11, "bf16"),
    (3, 6, 3, 32, 8, 33, 0, "f32"),
]
IDS = ["D128-R8-bf16", "D64-R4-f32", "D128-R16-G4", "D32-R8-notail"]


def _png_cache(w, data):
    cache = CodecKVCache(w.B, w.Hk, w.D, w.R, w.R, token_dtype=synth.torch_dtype(
        w.in_dtype), device=DEV, codec="png")
    cache.prefill(data["k"][:, :, :w.T].to(DEV), data["v"][:, :, :w.T].to(DEV))
    return cache


def _rows(stream):
    return f64(stream.live_coeffs())


def _workload(case, seed):
    B, Hq, Hk, D, R, nb, nr, ind = case
    return synth.Workload("png", B=B, Hq=Hq, Hk=Hk, D=D, T=nb * R + nr, R=R,
                          S=R, k_coeff="f32", v_coeff="f32", in_dtype=ind,
                          seed=seed)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_png_archive_rows_are_the_oracles_bitwise(case):
    w = _workload(case, 70)
    data = synth.generate(w, q_steps=0)
    cache = _png_cache(w, data)
    torch.cuda.synchronize()
    assert cache.k.n_blocks == w.T // w.R and cache.k.tail_len == w.T % w.R
    for st, x in ((cache.k, data["k"]), (cache.v, data["v"])):
        anchors, deltas, tail = oracle.png_filter(f64(x), w.R)
        ref = oracle.png_rows(anchors, oracle.png_store(deltas))
        got = _rows(st)
        assert np.array_equal(got, ref), float(np.max(np.abs(got - ref)))
        assert np.array_equal(f64(st.live_tail()), tail)
    # storage: every row in fp32 (the anchor too), plus the raw tail
    esz = 2 if w.in_dtype == "bf16" else 4
    assert cache.k.storage_bytes() == w.B * w.Hk * (
        cache.k.n_blocks * w.R * w.D * 4 + cache.k.tail_len * w.D * esz)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_png_decode_attention_matches_oracle(case):
    w = _workload(case, 71)
    data = synth.generate(w, q_steps=0)
    cache = _png_cache(w, data)
    q = data["q"].to(DEV)
    rk, rv = _rows(cache.k), _rows(cache.v)
    ref = oracle.png_decode_attention_reference(
        f64(data["q"]), rk[:, :, :, 0], rk[:, :, :, 1:], rv[:, :, :, 0],
        rv[:, :, :, 1:], f64(cache.k.live_tail()), f64(cache.v.live_tail()),
        w.R)
    assert not cache.tensor_core_path(w.Hq)
    nb = cache.k.n_blocks
    for ns in (0, 1, 3, nb, nb + 2):
        for fuse in (True, False):
            out = cache.attention(q, num_splits=ns, fuse_combine=fuse)
            torch.cuda.synchronize()
            check_out(f64(out), ref, "ns=%d fuse=%s" % (ns, fuse))


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_png_view_is_lossless_and_appends_equal_prefill(case):
    """The reconstructed view returns bf16 input tokens exactly (fp32 tokens
    within one rounding of their deltas); token-by-token appends build the
    prefill's archive bitwise; for bf16, a crop into a block and the
    re-append of the removed tokens restore it."""
    w = _workload(case, 72)
    data = synth.generate(w.replace(steps=2 * w.R + 1), q_steps=0)
    cache = _png_cache(w, data)
    kv, vv = cache.read()
    torch.cuda.synchronize()
    exact = w.in_dtype == "bf16"
    for got, x, st in ((kv, data["k"], cache.k), (vv, data["v"], cache.v)):
        want = x[:, :, :w.T].to(DEV)
        if exact:
            # a difference of two bf16 tokens fits fp32 unless their
            # exponents are far apart, so the fp32 cumulative sum gives the
            # tokens back bitwise almost everywhere; elsewhere the view is
            # the oracle's fp64 cumulative sum of the same rows, to one bf16
            # rounding
            diff = got != want
            frac = diff.float().mean().item()
            assert frac <= 1e-3, frac
            rows = _rows(st)
            rec = oracle.round_to_dtype(oracle.png_reconstruct(
                rows[:, :, :, 0], rows[:, :, :, 1:]), "bf16")
            full = np.concatenate([rec, f64(st.live_tail())], axis=2)
            g = f64(got)
            ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(full), 1e-30))[1] - 8)
            assert np.all(np.abs(g - full) <= ulp)
        else:                      # fp32 deltas of fp32 tokens: rounded once
            err = (got - want).abs().max().item()
            assert err <= 1e-6 * want.abs().max().item(), err
    steps = CodecKVCache(w.B, w.Hk, w.D, w.R, w.R,
                         token_dtype=synth.torch_dtype(w.in_dtype),
                         device=DEV, codec="png")
    k, v = data["k"].to(DEV), data["v"].to(DEV)
    T2 = w.T + 2 * w.R + 1
    for t in range(T2):
        steps.append(k[:, :, t:t + 1], v[:, :, t:t + 1])
    cache.prefill(k[:, :, w.T:T2], v[:, :, w.T:T2])
    torch.cuda.synchronize()
    for a, b in ((cache.k, steps.k), (cache.v, steps.v)):
        assert (a.n_blocks, a.tail_len) == (b.n_blocks, b.tail_len)
        assert torch.equal(a.live_coeffs(), b.live_coeffs())
        assert torch.equal(a.live_tail(), b.live_tail())
    n_cut = w.R + 3
    # a crop into a block returns that block's first tokens to the tail from
    # the view; when those view rows equal the input tokens, re-appending the
    # removed tokens rebuilds the archive bitwise
    keep = T2 - n_cut
    b0 = keep // w.R * w.R
    kv_all, vv_all = cache.read()
    if not (exact and torch.equal(kv_all[:, :, b0:keep], k[:, :, b0:keep]) and
            torch.equal(vv_all[:, :, b0:keep], v[:, :, b0:keep])):
        return
    before = [c.clone() for c in (cache.k.live_coeffs(), cache.v.live_coeffs())]
    cache.crop(-n_cut)
    cache.prefill(k[:, :, T2 - n_cut:T2], v[:, :, T2 - n_cut:T2])
    torch.cuda.synchronize()
    assert torch.equal(cache.k.live_coeffs(), before[0])
    assert torch.equal(cache.v.live_coeffs(), before[1])
    kv2, _ = cache.read()
    assert torch.equal(kv2[:, :, :b0], kv_all[:, :, :b0])


def test_png_rejects_inconsistent_descriptors():
    """The tier keeps every row in fp32: S != R or an int8 archive is
    refused on the host."""
    c = CodecKVCache(1, 2, 64, 8, 8, device=DEV, codec="png")
    x = torch.randn(1, 2, 20, 64, dtype=torch.bfloat16, device=DEV)
    c.prefill(x, x)
    bad = _lib.FcArchive()
    from compressed_decode_attention_blockwise_b200.archive import ctypes_copy
    ctypes_copy(bad, c.k.arc)
    bad.S = 4
    with pytest.raises(_lib.FcError) as e:
        _lib.fc_compress_blocks(x, bad)
    assert e.value.status == _lib.FC_ERR_INVALID
