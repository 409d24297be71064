"""Exact save and restore of a stream through host memory (fc_state_save /
fc_state_restore), and the pages' lossy legacy export / import
(flashcodec/cache.py, FlashCodecCache.to_legacy_cache / from_legacy_cache)."""

import pytest
import torch

import synth
from compressed_decode_attention_blockwise_b200 import CodecKVCache, _lib
from _helpers import check_out, f64, oracle_on_gpu_archive

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _cache(w, data, capacity=0):
    c = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                     token_dtype=synth.torch_dtype(w.in_dtype), device=DEV,
                     capacity=capacity)
    c.prefill(data["k"][:, :, :w.T].to(DEV), data["v"][:, :, :w.T].to(DEV))
    return c


def _same(a, b):
    assert (a.k.n_blocks, a.k.tail_len) == (b.k.n_blocks, b.k.tail_len)
    for sa, sb in ((a.k, b.k), (a.v, b.v)):
        assert torch.equal(sa.live_coeffs(), sb.live_coeffs())
        if sa.scales is not None:
            assert torch.equal(sa.live_scales(), sb.live_scales())
        assert torch.equal(sa.live_tail(), sb.live_tail())


@pytest.mark.parametrize("w", [
    synth.WORKLOADS["gqa"].replace(B=2, T=8 * 50 + 5, seed=41, steps=11),
    synth.WORKLOADS["large"].replace(B=2, T=8 * 33 + 7, seed=42, steps=11),
    synth.Workload("f32", B=1, Hq=4, Hk=2, D=64, T=16 * 9, R=16, S=4,
                   in_dtype="f32", seed=43, steps=11),
    synth.WORKLOADS["gqa"].replace(B=2, T=5, seed=44, steps=11),
], ids=["i8-tail5", "i8k-bf16v-tail7", "f32-tokens-no-tail", "tail-only"])
def test_save_restore_is_bitwise_and_resumes(w):
    data = synth.generate(w, q_steps=2)
    src = _cache(w, data)
    q = data["q"][0].to(DEV)
    out_src = src.attention(q)
    state = src.save_state()
    hd = _lib.fc_state_header(state["k"])
    assert (hd.n_blocks, hd.tail_len) == (src.k.n_blocks, src.k.tail_len)
    assert state["k"].numel() == _lib.fc_state_bytes(src.k.arc,
                                                     src.k.tail_desc)
    # a fresh cache of another capacity, holding other data first
    dst = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                       token_dtype=synth.torch_dtype(w.in_dtype), device=DEV)
    junk = torch.randn((w.B, w.Hk, 3 * w.R + 1, w.D), device=DEV).to(
        synth.torch_dtype(w.in_dtype))
    dst.prefill(junk, junk)
    dst.restore_state(state)
    torch.cuda.synchronize()
    _same(src, dst)
    assert torch.equal(dst.attention(q), out_src)
    # both continue identically (the restored stream is a working stream)
    for s in range(w.steps):
        t = w.T + s
        for c in (src, dst):
            c.append(data["k"][:, :, t:t + 1].to(DEV),
                     data["v"][:, :, t:t + 1].to(DEV))
    q1 = data["q"][1].to(DEV)
    o1, o2 = src.attention(q1), dst.attention(q1)
    torch.cuda.synchronize()
    _same(src, dst)
    assert torch.equal(o1, o2)
    check_out(f64(o2), oracle_on_gpu_archive(dst, q1), "restored + appended")


def test_restore_rejects_another_geometry():
    w = synth.WORKLOADS["gqa"].replace(B=1, T=8 * 20 + 3, seed=45)
    data = synth.generate(w, q_steps=0)
    state = _cache(w, data).save_state()
    other = CodecKVCache(w.B, w.Hk, w.D, w.R, 3, device=DEV)   # S = 3
    with pytest.raises(_lib.FcError) as e:
        other.k.restore_state(state["k"])
    assert e.value.status == _lib.FC_ERR_INVALID
    assert other.k.n_blocks == 0
    bad = state["k"].clone()
    bad[0] = ord("X")                                          # magic
    same = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, device=DEV)
    with pytest.raises(_lib.FcError):
        same.k.restore_state(bad)


def test_legacy_export_import_goes_through_the_codec_again():
    """to_legacy hands out the reconstructed views; from_legacy builds a new
    cache from them (lossy a second time): a valid stream of the same length
    whose attention matches the oracle on its own archive."""
    w = synth.WORKLOADS["gqa"].replace(B=2, T=8 * 40 + 6, seed=46)
    data = synth.generate(w, q_steps=0)
    src = _cache(w, data)
    keys, values = src.to_legacy()
    assert keys.shape == (w.B, w.Hk, w.T, w.D)
    new = CodecKVCache.from_legacy(keys, values, R=w.R, S=w.S)
    assert new.seq_len == src.seq_len and new.k.n_blocks == src.k.n_blocks
    assert torch.equal(new.k.live_tail(), src.k.live_tail())
    q = data["q"].to(DEV)
    out = new.attention(q)
    torch.cuda.synchronize()
    check_out(f64(out), oracle_on_gpu_archive(new, q), "legacy import")
