"""The streaming workload on the GPU: a bf16 prefill compressed into the int8
archive, then single-token decode steps crossing block boundaries, each
followed by decode attention; checked against the fp64 oracle replaying the
same appends."""

import numpy as np
import pytest
import torch

import oracle
import synth
from compressed_decode_attention_blockwise_b200 import CodecKVCache
from _helpers import check_codes, check_out, check_scales, f64, \
    oracle_on_gpu_archive

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _run_stream(w, check_steps):
    data = synth.generate(w)
    k, v, q = data["k"].to(DEV), data["v"].to(DEV), data["q"].to(DEV)
    cache = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, device=DEV)
    cache.prefill(k[:, :, :w.T], v[:, :, :w.T])
    outs = {}
    for s in range(w.steps):
        t = w.T + s
        cache.append(k[:, :, t:t + 1], v[:, :, t:t + 1])
        out = cache.attention(q[s])
        if s in check_steps:
            torch.cuda.synchronize()
            outs[s] = (f64(out), oracle_on_gpu_archive(cache, q[s]),
                       cache.k.n_blocks, cache.k.tail_len)
    torch.cuda.synchronize()
    return cache, data, outs


def test_stream_small_against_oracle_replay():
    w = synth.WORKLOADS["stream"].replace(B=2, T=8 * 64, steps=40, seed=9)
    cache, data, outs = _run_stream(w, set(range(40)))
    for s, (got, ref, nb, nr) in outs.items():
        check_out(got, ref, "step %d" % s)
        assert nb * w.R + nr == w.T + s + 1
    # the oracle's own stream replay gives the same archive (+-1 rule)
    ko = oracle.CodecStreamOracle(w.R, w.S, "i8", "bf16")
    ko.append(f64(data["k"][:, :, :w.T]))
    for s in range(w.steps):
        ko.append(f64(data["k"][:, :, w.T + s:w.T + s + 1]))
    nb = ko.n_blocks
    assert cache.k.n_blocks == nb and cache.k.tail_len == ko.tail_len
    check_codes(cache.k.live_coeffs().cpu().numpy(), ko.pre_round[:, :, :nb])
    check_scales(cache.k.live_scales().cpu().numpy(), ko.scales[:, :, :nb])


def test_stream_full_size():
    w = synth.WORKLOADS["stream"]
    steps = {0, 6, 7, 8, 100, 255}
    cache, data, outs = _run_stream(w, steps)
    assert cache.k.n_blocks == (w.T + w.steps) // w.R
    for s, (got, ref, nb, nr) in outs.items():
        check_out(got, ref, "step %d" % s)
