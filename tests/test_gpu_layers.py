"""fc_decode_step_layers: the fused decode steps of several layers' streams
in one launch, against the same steps issued layer by layer (bitwise: each
CTA runs the single call's code) and against the fp64 oracle on each
layer's own archive, at the `long` workload's shape with tails that cross a
block boundary during the steps."""

import numpy as np
import pytest
import torch

import oracle
import synth
from compressed_decode_attention_blockwise_b200 import (CodecKVCache, _lib,
                                                        decode_step_layers)
from _helpers import check_out, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _dequant(stream, b, h):
    c = stream.coeffs[b:b + 1, h:h + 1, :stream.n_blocks].cpu().numpy()
    s = stream.scales[b:b + 1, h:h + 1, :stream.n_blocks].cpu().numpy()
    return oracle.dequantize(c, s)


def _layers(w, tails, data):
    """One cache per layer: layer l holds the first n_blocks * R + tails[l]
    tokens of the workload's streams (its own copy)."""
    k, v = data["k"].to(DEV), data["v"].to(DEV)
    nb = w.T // w.R
    caches, lens = [], []
    for tail in tails:
        T = nb * w.R + tail
        c = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, device=DEV,
                         capacity=nb + 4)
        c.prefill(k[:, :, :T], v[:, :, :T])
        caches.append(c)
        lens.append(T)
    return caches, lens, k, v


@pytest.mark.parametrize("name,tails,steps,overlap", [
    ("long", (3, 14, 15, 7), 3, False),
    ("gqa", (5, 6, 7, 0, 1, 2), 3, False),
    ("long", (3, 14, 15, 7), 3, True),
])
def test_layers_in_one_launch_match_per_layer_steps_and_oracle(name, tails,
                                                              steps, overlap):
    # overlap: the layer launches of consecutive steps run as programmatic
    # dependents with every query final up front (FC_DECODE_OVERLAP |
    # FC_DECODE_Q_FINAL); pure scheduling, so the results are bitwise those
    # of the plain per-layer steps
    w = synth.WORKLOADS[name]
    w = w.replace(T=(w.T // w.R) * w.R + w.R, steps=steps + w.R)
    data = synth.generate(w, q_steps=steps * len(tails))
    one, lens, k, v = _layers(w, tails, data)
    per, _, _, _ = _layers(w, tails, data)
    L = len(tails)
    q = data["q"].to(DEV)
    G = w.G
    all_outs = []
    for s in range(steps):
        qs = [q[s * L + l] for l in range(L)]
        kn = [k[:, :, lens[l] + s:lens[l] + s + 1] for l in range(L)]
        vn = [v[:, :, lens[l] + s:lens[l] + s + 1] for l in range(L)]
        outs = decode_step_layers(one, qs, kn, vn, overlap=overlap,
                                  q_final=overlap)
        all_outs.append(outs)
    torch.cuda.synchronize()
    for s in range(steps):
        qs = [q[s * L + l] for l in range(L)]
        kn = [k[:, :, lens[l] + s:lens[l] + s + 1] for l in range(L)]
        vn = [v[:, :, lens[l] + s:lens[l] + s + 1] for l in range(L)]
        outs = all_outs[s]
        refs = [per[l].step(qs[l], kn[l], vn[l]) for l in range(L)]
        torch.cuda.synchronize()
        for l in range(L):
            assert torch.equal(outs[l], refs[l]), (s, l)
    # after the last step every layer's streams equal the per-layer ones
    for l in range(L):
        a, b = one[l], per[l]
        assert (a.k.n_blocks, a.k.tail_len) == (b.k.n_blocks, b.k.tail_len)
        assert torch.equal(a.k.live_coeffs(), b.k.live_coeffs())
        assert torch.equal(a.v.live_scales(), b.v.live_scales())
        assert torch.equal(a.k.live_tail(), b.k.live_tail())
    # the last step of every layer against the oracle on its own archive
    s = steps - 1
    for l in range(L):
        c = one[l]
        got = f64(outs[l])
        ref = np.empty_like(got)
        qq = f64(q[s * L + l])
        for b in range(w.B):
            for h in range(w.Hk):
                ref[b:b + 1, h * G:(h + 1) * G] = \
                    oracle.decode_attention_reference(
                        qq[b:b + 1, h * G:(h + 1) * G], _dequant(c.k, b, h),
                        _dequant(c.v, b, h),
                        f64(c.k.live_tail()[b:b + 1, h:h + 1]),
                        f64(c.v.live_tail()[b:b + 1, h:h + 1]), w.R)
        check_out(got, ref, "%s layer %d" % (name, l))
    for c in one:
        assert _lib.fc_workspace_status(c._ws) == 0


def test_layers_reject_a_capacity_shortfall_without_touching_any_layer():
    w = synth.WORKLOADS["gqa"].replace(B=1, T=8 * 16 + 7, seed=77, steps=1)
    data = synth.generate(w, q_steps=1)
    k, v = data["k"].to(DEV), data["v"].to(DEV)
    caches = []
    for T in (8 * 15 + 2, w.T):
        c = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, device=DEV, capacity=16)
        c.prefill(k[:, :, :T], v[:, :, :T])
        caches.append(c)
    # layer 1 would complete a 17th block in its 16-block archive
    assert caches[1].k.n_blocks == caches[1].k.capacity == 16
    state = [(c.k.n_blocks, c.k.tail_len) for c in caches]
    q = data["q"][0].to(DEV)
    tok = (k[:, :, w.T:w.T + 1], v[:, :, w.T:w.T + 1])
    outs = [torch.empty((w.B, w.Hq, 1, w.D), device=DEV) for _ in caches]
    wss = [c.workspace(w.Hq, c.num_splits(w.Hq)) for c in caches]
    with pytest.raises(_lib.FcError) as e:
        _lib.fc_decode_step_layers(
            [q, q], [tok[0]] * 2, [tok[1]] * 2, [c.k.arc for c in caches],
            [c.v.arc for c in caches], [c.k.tail_desc for c in caches],
            [c.v.tail_desc for c in caches], outs, wss)
    assert e.value.status == _lib.FC_ERR_CAPACITY
    assert [(c.k.n_blocks, c.k.tail_len) for c in caches] == state
