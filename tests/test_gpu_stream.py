"""The streaming workload on the GPU: a bf16 prefill compressed into the int8
archive, then single-token decode steps crossing block boundaries, each
followed by decode attention; checked against the fp64 oracle replaying the
same appends."""

import numpy as np
import pytest
import torch

import oracle
import synth
from compressed_decode_attention_blockwise_b200 import CodecKVCache, _lib
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


def _twin_caches(w, data):
    caches = []
    for _ in range(2):
        c = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, device=DEV)
        c.prefill(data["k"][:, :, :w.T].to(DEV), data["v"][:, :, :w.T].to(DEV))
        caches.append(c)
    return caches


def _same_stream(a, b):
    assert (a.k.n_blocks, a.k.tail_len) == (b.k.n_blocks, b.k.tail_len)
    for sa, sb in ((a.k, b.k), (a.v, b.v)):
        assert torch.equal(sa.live_coeffs(), sb.live_coeffs())
        assert torch.equal(sa.live_scales(), sb.live_scales())
        assert torch.equal(sa.live_tail(), sb.live_tail())


@pytest.mark.parametrize("name,S,R,G", [("gqa-like", 2, 8, 4),
                                       ("long-like", 4, 16, 4),
                                       ("S8", 8, 16, 2)])
def test_fused_step_equals_append_then_attention(name, S, R, G):
    """fc_decode_step (one launch: append + attention) against fc_append_step
    followed by fc_decode_attention: the archive and tail bitwise, the
    outputs within rounding, across two block completions; every output
    against the oracle on the GPU's own archive."""
    w = synth.Workload("fstep", B=2, Hq=2 * G, Hk=2, D=128, T=R * 40 + R - 3,
                       R=R, S=S, seed=R + S, steps=2 * R + 1)
    data = synth.generate(w, q_steps=w.steps)
    k, v, q = data["k"].to(DEV), data["v"].to(DEV), data["q"].to(DEV)
    two, one = _twin_caches(w, data)
    for s in range(w.steps):
        t = w.T + s
        two.append(k[:, :, t:t + 1], v[:, :, t:t + 1])
        o2 = two.attention(q[s])
        o1 = one.step(q[s], k[:, :, t:t + 1], v[:, :, t:t + 1],
                      overlap=s % 3 == 1, q_final=s % 3 == 2)
        torch.cuda.synchronize()
        _same_stream(two, one)
        # the fused launch folds the new token or block on the CUDA cores in
        # fp32, the two-launch path through the tensor-core limbs: rounding
        # apart, the same value (the oracle check below is the bar)
        diff = (o1 - o2).abs().max().item()
        assert diff <= 2e-4, (s, diff)
        check_out(f64(o1), oracle_on_gpu_archive(one, q[s]), "step %d" % s)


def test_fused_step_in_a_graph_and_portable_path():
    """Steps captured in a CUDA graph give what eager steps give; the
    portable flag (two launches) matches too, as does a stream that starts
    with no archived block (two launches until the first block exists)."""
    w = synth.Workload("fstep", B=1, Hq=8, Hk=2, D=128, T=8 * 30 + 2, R=8, S=2,
                       seed=5, steps=20)
    data = synth.generate(w, q_steps=w.steps)
    k, v, q = data["k"].to(DEV), data["v"].to(DEV), data["q"].to(DEV)
    eager, graphed = _twin_caches(w, data)
    cap = (w.T + w.steps) // w.R + 1
    eager._grow_to(cap)
    graphed._grow_to(cap)
    outs_e = [eager.step(q[s], k[:, :, w.T + s:w.T + s + 1],
                         v[:, :, w.T + s:w.T + s + 1]) for s in range(w.steps)]
    outs_g = [torch.empty_like(outs_e[0]) for _ in range(w.steps)]
    graphed.workspace(w.Hq, graphed.num_splits(w.Hq))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for s in range(w.steps):
            graphed.step(q[s], k[:, :, w.T + s:w.T + s + 1],
                         v[:, :, w.T + s:w.T + s + 1], out=outs_g[s],
                         overlap=True, q_final=True)
    g.replay()
    torch.cuda.synchronize()
    _same_stream(eager, graphed)
    for a, b in zip(outs_e, outs_g):
        assert torch.equal(a, b)
    # portable (append + CUDA-core attention) from an empty cache
    port = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, device=DEV)
    ref = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, device=DEV)
    for s in range(2 * w.R + 3):
        kt, vt = k[:, :, s:s + 1], v[:, :, s:s + 1]
        o_port = port.step(q[s % w.steps], kt, vt, portable=True)
        ref.append(kt, vt)
        o_ref = ref.attention(q[s % w.steps], portable=True)
        torch.cuda.synchronize()
        assert torch.equal(o_port, o_ref)
    _same_stream(port, ref)


@pytest.mark.parametrize("name", ["long", "stream"])
def test_benchmarked_decode_step_at_full_size(name):
    """fc_decode_step exactly as the benchmark times it: the full-size
    workload, the planner's split count (18 chunks per kv head on `long`), the
    fused combine, FC_DECODE_OVERLAP | FC_DECODE_Q_FINAL, the steps captured
    in a CUDA graph and replayed, R + 1 steps so that one of them completes a
    block (encoded in the kernel). The archive and tail end bitwise equal to
    those of fc_append_step + fc_decode_attention, and every output element of
    every step is checked against the fp64 oracle on the GPU's own archive
    (the archive of step s is the first n_blocks(s) blocks of the final one,
    which no step rewrites; its raw tail is the input tokens after them)."""
    w = synth.WORKLOADS[name]
    steps = w.R + 1
    data = synth.generate(w.replace(steps=steps), q_steps=steps)
    k, v, q = data["k"].to(DEV), data["v"].to(DEV), data["q"].to(DEV)
    graphed, two = _twin_caches(w, data)
    cap = (w.T + steps) // w.R + 1
    for c in (graphed, two):
        c._grow_to(cap)
    ns = graphed.num_splits(w.Hq)
    if name == "long":
        assert ns == _lib.fc_decode_plan(graphed.k.arc, graphed.k.tail_desc,
                                         w.Hq) and ns > 8
    graphed.workspace(w.Hq, ns)
    outs = [torch.full((w.B, w.Hq, 1, w.D), float("nan"), device=DEV)
            for _ in range(steps)]
    state = []                            # (n_blocks, tail_len) after step s
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for s in range(steps):
            t = w.T + s
            graphed.step(q[s], k[:, :, t:t + 1], v[:, :, t:t + 1],
                         out=outs[s], overlap=True, q_final=True)
            state.append((graphed.k.n_blocks, graphed.k.tail_len))
    g.replay()
    torch.cuda.synchronize()
    assert any(nr == 0 for _, nr in state)          # a block was completed
    two_outs = []
    for s in range(steps):
        t = w.T + s
        two.append(k[:, :, t:t + 1], v[:, :, t:t + 1])
        two_outs.append(two.attention(q[s]))
    torch.cuda.synchronize()
    _same_stream(graphed, two)
    assert _lib.fc_workspace_status(graphed._ws) == 0
    # the oracle at every step, over the final archive's prefix
    ck_all = {}
    for (b, h) in [(b, h) for b in range(w.B) for h in range(w.Hk)]:
        ck_all[(b, h)] = (_dequant(graphed.k, b, h), _dequant(graphed.v, b, h))
    G = w.G
    for s, (nb, nr) in enumerate(state):
        got = f64(outs[s])
        assert np.isfinite(got).all()
        ref = np.empty_like(got)
        t_end = w.T + s + 1
        for (b, h), (ck, cv) in ck_all.items():
            tk = f64(data["k"][b:b + 1, h:h + 1, nb * w.R:t_end])
            tv = f64(data["v"][b:b + 1, h:h + 1, nb * w.R:t_end])
            assert tk.shape[2] == nr
            ref[b:b + 1, h * G:(h + 1) * G] = oracle.decode_attention_reference(
                f64(q[s][b:b + 1, h * G:(h + 1) * G]), ck[:, :, :nb],
                cv[:, :, :nb], tk, tv, w.R)
        check_out(got, ref, "%s step %d" % (name, s))
        # the fused step folds the new token (or the block it completes)
        # together with the raw tail, the plain attention launch reads it from
        # the tail or the archive: different summation orders over 131k tokens
        diff = (outs[s] - two_outs[s]).abs().max().item()
        assert diff <= 2e-5 * float(np.abs(ref).max()) + 1e-4, (s, diff)


def _dequant(stream, b, h):
    c = stream.coeffs[b:b + 1, h:h + 1, :stream.n_blocks].cpu().numpy()
    sc = stream.scales[b:b + 1, h:h + 1, :stream.n_blocks].cpu().numpy()
    return oracle.dequantize(c, sc)


@pytest.mark.parametrize("pinned", [True, False], ids=["pinned", "pageable"])
def test_host_buffer_step_equals_device_step(pinned):
    """fc_decode_step_host (inputs from one host block, output to host
    memory; pinned buffers are read and written by the kernels in place,
    pageable ones go through the staging copies) gives the archive, tail and
    output of fc_decode_step on device copies of the same inputs, across a
    block completion."""
    w = synth.Workload("hstep", B=2, Hq=8, Hk=2, D=128, T=8 * 50 + 5, R=8,
                       S=2, seed=17, steps=6)
    data = synth.generate(w, q_steps=w.steps)
    dev_cache, host_cache = _twin_caches(w, data)
    for c in (dev_cache, host_cache):
        c._grow_to((w.T + w.steps) // w.R + 1)
    nk, nq = w.B * w.Hk * w.D, w.B * w.Hq * w.D
    staging = torch.empty(_lib.fc_decode_step_staging_bytes(
        w.B, w.Hk, w.Hq, w.D, torch.bfloat16, torch.float32),
        dtype=torch.uint8, device=DEV)
    ws = host_cache.workspace(w.Hq, host_cache.num_splits(w.Hq))
    for s in range(w.steps):
        t = w.T + s
        blk = torch.empty(2 * nk + nq, dtype=torch.bfloat16, pin_memory=pinned)
        blk[:nk] = data["k"][:, :, t].reshape(-1)
        blk[nk:2 * nk] = data["v"][:, :, t].reshape(-1)
        blk[2 * nk:] = data["q"][s].reshape(-1)
        out_h = torch.empty((w.B, w.Hq, 1, w.D), pin_memory=pinned)
        _lib.HostStep(host_cache, w.Hq, blk, out_h, staging, ws)()
        torch.cuda.synchronize()
        ref = dev_cache.step(data["q"][s].to(DEV),
                             data["k"][:, :, t:t + 1].to(DEV),
                             data["v"][:, :, t:t + 1].to(DEV))
        torch.cuda.synchronize()
        _same_stream(dev_cache, host_cache)
        assert torch.equal(out_h, ref.cpu())
