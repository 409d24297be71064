"""The tensor-core decode kernel's error path, made to run without a GPU
fault: FC_DECODE_TEST_TIMEOUT makes every CTA wait on a barrier phase that
nothing completes, with a short limit. The wait runs out, the kernel records
the error in the workspace status word, stops, drains what it issued, frees
its TMEM and returns; the host reads FC_ERR_DEVICE, and the next normal call
on the same workspace matches the oracle."""

import pytest
import torch

import synth
from compressed_decode_attention_blockwise_b200 import CodecKVCache, _lib
from _helpers import check_out, f64, oracle_on_gpu_archive

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.mark.parametrize("ns", [2, 0])
def test_timed_out_wait_is_reported_and_the_workspace_recovers(ns):
    # 300 blocks of R=16, S=4 (10 coefficient tiles per kv head) and a
    # 3-token tail: every CTA has tiles in flight when the wait gives up
    w = synth.Workload("timeout", B=1, Hq=32, Hk=8, D=128, T=300 * 16 + 3,
                       R=16, S=4, k_coeff="i8", v_coeff="i8",
                       in_dtype="bf16", seed=41)
    data = synth.generate(w, q_steps=0)
    cache = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                         token_dtype=torch.bfloat16, device=DEV)
    cache.prefill(data["k"][:, :, :w.T].to(DEV), data["v"][:, :, :w.T].to(DEV))
    assert cache.tensor_core_path(w.Hq)
    q = data["q"].to(DEV)
    splits = ns or cache.num_splits(w.Hq)
    ws = cache.workspace(w.Hq, splits)
    assert _lib.fc_workspace_status(ws) == 0
    out = torch.empty((w.B, w.Hq, 1, w.D), dtype=torch.float32, device=DEV)

    _lib.fc_decode_attention(q, cache.k.arc, cache.v.arc, cache.k.tail_desc,
                             cache.v.tail_desc, out, ws, num_splits=ns,
                             test_timeout=True)
    torch.cuda.synchronize()  # the context is still usable
    assert _lib.fc_workspace_status(ws) != 0
    assert _lib.fc_workspace_status(ws) == 0  # the read cleared it

    ref = oracle_on_gpu_archive(cache, q)
    for _ in range(2):
        out.fill_(float("nan"))
        _lib.fc_decode_attention(q, cache.k.arc, cache.v.arc,
                                 cache.k.tail_desc, cache.v.tail_desc, out, ws,
                                 num_splits=ns)
        torch.cuda.synchronize()
        assert _lib.fc_workspace_status(ws) == 0
        check_out(f64(out), ref)
