"""The allocation-free decode-attention entry point, through the C ABI.

fc_decode_attention_noalloc serves callers that cannot hand the library a
workspace (a C host inside a fixed device-memory budget without an allocator,
or a serving loop that must not call cudaMalloc per step). It must give the
same result as fc_decode_attention with a caller workspace, call after call
(the static scratch it shares between calls keeps the previous call's bytes),
and reject requests larger than its scratch; the status word of that
scratch stays readable through fc_noalloc_status. This file is collected last so
that a run stopping at the first failure has already run every other test.
"""

import ctypes

import pytest
import torch

import synth
from compressed_decode_attention_blockwise_b200 import CodecKVCache, _lib
from _helpers import check_out, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.mark.parametrize("w", [
    synth.WORKLOADS["gqa"].replace(B=2, T=8 * 300 + 5, seed=31),
    synth.WORKLOADS["long"].replace(T=16 * 4096 + 3, seed=32),
    synth.WORKLOADS["tiny"],
], ids=["gqa-small", "long-half", "tiny"])
def test_noalloc_matches_workspace_entry_point(w):
    data = synth.generate(w, q_steps=0)
    cache = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                         token_dtype=synth.torch_dtype(w.in_dtype), device=DEV)
    cache.prefill(data["k"].to(DEV), data["v"].to(DEV))
    q = data["q"].to(DEV)
    ref = cache.attention(q)                       # caller workspace
    torch.cuda.synchronize()
    for _ in range(2):                             # two calls in a row
        out = torch.full_like(ref, float("nan"))
        _lib.fc_decode_attention_noalloc(q, cache.k.arc, cache.v.arc,
                                         cache.k.tail_desc, cache.v.tail_desc,
                                         out)
        torch.cuda.synchronize()
        check_out(f64(out), f64(ref), "noalloc vs workspace")
        # no kernel reported an error in the scratch's status word, which
        # the calls themselves never clear (reading it does)
        assert _lib.fc_noalloc_status() == 0


def test_noalloc_rejects_requests_beyond_its_scratch():
    cache = CodecKVCache(64, 8, 128, 8, 2, device=DEV)
    x = torch.randn(64, 8, 8 * 40, 128, dtype=torch.bfloat16, device=DEV)
    cache.prefill(x, x)
    q = torch.randn(64, 64, 1, 128, dtype=torch.bfloat16, device=DEV)
    out = torch.empty((64, 64, 1, 128), device=DEV)
    need = _lib.fc_decode_workspace_bytes(64, 64, 128, 40)
    assert need > _lib.FC_NOALLOC_SCRATCH_BYTES
    with pytest.raises(_lib.FcError) as e:
        _lib.fc_decode_attention_noalloc(q, cache.k.arc, cache.v.arc,
                                         cache.k.tail_desc, cache.v.tail_desc,
                                         out, num_splits=40)
    assert e.value.status == _lib.FC_ERR_SCRATCH_LIMIT
