"""Host bookkeeping of the device cache binding (``archive.py``) on the CPU:
libfc's launching calls are replaced by host fakes that only advance the
descriptors as ``include/fc.h`` / ``include/fc_view.h`` document, so the
memoised view (which blocks each read decodes, buffer growth), crop, batch
gather (new storage, cleared plans) and reset are checked without a kernel."""

import pytest
import torch

from compressed_decode_attention_blockwise_b200 import _lib
from compressed_decode_attention_blockwise_b200.archive import CodecKVCache


class FakeLib:
    """Descriptor-level stand-ins for the calls archive.py makes."""

    def __init__(self):
        self.reads = []      # (first_block, n_blocks, tail len, out rows, ptr)
        self.gathers = []

    def fc_compress_blocks(self, x, arc, tail=None, stream=None):
        T = x.shape[2]
        if arc.n_blocks + T // arc.R > arc.capacity:
            raise _lib.FcError(_lib.FC_ERR_CAPACITY, "fc_compress_blocks")
        arc.n_blocks += T // arc.R
        if tail is not None:
            tail.len = T % arc.R

    def fc_append_step(self, k, v, ka, va, kt, vt, stream=None):
        if kt.len + 1 == ka.R:
            if ka.n_blocks == ka.capacity:
                raise _lib.FcError(_lib.FC_ERR_CAPACITY, "fc_append_step")
            ka.n_blocks += 1
            va.n_blocks += 1
            kt.len = vt.len = 0
        else:
            kt.len += 1
            vt.len += 1

    def fc_archive_copy_prefix(self, src, dst, stream=None, device=None):
        assert dst.capacity >= src.n_blocks
        dst.n_blocks = src.n_blocks

    def fc_read_view(self, arc, tail, first_block, out, stream=None):
        n_raw = 0 if tail is None else tail.len
        assert 0 <= first_block <= arc.n_blocks
        assert out.shape[2] >= arc.n_blocks * arc.R + n_raw
        self.reads.append((first_block, arc.n_blocks, n_raw, out.shape[2],
                           out.data_ptr()))
        # marker values: block n's rows hold n + 1, raw token i holds -(i + 1)
        for n in range(first_block, arc.n_blocks):
            out[:, :, n * arc.R:(n + 1) * arc.R] = n + 1
        for i in range(n_raw):
            out[:, :, arc.n_blocks * arc.R + i] = -(i + 1)

    def fc_crop(self, arc, tail, tokens_to_remove, stream=None, device=None):
        assert tokens_to_remove <= 0
        keep = max(0, arc.n_blocks * arc.R + tail.len + tokens_to_remove)
        kb, rest = divmod(keep, arc.R)
        arc.n_blocks = min(arc.n_blocks, kb)
        tail.len = rest

    def fc_select_batch(self, src, src_tail, idx, dst, dst_tail, stream=None,
                        device=None):
        assert all(0 <= i < src.B for i in idx) and dst.B == len(idx)
        assert dst.capacity >= src.n_blocks
        self.gathers.append(list(idx))
        dst.n_blocks = src.n_blocks
        dst_tail.len = src_tail.len


@pytest.fixture
def fake(monkeypatch):
    f = FakeLib()
    for name in ("fc_compress_blocks", "fc_append_step",
                 "fc_archive_copy_prefix", "fc_read_view", "fc_crop",
                 "fc_select_batch"):
        monkeypatch.setattr(_lib, name, getattr(f, name))
    return f


def _cache(B=2, H=2, D=32, R=8):
    return CodecKVCache(B, H, D, R, 2, device="cpu")


def _tokens(c, T):
    return (torch.zeros((c.B, c.Hk, T, c.D), dtype=torch.bfloat16),
            torch.zeros((c.B, c.Hk, T, c.D), dtype=torch.bfloat16))


def test_view_decodes_each_block_once_and_grows_by_doubling(fake):
    c = _cache()
    assert c.read() == (None, None)                 # empty: nothing to read
    c.prefill(*_tokens(c, 5))
    kv, vv = c.read()                               # tail only: the tail itself
    assert kv.shape == (2, 2, 5, 32) and not fake.reads
    c.prefill(*_tokens(c, 8 * 14 + 6))              # 15 blocks + 3 raw
    kv, vv = c.read()
    assert kv.shape[2] == vv.shape[2] == 8 * 15 + 3
    assert fake.reads[-4][:4] == (0, 15, 0, 16 * 8)   # K's blocks: 16-block buffer
    assert fake.reads[-3][:4] == (15, 15, 3, 123)     # K's tail: a fresh tensor
    ptr = fake.reads[-4][4]
    kv = c.k.read()                                 # nothing new to decode
    assert fake.reads[-1][:4] == (15, 15, 3, 123) and fake.reads[-1][4] != ptr
    n = len(fake.reads)
    for _ in range(5):                              # completes block 16
        c.append(*_tokens(c, 1))
    view = c.k.read()
    assert fake.reads[n:] == [(15, 16, 0, 128, ptr)]  # only the new block
    assert view.data_ptr() == ptr and view.shape[2] == 128
    c.append(*_tokens(c, 1))                        # 129 tokens: one raw
    view = c.k.read()
    assert view.shape[2] == 129
    assert fake.reads[-1][:4] == (16, 16, 1, 129)   # tail rows only
    for _ in range(7):                              # 17 blocks > 16 in the buffer
        c.append(*_tokens(c, 1))
    view = c.k.read()
    assert fake.reads[-1][:4] == (0, 17, 0, 256)    # doubled, decoded afresh
    assert fake.reads[-1][4] != ptr


def test_view_handed_out_earlier_keeps_its_tail_rows(fake):
    """A read with raw tokens returns a fresh tensor: when those tokens are
    archived later, the earlier tensor still holds the raw rows
    (flashcodec/cache.py, _CodecStream.read)."""
    c = _cache()
    c.prefill(*_tokens(c, 8 * 15 + 3))
    early = c.k.read()
    assert early[0, 0, 120:123, 0].tolist() == [-1, -2, -3]
    for _ in range(5):                              # archives tokens 120..127
        c.append(*_tokens(c, 1))
    later = c.k.read()
    assert later[0, 0, 120:128, 0].tolist() == [16] * 8
    assert early[0, 0, 120:123, 0].tolist() == [-1, -2, -3]
    assert early[0, 0, :120, 0].tolist() == later[0, 0, :120, 0].tolist()


def test_crop_rewinds_the_memoised_view(fake):
    c = _cache()
    c.prefill(*_tokens(c, 8 * 20 + 5))
    c.read()
    with pytest.raises(ValueError):
        c.crop(3)
    c.crop(-2)                                      # tail only
    assert (c.k.n_blocks, c.k.tail_len, c.k._rec_blocks) == (20, 3, 20)
    c.crop(-30)                                     # 133 tokens: 16 blocks + 5
    assert (c.k.n_blocks, c.k.tail_len, c.v.tail_len) == (16, 5, 5)
    assert c.k._rec_blocks == 16
    c.k.read()
    assert fake.reads[-1][:3] == (16, 16, 5)        # tail rows only
    c.crop(-1000)
    assert c.seq_len == 0 and c.read() == (None, None)


def test_batch_gather_replaces_storage_and_plans(fake):
    c = _cache(B=3)
    c.prefill(*_tokens(c, 8 * 20 + 5))
    c.read()
    c._plans[(8, 20)] = 4
    c._ws_need[(8, 4)] = 1 << 20
    cap = c.k.capacity
    old_ptr = c.k.coeffs.data_ptr()
    c.reorder_cache(torch.tensor([2, 0, 2, 1]))
    assert fake.gathers[-2:] == [[2, 0, 2, 1], [2, 0, 2, 1]]   # K and V
    assert c.B == c.k.B == c.v.B == 4
    assert c.k.coeffs.shape == (4, 2, cap, 2, 32) and c.k.capacity == cap
    assert c.k.scales.shape == (4, 2, cap, 2)
    assert c.k.tail.shape == (4, 2, 8, 32)
    assert c.k.arc.coeffs == c.k.coeffs.data_ptr() != old_ptr
    assert c.k.tail_desc.data == c.k.tail.data_ptr()
    assert (c.k.n_blocks, c.k.tail_len) == (20, 5)
    assert c.k._rec is None and not c._plans and not c._ws_need
    c.batch_select_indices([3, 0])
    assert c.B == 2 and fake.gathers[-1] == [3, 0]
    c.batch_repeat_interleave(3)
    assert c.B == 6 and fake.gathers[-1] == [0, 0, 0, 1, 1, 1]
    kv, vv = c.read()
    assert kv.shape == (6, 2, 165, 32)
    assert fake.reads[-4][:2] == (0, 20)            # rebuilt from block 0


def test_reset_keeps_capacity_and_update_returns_the_view(fake):
    c = _cache()
    c.prefill(*_tokens(c, 8 * 40 + 1))
    c.read()
    cap = c.k.capacity
    c.reset()
    assert (c.seq_len, c.k.capacity, c.k._rec_blocks) == (0, cap, 0)
    kv, vv = c.update(*_tokens(c, 8 * 3 + 2))
    assert kv.shape == (2, 2, 26, 32) and c.get_seq_length() == 26
    assert fake.reads[-4][:3] == (0, 3, 0)          # K's blocks from block 0
    assert fake.reads[-3][:3] == (3, 3, 2)          # then its tail rows



def test_failed_gather_leaves_the_cache_unchanged(fake, monkeypatch):
    c = _cache(B=3)
    c.prefill(*_tokens(c, 8 * 5 + 2))
    k_arc, v_arc = c.k.arc, c.v.arc
    calls = []

    def failing(src, src_tail, idx, dst, dst_tail, stream=None, device=None):
        calls.append(idx)
        if len(calls) == 2:                         # the V stream
            raise _lib.FcError(_lib.FC_ERR_CUDA, "fc_select_batch")
        dst.n_blocks = src.n_blocks
        dst_tail.len = src_tail.len

    monkeypatch.setattr(_lib, "fc_select_batch", failing)
    with pytest.raises(_lib.FcError):
        c.reorder_cache([1, 0])
    assert c.B == c.k.B == c.v.B == 3
    assert c.k.arc is k_arc and c.v.arc is v_arc
    assert c.k.coeffs.shape[0] == c.v.coeffs.shape[0] == 3


def test_failed_crop_leaves_both_streams_as_they_were(fake, monkeypatch):
    c = _cache()
    c.prefill(*_tokens(c, 8 * 6 + 5))
    c.k.tail.fill_(3.0)
    calls = []

    def failing(arc, tail, tokens_to_remove, stream=None, device=None):
        calls.append(tokens_to_remove)
        if len(calls) == 2:                         # the V stream
            raise _lib.FcError(_lib.FC_ERR_CUDA, "fc_crop")
        fake.fc_crop(arc, tail, tokens_to_remove)
        c.k.tail.fill_(7.0)                         # the boundary rows rewritten

    monkeypatch.setattr(_lib, "fc_crop", failing)
    with pytest.raises(_lib.FcError):
        c.crop(-9)
    assert (c.k.n_blocks, c.k.tail_len) == (c.v.n_blocks, c.v.tail_len) == (6, 5)
    assert torch.all(c.k.tail == 3.0)
    with pytest.raises(ValueError):
        c.crop(1)


def test_a_step_that_grows_the_archive_runs_without_the_overlap_flags(
        fake, monkeypatch):
    """FC_DECODE_OVERLAP lets the kernel stream archive blocks before the
    preceding stream work has finished; a growth copy (which writes every
    block of the new storage) right before the step would break that, so
    the binding drops the flags for that one step, for single steps and for
    the multi-layer launch."""
    from compressed_decode_attention_blockwise_b200.archive import \
        decode_step_layers
    calls = []

    def fake_step(q, k_new, v_new, ka, va, kt, vt, out, ws, softmax_scale=0.0,
                  num_splits=0, fuse_combine=True, portable=False,
                  overlap=False, q_final=False, stream=None):
        calls.append((int(ka.capacity), overlap, q_final))
        fake.fc_append_step(k_new, v_new, ka, va, kt, vt)

    def fake_layers(qs, k_news, v_news, kas, vas, kts, vts, outs, wss,
                    softmax_scale=0.0, num_splits=0, fuse_combine=True,
                    overlap=False, q_final=False, stream=None):
        calls.append((tuple(int(a.capacity) for a in kas), overlap, q_final))
        for i in range(len(kas)):
            fake.fc_append_step(k_news[i], v_news[i], kas[i], vas[i], kts[i],
                                vts[i])

    monkeypatch.setattr(_lib, "fc_decode_step", fake_step)
    monkeypatch.setattr(_lib, "fc_decode_step_layers", fake_layers)
    monkeypatch.setattr(_lib, "fc_decode_plan", lambda ka, kt, Hq: 1)
    monkeypatch.setattr(_lib, "fc_decode_workspace_bytes",
                        lambda B, Hq, D, ns: 1024)
    c = _cache()                                    # R = 8
    c.prefill(*_tokens(c, 8 * 16 + 6))              # 16 blocks fill capacity 16
    assert c.k.capacity == 16
    q = torch.zeros((c.B, 4, 1, c.D))
    tok = _tokens(c, 1)
    for _ in range(3):                              # the second completes block 17
        c.step(q, *tok, overlap=True, q_final=True)
    assert calls == [(16, True, True), (32, False, False), (32, True, True)]
    calls.clear()
    a, b = _cache(), _cache()
    for x in (a, b):
        x.prefill(*_tokens(x, 8 * 16 + 7))
    for _ in range(2):                              # the first completes a block
        decode_step_layers([a, b], [q, q], [tok[0]] * 2, [tok[1]] * 2,
                           overlap=True, q_final=True)
    assert calls == [((32, 32), False, False), ((32, 32), True, True)]
