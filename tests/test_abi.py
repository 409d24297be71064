"""The C-ABI library on the host: it loads, exports every declared symbol,
and its host-only logic (validation, workspace sizing, storage accounting)
behaves; no kernel is launched here."""

import ctypes
import json
import os
import re
from decimal import Decimal, ROUND_HALF_UP

import pytest

from compressed_decode_attention_blockwise_b200 import _lib
from compressed_decode_attention_blockwise_b200.archive import grown_capacity
from oracle.stream import grown_capacity as oracle_grown_capacity

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
FAKE = 0x10000  # aligned non-null address; never dereferenced here


def declared_functions():
    names = set()
    for fn in sorted(os.listdir(INCLUDE)):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(INCLUDE, fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names.update(re.findall(
            r"^\s*(?:const\s+)?[A-Za-z_0-9]+\s*\*?\s+(fc_[a-z_0-9]+)\s*\(",
            src, flags=re.M))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = declared_functions()
    assert len(names) == len(_lib.EXPORTS), names
    assert sorted(names) == sorted(_lib.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for code in range(7):
        assert _lib.fc_status_string(code)
    assert "unknown" in _lib.fc_status_string(99)


def _arc(B=1, H=8, D=64, R=8, S=2, dtype=_lib.FC_DTYPE_I8, cap=16, nb=0):
    a = _lib.FcArchive()
    a.coeffs = FAKE
    a.scales = FAKE if dtype == _lib.FC_DTYPE_I8 else None
    a.coeff_dtype = dtype
    a.R, a.S = R, S
    a.B, a.H, a.D = B, H, D
    a.capacity, a.n_blocks = cap, nb
    a.coeff_stride_h = cap * S * D
    a.coeff_stride_b = H * a.coeff_stride_h
    a.scale_stride_h = cap * S
    a.scale_stride_b = H * a.scale_stride_h
    return a


def _tail(a, length=0, dtype=_lib.FC_DTYPE_BF16):
    t = _lib.FcTail()
    t.data = FAKE
    t.dtype = dtype
    t.len = length
    t.stride_h = a.R * a.D
    t.stride_b = a.H * t.stride_h
    return t


def test_storage_bytes_matches_oracle_and_pages():
    """libfc's storage accounting reproduces the README's cache-footprint
    table (B*H*D = 512 fp32 streams, r = 8, K and V)."""
    with open(os.path.join(ROOT, "tests", "golden",
                           "storage_footprint.json")) as f:
        gold = json.load(f)
    for row in gold["rows"]:
        dt = _lib.FC_DTYPE_I8 if row["quant_bits"] == 8 else _lib.FC_DTYPE_F32
        nb = row["seq"] // 8
        a = _arc(B=1, H=8, D=64, R=8, S=row["keep"], dtype=dt, cap=nb, nb=nb)
        total = 2 * _lib.fc_storage_bytes(a, _tail(a, 0, _lib.FC_DTYPE_F32))
        mb = Decimal(repr(total / 2 ** 20)).quantize(Decimal("0.1"),
                                                     ROUND_HALF_UP)
        assert str(mb) == row["storage"], row
    # raw tail tokens count at the input precision
    a = _arc(nb=3)
    assert _lib.fc_storage_bytes(a, _tail(a, 5)) == \
        _lib.fc_storage_bytes(a, None) + 1 * 8 * 5 * 64 * 2


def test_workspace_bytes():
    n = _lib.fc_decode_workspace_bytes(2, 8, 128, 3)
    rows = 2 * 8 * 3
    pad = lambda x: (x + 255) // 256 * 256
    assert n == 256 + pad(2 * 8 * 4) + 2 * pad(rows * 4) + pad(rows * 128 * 4)
    assert _lib.fc_decode_workspace_bytes(0, 8, 128, 3) == 0


def test_validation_rejects_bad_arguments_without_launching():
    lib = _lib.load()
    a = _arc()
    t = _tail(a)
    strides = (ctypes.c_int64 * 4)(8 * 100 * 64, 100 * 64, 64, 1)
    # null input
    assert lib.fc_compress_blocks(None, _lib.FC_DTYPE_BF16, strides, 100,
                                  ctypes.byref(a), None, None) == \
        _lib.FC_ERR_INVALID
    # capacity: 100 tokens = 12 blocks > 4 free blocks
    small = _arc(cap=4)
    assert lib.fc_compress_blocks(FAKE, _lib.FC_DTYPE_BF16, strides, 100,
                                  ctypes.byref(small), None, None) == \
        _lib.FC_ERR_CAPACITY
    assert small.n_blocks == 0
    # unsupported head dim, S > R, S above the supported maximum
    for bad, code in ((_arc(D=100), _lib.FC_ERR_UNSUPPORTED),
                      (_arc(R=4, S=5), _lib.FC_ERR_INVALID),
                      (_arc(R=32, S=17), _lib.FC_ERR_UNSUPPORTED)):
        assert lib.fc_compress_blocks(FAKE, _lib.FC_DTYPE_BF16, strides, 100,
                                      ctypes.byref(bad), None, None) == code
    # int8 archive without scales
    noscale = _arc()
    noscale.scales = None
    assert lib.fc_storage_bytes(ctypes.byref(noscale), None) == -1
    # misaligned coefficient pointer
    mis = _arc()
    mis.coeffs = FAKE + 4
    assert lib.fc_storage_bytes(ctypes.byref(mis), None) == -1
    # decode: Hq not a multiple of Hk, unsupported group size, empty input
    q_str = (ctypes.c_int64 * 4)(12 * 64, 64, 64, 1)
    ws = ctypes.c_void_p(FAKE)

    def attn(Hq, ka, kt=None, vt=None, ns=0):
        return lib.fc_decode_attention(
            FAKE, _lib.FC_DTYPE_BF16, q_str, Hq, ctypes.byref(ka),
            ctypes.byref(ka), None if kt is None else ctypes.byref(kt),
            None if vt is None else ctypes.byref(vt), 0.0, ns, 1, ws,
            1 << 30, FAKE, _lib.FC_DTYPE_F32, q_str, None)

    full = _arc(nb=5)
    assert attn(12, full) == _lib.FC_ERR_INVALID          # 12 % 8
    assert attn(8 * 3, full) == _lib.FC_ERR_UNSUPPORTED   # G = 3
    assert attn(8, _arc(nb=0)) == _lib.FC_ERR_INVALID     # nothing to attend
    assert attn(8, full, _tail(full, 1), None) == _lib.FC_ERR_INVALID
    assert attn(8, full, ns=10000) == _lib.FC_ERR_INVALID
    # combine: workspace too small
    out_str = (ctypes.c_int64 * 4)(8 * 64, 64, 64, 1)
    assert lib.fc_combine(FAKE, 16, 1, 8, 64, 4, FAKE, _lib.FC_DTYPE_F32,
                          out_str, None) == _lib.FC_ERR_INVALID


def test_decode_step_validates_without_launching():
    """fc_decode_step checks the append and the attention arguments on the
    host: missing token or tails, capacity (nothing written), bad flags."""
    s4 = lambda *x: (ctypes.c_int64 * 4)(*x)
    q_str = s4(8 * 64, 64, 64, 1)
    tok = s4(2 * 64, 64, 64, 1)
    ka, va = _arc(H=2, cap=2, nb=2), _arc(H=2, cap=2, nb=2)
    kt, vt = _tail(ka, 7), _tail(va, 7)

    def step(k_new=FAKE, flags=1, kt_=kt, vt_=vt):
        return _lib.load().fc_decode_step(
            FAKE, _lib.FC_DTYPE_BF16, q_str, 8, k_new, FAKE, _lib.FC_DTYPE_BF16,
            tok, tok, ctypes.byref(ka), ctypes.byref(va),
            None if kt_ is None else ctypes.byref(kt_),
            None if vt_ is None else ctypes.byref(vt_), 0.0, 0, flags,
            FAKE, 1 << 30, FAKE, _lib.FC_DTYPE_F32, q_str, None)

    assert step(k_new=None) == _lib.FC_ERR_INVALID
    assert step(kt_=None) == _lib.FC_ERR_INVALID
    assert step(flags=1 << 8) == _lib.FC_ERR_INVALID
    assert step(flags=1 | _lib.FC_DECODE_TEST_TIMEOUT) == _lib.FC_ERR_INVALID
    assert step() == _lib.FC_ERR_CAPACITY        # the token completes block 3
    assert (ka.n_blocks, kt.len, vt.len) == (2, 7, 7)


def test_append_capacity_error_leaves_state():
    lib = _lib.load()
    ka, va = _arc(cap=2, nb=2), _arc(cap=2, nb=2)
    kt, vt = _tail(ka, 7), _tail(va, 7)
    s = (ctypes.c_int64 * 4)(8 * 64, 64, 64, 1)
    st = lib.fc_append_step(FAKE, FAKE, _lib.FC_DTYPE_BF16, s, s,
                            ctypes.byref(ka), ctypes.byref(va),
                            ctypes.byref(kt), ctypes.byref(vt), None)
    assert st == _lib.FC_ERR_CAPACITY
    assert (ka.n_blocks, kt.len, vt.len) == (2, 7, 7)
    # mismatched tail lengths
    vt.len = 6
    st = lib.fc_append_step(FAKE, FAKE, _lib.FC_DTYPE_BF16, s, s,
                            ctypes.byref(ka), ctypes.byref(va),
                            ctypes.byref(kt), ctypes.byref(vt), None)
    assert st == _lib.FC_ERR_INVALID


@pytest.mark.parametrize("cap,need", [(0, 1), (0, 16), (16, 17), (32, 100),
                                      (128, 100), (0, 1000)])
def test_capacity_policy_matches_oracle(cap, need):
    assert grown_capacity(cap, need) == oracle_grown_capacity(cap, need)


def test_product_path_has_no_oracle_or_fallback():
    """The package never imports the oracle and has no CPU compute path."""
    pkg = os.path.join(ROOT, "compressed_decode_attention_blockwise_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "oracle" not in src, fn
            assert "numpy" not in src, fn


def test_split_planner():
    """fc_decode_plan on the host (148 SMs: the B200 count, also the
    fallback when no device is visible). Tensor-core shapes (int8, D = 128):
    one CTA per SM over the (b, kv head) pairs, rounded down, at most one
    split per 128-row tile. Other shapes: four CTAs per SM rounded down to
    one wave, at least 16 blocks per split."""
    def plan(B, H, D, R, S, nb, Hq, dt=_lib.FC_DTYPE_I8):
        a = _arc(B=B, H=H, D=D, R=R, S=S, dtype=dt, cap=nb, nb=nb)
        return _lib.fc_decode_plan(a, None, Hq)

    assert plan(1, 8, 128, 16, 4, 8192, 32) == 18      # long: 144 CTAs
    assert plan(1, 8, 128, 16, 4, 40, 32) == 2         # capped by 2 tiles
    assert plan(8, 8, 128, 8, 2, 512, 32) == 2         # gqa: 64 pairs
    assert plan(64, 8, 64, 8, 3, 1024, 64) == 1        # 512 pairs > 148 * 4 / 2
    assert plan(16, 8, 64, 8, 3, 1024, 64) == 4        # floor(592 / 128)
    assert plan(1, 4, 64, 8, 2, 32, 4, _lib.FC_DTYPE_F32) == 2  # nb / 16


def test_view_crop_and_gather_validate_without_launching():
    """fc_read_view, fc_crop and fc_select_batch check their arguments on
    the host; the cases below either fail validation or need no launch."""
    lib = _lib.load()
    s4 = lambda *x: (ctypes.c_int64 * 4)(*x)
    a = _arc(H=2, cap=4, nb=3)
    t = _tail(a, 5)
    rows = 3 * 8 + 5
    out_str = s4(2 * 32 * 64, 32 * 64, 64, 1)

    def view(first=0, out=FAKE, dt=_lib.FC_DTYPE_BF16, strides=out_str,
             tokens=32, tail=t):
        return lib.fc_read_view(ctypes.byref(a), _ref(tail), first, out, dt,
                                strides, tokens, None)

    _ref = lambda x: None if x is None else ctypes.byref(x)
    assert view(first=-1) == _lib.FC_ERR_INVALID
    assert view(first=4) == _lib.FC_ERR_INVALID            # > n_blocks
    assert view(out=None) == _lib.FC_ERR_INVALID
    assert view(out=FAKE + 8) == _lib.FC_ERR_INVALID       # misaligned
    assert view(dt=_lib.FC_DTYPE_I8) == _lib.FC_ERR_INVALID
    assert view(tokens=rows - 1) == _lib.FC_ERR_INVALID    # too few rows
    assert view(strides=s4(2 * 32 * 64, 32 * 64, 64, 2)) == \
        _lib.FC_ERR_INVALID                                # inner stride
    assert view(strides=s4(2 * 32 * 64, 32 * 64, 60, 1)) == \
        _lib.FC_ERR_INVALID                                # rows overlap
    # nothing to write: every block already decoded, empty tail
    assert view(first=3, tail=None) == _lib.FC_OK

    # crop: sign convention, missing tail, host-only cases
    c = _arc(H=2, cap=4, nb=3)
    ct = _tail(c, 5)
    assert lib.fc_crop(ctypes.byref(c), ctypes.byref(ct), 2, None) == \
        _lib.FC_ERR_INVALID
    assert lib.fc_crop(ctypes.byref(c), None, -2, None) == \
        _lib.FC_ERR_INVALID
    assert lib.fc_crop(ctypes.byref(c), ctypes.byref(ct), 0, None) == \
        _lib.FC_OK
    assert (c.n_blocks, ct.len) == (3, 5)
    assert lib.fc_crop(ctypes.byref(c), ctypes.byref(ct), -2, None) == \
        _lib.FC_OK                                         # tail only
    assert (c.n_blocks, ct.len) == (3, 3)
    assert lib.fc_crop(ctypes.byref(c), ctypes.byref(ct), -11, None) == \
        _lib.FC_OK                                         # to a boundary
    assert (c.n_blocks, ct.len) == (2, 0)
    assert lib.fc_crop(ctypes.byref(c), ctypes.byref(ct), -1000, None) == \
        _lib.FC_OK                                         # everything
    assert (c.n_blocks, ct.len) == (0, 0)

    # select_batch: index range, batch size, overlap, capacity, tails
    src = _arc(B=3, H=2, cap=4, nb=3)
    dst = _arc(B=2, H=2, cap=4)
    dst.coeffs = FAKE + (1 << 24)
    dst.scales = FAKE + (2 << 24)
    src.scales = FAKE + (3 << 24)

    def gather(idx, d=dst, st=None, dt=None):
        arr = (ctypes.c_int64 * len(idx))(*idx)
        return lib.fc_select_batch(ctypes.byref(src), _ref(st), arr, len(idx),
                                   ctypes.byref(d), _ref(dt), None)

    assert gather([0, 3]) == _lib.FC_ERR_INVALID           # index >= B
    assert gather([0, -1]) == _lib.FC_ERR_INVALID
    assert gather([0, 1, 2]) == _lib.FC_ERR_INVALID        # dst.B != n_idx
    same = _arc(B=2, H=2, cap=4)                           # overlaps src
    same.scales = FAKE + (2 << 24)
    assert gather([0, 1], d=same) == _lib.FC_ERR_INVALID
    small = _arc(B=2, H=2, cap=2)
    small.coeffs, small.scales = dst.coeffs, dst.scales
    assert gather([0, 1], d=small) == _lib.FC_ERR_CAPACITY
    assert gather([0, 1], st=_tail(src, 2)) == _lib.FC_ERR_INVALID  # one tail
    assert dst.n_blocks == 0
    assert lib.fc_select_batch(ctypes.byref(src), None, None, 2,
                               ctypes.byref(dst), None, None) == \
        _lib.FC_ERR_INVALID
    big = (ctypes.c_int64 * 1025)(*([0] * 1025))
    assert lib.fc_select_batch(ctypes.byref(src), None, big, 1025,
                               ctypes.byref(dst), None, None) == \
        _lib.FC_ERR_UNSUPPORTED


def test_state_save_restore_validate_on_the_host():
    """Image size arithmetic and header checks of fc_state_* (no copy is
    issued: every case fails validation, or has nothing to copy)."""
    arc = _lib.FcArchive(coeffs=FAKE, scales=FAKE, coeff_dtype=_lib.FC_DTYPE_I8,
                         R=8, S=2, B=2, H=3, D=64, capacity=32, n_blocks=10,
                         coeff_stride_b=3 * 32 * 2 * 64,
                         coeff_stride_h=32 * 2 * 64,
                         scale_stride_b=3 * 32 * 2, scale_stride_h=32 * 2)
    tail = _lib.FcTail(data=FAKE, dtype=_lib.FC_DTYPE_BF16, len=5,
                       stride_b=3 * 8 * 64, stride_h=8 * 64)
    hdr = ctypes.sizeof(_lib.FcStateHeader)
    assert hdr == 88
    n = _lib.fc_state_bytes(arc, tail)
    assert n == hdr + 6 * 10 * 2 * 64 + 6 * 10 * 2 * 4 + 6 * 5 * 64 * 2
    lib = _lib.load()
    import torch
    buf = torch.zeros(n, dtype=torch.uint8)
    # a zeroed image: no magic
    st = lib.fc_state_restore(ctypes.c_void_p(buf.data_ptr()), n,
                              ctypes.byref(arc), ctypes.byref(tail), None)
    assert st == _lib.FC_ERR_INVALID
    # a correct header for another S
    h = _lib.FcStateHeader(magic=b"FCSTATE1", version=1,
                           coeff_dtype=_lib.FC_DTYPE_I8,
                           tail_dtype=_lib.FC_DTYPE_BF16, R=8, S=3,
                           tail_len=0, B=2, H=3, D=64, n_blocks=0)
    ctypes.memmove(buf.data_ptr(), ctypes.byref(h), hdr)
    st = lib.fc_state_restore(ctypes.c_void_p(buf.data_ptr()), n,
                              ctypes.byref(arc), ctypes.byref(tail), None)
    assert st == _lib.FC_ERR_INVALID
    # the right geometry but more blocks than the capacity
    h.S, h.n_blocks = 2, 33
    h.coeff_bytes, h.scale_bytes = 6 * 33 * 2 * 64, 6 * 33 * 2 * 4
    big = torch.zeros(hdr + h.coeff_bytes + h.scale_bytes, dtype=torch.uint8)
    ctypes.memmove(big.data_ptr(), ctypes.byref(h), hdr)
    st = lib.fc_state_restore(ctypes.c_void_p(big.data_ptr()), big.numel(),
                              ctypes.byref(arc), ctypes.byref(tail), None)
    assert st == _lib.FC_ERR_CAPACITY
    assert (arc.n_blocks, tail.len) == (10, 5)
    # payload sizes that do not match the geometry
    h.n_blocks = 4
    ctypes.memmove(big.data_ptr(), ctypes.byref(h), hdr)
    st = lib.fc_state_restore(ctypes.c_void_p(big.data_ptr()), big.numel(),
                              ctypes.byref(arc), ctypes.byref(tail), None)
    assert st == _lib.FC_ERR_INVALID
    # saving into a buffer that is too small
    st = lib.fc_state_save(ctypes.byref(arc), ctypes.byref(tail),
                           ctypes.c_void_p(buf.data_ptr()), n - 1, None)
    assert st == _lib.FC_ERR_INVALID


def test_png_codec_descriptors_validate_on_the_host():
    """FC_CODEC_PNG needs S == R and fp32 rows; an unknown codec is refused;
    storage counts R fp32 rows per block."""
    def arc(S, dtype, codec, R=8):
        a = _arc(B=1, H=2, D=64, R=R, S=S, dtype=dtype, cap=16, nb=5)
        a.codec = codec
        return a
    lib = _lib.load()
    ok = arc(8, _lib.FC_DTYPE_F32, _lib.FC_CODEC_PNG)
    assert _lib.fc_storage_bytes(ok) == 1 * 2 * 5 * 8 * 64 * 4
    for bad in (arc(4, _lib.FC_DTYPE_F32, _lib.FC_CODEC_PNG),
                arc(8, _lib.FC_DTYPE_BF16, _lib.FC_CODEC_PNG),
                arc(2, _lib.FC_DTYPE_F32, 7)):
        assert lib.fc_storage_bytes(ctypes.byref(bad), None) == -1
    k = ctypes.c_int32(-1)
    assert lib.fc_decode_kernel(ctypes.byref(ok), ctypes.byref(ok), 4, 0,
                                ctypes.byref(k)) == _lib.FC_OK
    assert k.value == _lib.FC_KERNEL_CUDA_CORE


def test_decode_step_layers_validate_on_the_host():
    """fc_decode_step_layers refuses, before any launch: a layer count out of
    range, the overlap flags, layers of different (S, R), and two layers that
    share a stream."""
    lib = _lib.load()

    def layer(S=2, R=8, arcs=None):
        ka = arcs[0] if arcs else _arc(B=1, H=2, D=128, R=R, S=S, cap=32,
                                       nb=10)
        va = arcs[1] if arcs else _arc(B=1, H=2, D=128, R=R, S=S, cap=32,
                                       nb=10)
        kt, vt = _tail(ka, 3), _tail(va, 3)
        L = _lib.FcLayerStep()
        L.q = FAKE
        L.q_strides[:] = [2 * 4 * 128, 4 * 128, 128, 1]
        L.k_new = L.v_new = FAKE
        L.k_strides[:] = [2 * 128, 128, 128, 1]
        L.v_strides[:] = [2 * 128, 128, 128, 1]
        L.ka, L.va = ctypes.addressof(ka), ctypes.addressof(va)
        L.kt, L.vt = ctypes.addressof(kt), ctypes.addressof(vt)
        L.workspace = 0x100000
        L.workspace_bytes = 1 << 20
        L.out = FAKE
        L.out_strides[:] = [2 * 4 * 128, 4 * 128, 128, 1]
        return L, (ka, va, kt, vt)

    def call(layers, flags=_lib.FC_DECODE_FUSE_COMBINE, n=None):
        arr = (_lib.FcLayerStep * max(1, len(layers)))(*[x[0] for x in layers])
        return lib.fc_decode_step_layers(
            len(layers) if n is None else n, arr, _lib.FC_DTYPE_BF16,
            _lib.FC_DTYPE_BF16, _lib.FC_DTYPE_F32, 4, 0.0, 0, flags, None)

    a, b = layer(), layer()
    assert call([a, b], n=0) == _lib.FC_ERR_INVALID
    assert call([a, b], n=_lib.FC_MAX_LAYERS + 1) == _lib.FC_ERR_INVALID
    assert call([a, b], flags=_lib.FC_DECODE_FUSE_COMBINE |
                _lib.FC_DECODE_PORTABLE) == _lib.FC_ERR_INVALID
    assert call([a, b], flags=_lib.FC_DECODE_FUSE_COMBINE |
                _lib.FC_DECODE_TEST_TIMEOUT) == _lib.FC_ERR_INVALID
    c = layer(S=4, R=16)
    assert call([a, c]) == _lib.FC_ERR_UNSUPPORTED
    shared = layer(arcs=a[1][:2])
    assert call([a, shared]) == _lib.FC_ERR_INVALID


def test_timeout_hook_validates_on_the_host():
    """FC_DECODE_TEST_TIMEOUT needs the tensor-core kernel and a status word:
    unsupported on the portable kernel and for archives the tensor-core
    kernel does not serve, invalid for a fused single-split call (no
    workspace)."""
    lib = _lib.load()
    q_str = (ctypes.c_int64 * 4)(32 * 128, 128, 128, 1)
    tc = _arc(H=8, D=128, R=16, S=4, cap=64, nb=40)
    narrow = _arc(H=8, D=64, R=8, S=2, cap=64, nb=40)
    T = _lib.FC_DECODE_TEST_TIMEOUT

    def attn(ka, ns, flags):
        return lib.fc_decode_attention(
            FAKE, _lib.FC_DTYPE_BF16, q_str, 32, ctypes.byref(ka),
            ctypes.byref(ka), None, None, 0.0, ns, flags, FAKE, 1 << 30,
            FAKE, _lib.FC_DTYPE_F32, q_str, None)

    assert attn(tc, 1, _lib.FC_DECODE_FUSE_COMBINE | T) == _lib.FC_ERR_INVALID
    assert attn(tc, 2, _lib.FC_DECODE_FUSE_COMBINE | _lib.FC_DECODE_PORTABLE
                | T) == _lib.FC_ERR_UNSUPPORTED
    assert attn(narrow, 2, _lib.FC_DECODE_FUSE_COMBINE | T) == \
        _lib.FC_ERR_UNSUPPORTED


def test_host_step_sizes_and_validates_before_queuing_anything():
    """fc_decode_step_staging_bytes is host arithmetic (three 256-byte
    aligned input slots and the output slot); fc_decode_step_host rejects
    bad arguments before it queues a copy or a kernel, so these calls return
    on a machine without a GPU."""
    lib = _lib.load()
    B, H, Hq, D = 2, 8, 32, 128
    tok, q, out = B * H * D * 2, B * Hq * D * 2, B * Hq * D * 4
    pad = lambda n: (n + 255) // 256 * 256
    need = lib.fc_decode_step_staging_bytes(B, H, Hq, D, _lib.FC_DTYPE_BF16,
                                            _lib.FC_DTYPE_F32)
    assert need == 2 * pad(tok) + pad(q) + pad(out)
    assert lib.fc_decode_step_staging_bytes(B, H, Hq, D, _lib.FC_DTYPE_I8,
                                            _lib.FC_DTYPE_F32) == 0
    assert lib.fc_decode_step_staging_bytes(0, H, Hq, D, _lib.FC_DTYPE_BF16,
                                            _lib.FC_DTYPE_F32) == 0
    ka = _arc(B=B, H=H, D=D, R=16, S=4, cap=64, nb=40)
    va = _arc(B=B, H=H, D=D, R=16, S=4, cap=64, nb=40)
    kt, vt = _tail(ka, 3), _tail(va, 3)

    def call(staging=FAKE * 16, nbytes=need, flags=_lib.FC_DECODE_FUSE_COMBINE,
             in_host=FAKE, io=_lib.FC_DTYPE_BF16):
        return lib.fc_decode_step_host(
            in_host, FAKE, staging, nbytes, io, _lib.FC_DTYPE_F32, Hq,
            ctypes.byref(ka), ctypes.byref(va), ctypes.byref(kt),
            ctypes.byref(vt), 0.0, 0, flags, FAKE * 16, 1 << 30, None)

    assert call(in_host=None) == _lib.FC_ERR_INVALID
    assert call(staging=FAKE * 16 + 16) == _lib.FC_ERR_INVALID   # 256-byte aligned
    assert call(nbytes=need - 1) == _lib.FC_ERR_INVALID
    assert call(io=_lib.FC_DTYPE_I8) == _lib.FC_ERR_INVALID
    assert call(flags=1 << 8) == _lib.FC_ERR_INVALID
    assert call(flags=_lib.FC_DECODE_FUSE_COMBINE |
                _lib.FC_DECODE_TEST_TIMEOUT) == _lib.FC_ERR_INVALID
    ka.n_blocks = ka.capacity = 40                 # the token would complete
    kt.len = vt.len = 15                           # a block with no room
    ka.coeff_stride_h = 40 * 4 * D
    ka.coeff_stride_b = H * ka.coeff_stride_h
    ka.scale_stride_h = 40 * 4
    ka.scale_stride_b = H * ka.scale_stride_h
    assert call() == _lib.FC_ERR_CAPACITY
    assert (ka.n_blocks, kt.len) == (40, 15)
