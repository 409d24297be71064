"""Thin ctypes binding of libfc (``include/fc.h``, ``include/fc_view.h``).

Argument marshalling only: tensors become device pointers, element strides
and the current CUDA stream; every computation runs in libfc's kernels. A
missing library is an error, never a fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfc.so")

FC_OK = 0
FC_ERR_INVALID = 1
FC_ERR_UNSUPPORTED = 2
FC_ERR_CAPACITY = 3
FC_ERR_CUDA = 4
FC_ERR_DEVICE = 5
FC_ERR_SCRATCH_LIMIT = 6
FC_NOALLOC_SCRATCH_BYTES = 8 << 20

FC_DECODE_FUSE_COMBINE = 1
FC_DECODE_PORTABLE = 2
FC_DECODE_OVERLAP = 4
FC_DECODE_Q_FINAL = 8
FC_DECODE_TEST_TIMEOUT = 16

FC_KERNEL_CUDA_CORE = 0
FC_KERNEL_TENSOR_CORE = 1

FC_SELECT_MAX_BATCH = 1024

FC_CODEC_DCT = 0
FC_CODEC_PNG = 1

FC_DTYPE_F32 = 0
FC_DTYPE_BF16 = 1
FC_DTYPE_I8 = 2

_DTYPE_CODE = {torch.float32: FC_DTYPE_F32, torch.bfloat16: FC_DTYPE_BF16,
               torch.int8: FC_DTYPE_I8}

# Every symbol include/fc.h and include/fc_view.h declare.
EXPORTS = (
    "fc_compress_blocks", "fc_append_step", "fc_archive_copy_prefix",
    "fc_decode_plan", "fc_decode_workspace_bytes", "fc_decode_attention",
    "fc_combine", "fc_decode_attention_noalloc", "fc_workspace_status",
    "fc_storage_bytes", "fc_status_string", "fc_decode_step",
    "fc_read_view", "fc_crop", "fc_select_batch", "fc_noalloc_status",
    "fc_decode_kernel", "fc_state_bytes", "fc_state_save", "fc_state_restore",
    "fc_decode_step_layers", "fc_decode_step_staging_bytes",
    "fc_decode_step_host",
)

FC_MAX_LAYERS = 16


class FcError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)"
                         % (where, fc_status_string(status), status))


class FcArchive(ctypes.Structure):
    _fields_ = [
        ("coeffs", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("coeff_dtype", ctypes.c_int32), ("R", ctypes.c_int32),
        ("S", ctypes.c_int32), ("codec", ctypes.c_int32),
        ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("D", ctypes.c_int64),
        ("capacity", ctypes.c_int64), ("n_blocks", ctypes.c_int64),
        ("coeff_stride_b", ctypes.c_int64), ("coeff_stride_h", ctypes.c_int64),
        ("scale_stride_b", ctypes.c_int64), ("scale_stride_h", ctypes.c_int64),
    ]


class FcLayerStep(ctypes.Structure):
    """fc_layer_step of include/fc.h (one layer of fc_decode_step_layers)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("q_strides", ctypes.c_int64 * 4),
        ("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p),
        ("k_strides", ctypes.c_int64 * 4), ("v_strides", ctypes.c_int64 * 4),
        ("ka", ctypes.c_void_p), ("va", ctypes.c_void_p),
        ("kt", ctypes.c_void_p), ("vt", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("out", ctypes.c_void_p), ("out_strides", ctypes.c_int64 * 4),
    ]


class FcStateHeader(ctypes.Structure):
    """fc_state_header of include/fc_state.h."""
    _fields_ = [
        ("magic", ctypes.c_char * 8), ("version", ctypes.c_int32),
        ("coeff_dtype", ctypes.c_int32), ("tail_dtype", ctypes.c_int32),
        ("R", ctypes.c_int32), ("S", ctypes.c_int32),
        ("tail_len", ctypes.c_int32), ("B", ctypes.c_int64),
        ("H", ctypes.c_int64), ("D", ctypes.c_int64),
        ("n_blocks", ctypes.c_int64), ("coeff_bytes", ctypes.c_int64),
        ("scale_bytes", ctypes.c_int64), ("tail_bytes", ctypes.c_int64),
    ]


class FcTail(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p), ("dtype", ctypes.c_int32),
        ("len", ctypes.c_int32), ("stride_b", ctypes.c_int64),
        ("stride_h", ctypes.c_int64),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load libfc.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libfc.so is missing at %s: build it with `python -m "
            "compressed_decode_attention_blockwise_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I32 = ctypes.c_int32
    I64 = ctypes.c_int64
    PI64 = ctypes.POINTER(ctypes.c_int64)
    PA = ctypes.POINTER(FcArchive)
    PT = ctypes.POINTER(FcTail)
    sig = {
        "fc_compress_blocks": (ctypes.c_int, [P, I32, PI64, I64, PA, PT, P]),
        "fc_append_step": (ctypes.c_int, [P, P, I32, PI64, PI64, PA, PA, PT,
                                          PT, P]),
        "fc_archive_copy_prefix": (ctypes.c_int, [PA, PA, P]),
        "fc_decode_plan": (ctypes.c_int, [PA, PT, I64,
                                          ctypes.POINTER(ctypes.c_int32)]),
        "fc_decode_workspace_bytes": (ctypes.c_size_t, [I64, I64, I64, I32]),
        "fc_decode_kernel": (ctypes.c_int, [PA, PA, I64, I32,
                                            ctypes.POINTER(ctypes.c_int32)]),
        "fc_decode_attention": (ctypes.c_int, [P, I32, PI64, I64, PA, PA, PT,
                                               PT, ctypes.c_float, I32, I32,
                                               P, ctypes.c_size_t, P, I32,
                                               PI64, P]),
        "fc_decode_step": (ctypes.c_int, [P, I32, PI64, I64, P, P, I32, PI64,
                                          PI64, PA, PA, PT, PT,
                                          ctypes.c_float, I32, I32, P,
                                          ctypes.c_size_t, P, I32, PI64, P]),
        "fc_decode_step_staging_bytes": (ctypes.c_size_t, [I64, I64, I64, I64,
                                                            I32, I32]),
        "fc_decode_step_host": (ctypes.c_int, [P, P, P, ctypes.c_size_t, I32,
                                               I32, I64, PA, PA, PT, PT,
                                               ctypes.c_float, I32, I32, P,
                                               ctypes.c_size_t, P]),
        "fc_decode_step_layers": (ctypes.c_int, [I32,
                                                 ctypes.POINTER(FcLayerStep),
                                                 I32, I32, I32, I64,
                                                 ctypes.c_float, I32, I32, P]),
        "fc_combine": (ctypes.c_int, [P, ctypes.c_size_t, I64, I64, I64, I32,
                                      P, I32, PI64, P]),
        "fc_decode_attention_noalloc": (ctypes.c_int, [P, I32, PI64, I64, PA,
                                                       PA, PT, PT,
                                                       ctypes.c_float, I32, P,
                                                       I32, PI64, P]),
        "fc_workspace_status": (ctypes.c_int, [P, ctypes.c_size_t,
                                               ctypes.POINTER(ctypes.c_uint32),
                                               P]),
        "fc_noalloc_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32),
                                             P]),
        "fc_storage_bytes": (ctypes.c_int64, [PA, PT]),
        "fc_state_bytes": (ctypes.c_size_t, [PA, PT]),
        "fc_state_save": (ctypes.c_int, [PA, PT, P, ctypes.c_size_t, P]),
        "fc_state_restore": (ctypes.c_int, [P, ctypes.c_size_t, PA, PT, P]),
        "fc_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "fc_read_view": (ctypes.c_int, [PA, PT, I64, P, I32, PI64, I64, P]),
        "fc_crop": (ctypes.c_int, [PA, PT, I64, P]),
        "fc_select_batch": (ctypes.c_int, [PA, PT, PI64, I64, PA, PT, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def fc_status_string(status: int) -> str:
    return load().fc_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != FC_OK:
        raise FcError(status, where)


def dtype_code(dt: torch.dtype) -> int:
    try:
        return _DTYPE_CODE[dt]
    except KeyError:
        raise ValueError("unsupported dtype %s" % dt) from None


def _strides4(t: torch.Tensor):
    if t.dim() != 4:
        raise ValueError("expected a 4-d tensor, got shape %s"
                         % (tuple(t.shape),))
    return (ctypes.c_int64 * 4)(*t.stride())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, *tensors):
    """cudaStream_t handle: the given stream or torch's current one."""
    if stream is not None:
        return ctypes.c_void_p(int(getattr(stream, "cuda_stream", stream)))
    for t in tensors:
        if t is not None and t.is_cuda:
            return ctypes.c_void_p(torch.cuda.current_stream(t.device)
                                   .cuda_stream)
    return ctypes.c_void_p(0)


def _ref(x):
    return None if x is None else ctypes.byref(x)


# ------------------------------------------------------------------ calls

def fc_compress_blocks(x: torch.Tensor, arc: FcArchive,
                       tail: Optional[FcTail] = None, stream=None) -> None:
    st = load().fc_compress_blocks(_ptr(x), dtype_code(x.dtype), _strides4(x),
                                   x.shape[2], ctypes.byref(arc), _ref(tail),
                                   _stream(stream, x))
    _check(st, "fc_compress_blocks")


def fc_append_step(k_new: torch.Tensor, v_new: torch.Tensor, ka: FcArchive,
                   va: FcArchive, kt: FcTail, vt: FcTail, stream=None) -> None:
    if k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must share a dtype")
    st = load().fc_append_step(_ptr(k_new), _ptr(v_new),
                               dtype_code(k_new.dtype), _strides4(k_new),
                               _strides4(v_new), ctypes.byref(ka),
                               ctypes.byref(va), ctypes.byref(kt),
                               ctypes.byref(vt), _stream(stream, k_new))
    _check(st, "fc_append_step")


def fc_archive_copy_prefix(src: FcArchive, dst: FcArchive,
                           stream=None, device=None) -> None:
    s = _stream(stream) if stream is not None or device is None else \
        ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    st = load().fc_archive_copy_prefix(ctypes.byref(src), ctypes.byref(dst),
                                       s)
    _check(st, "fc_archive_copy_prefix")


def fc_decode_plan(ka: FcArchive, kt: Optional[FcTail], Hq: int) -> int:
    out = ctypes.c_int32(0)
    st = load().fc_decode_plan(ctypes.byref(ka), _ref(kt), int(Hq),
                               ctypes.byref(out))
    _check(st, "fc_decode_plan")
    return int(out.value)


def fc_decode_kernel(ka: FcArchive, va: FcArchive, Hq: int,
                     portable: bool = False) -> int:
    """FC_KERNEL_TENSOR_CORE or FC_KERNEL_CUDA_CORE: the kernel decode
    attention runs for these archives."""
    out = ctypes.c_int32(0)
    st = load().fc_decode_kernel(ctypes.byref(ka), ctypes.byref(va), int(Hq),
                                 FC_DECODE_PORTABLE if portable else 0,
                                 ctypes.byref(out))
    _check(st, "fc_decode_kernel")
    return int(out.value)


def fc_decode_workspace_bytes(B: int, Hq: int, D: int, num_splits: int) -> int:
    return int(load().fc_decode_workspace_bytes(int(B), int(Hq), int(D),
                                                int(num_splits)))


def fc_decode_attention(q: torch.Tensor, ka: FcArchive, va: FcArchive,
                        kt: Optional[FcTail], vt: Optional[FcTail],
                        out: torch.Tensor, workspace: Optional[torch.Tensor],
                        softmax_scale: float = 0.0, num_splits: int = 0,
                        fuse_combine: bool = True, portable: bool = False,
                        overlap: bool = False, q_final: bool = False,
                        test_timeout: bool = False, stream=None) -> None:
    ws_ptr = _ptr(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * \
        workspace.element_size()
    flags = (FC_DECODE_FUSE_COMBINE if fuse_combine else 0) | \
        (FC_DECODE_PORTABLE if portable else 0) | \
        (FC_DECODE_OVERLAP if overlap else 0) | \
        (FC_DECODE_Q_FINAL if q_final else 0) | \
        (FC_DECODE_TEST_TIMEOUT if test_timeout else 0)
    st = load().fc_decode_attention(
        _ptr(q), dtype_code(q.dtype), _strides4(q), q.shape[1],
        ctypes.byref(ka), ctypes.byref(va), _ref(kt), _ref(vt),
        float(softmax_scale), int(num_splits), flags,
        ws_ptr, ws_bytes, _ptr(out), dtype_code(out.dtype), _strides4(out),
        _stream(stream, q))
    _check(st, "fc_decode_attention")


def fc_decode_step(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                   ka: FcArchive, va: FcArchive, kt: FcTail, vt: FcTail,
                   out: torch.Tensor, workspace: Optional[torch.Tensor],
                   softmax_scale: float = 0.0, num_splits: int = 0,
                   fuse_combine: bool = True, portable: bool = False,
                   overlap: bool = False, q_final: bool = False,
                   stream=None) -> None:
    if k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must share a dtype")
    ws_ptr = _ptr(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * \
        workspace.element_size()
    flags = (FC_DECODE_FUSE_COMBINE if fuse_combine else 0) | \
        (FC_DECODE_PORTABLE if portable else 0) | \
        (FC_DECODE_OVERLAP if overlap else 0) | \
        (FC_DECODE_Q_FINAL if q_final else 0)
    st = load().fc_decode_step(
        _ptr(q), dtype_code(q.dtype), _strides4(q), q.shape[1],
        _ptr(k_new), _ptr(v_new), dtype_code(k_new.dtype), _strides4(k_new),
        _strides4(v_new), ctypes.byref(ka), ctypes.byref(va),
        ctypes.byref(kt), ctypes.byref(vt), float(softmax_scale),
        int(num_splits), flags, ws_ptr, ws_bytes, _ptr(out),
        dtype_code(out.dtype), _strides4(out), _stream(stream, q))
    _check(st, "fc_decode_step")


class HostStep:
    """fc_decode_step_host with its arguments marshalled once: calling it
    runs one step from the host block ``in_host`` ([k_new | v_new | q]) to
    ``out_host`` (both CPU tensors; pinned for asynchronous copies). The
    archive and tail descriptors are passed by reference, so the library's
    updates carry over from call to call."""

    def __init__(self, cache, Hq: int, in_host: torch.Tensor,
                 out_host: torch.Tensor, staging: torch.Tensor,
                 workspace: torch.Tensor, softmax_scale: float = 0.0,
                 num_splits: int = 0, fuse_combine: bool = True,
                 overlap: bool = False, q_final: bool = False, stream=None):
        flags = (FC_DECODE_FUSE_COMBINE if fuse_combine else 0) | \
            (FC_DECODE_OVERLAP if overlap else 0) | \
            (FC_DECODE_Q_FINAL if q_final else 0)
        self._fn = load().fc_decode_step_host
        self._args = (
            ctypes.c_void_p(in_host.data_ptr()),
            ctypes.c_void_p(out_host.data_ptr()),
            ctypes.c_void_p(staging.data_ptr()),
            ctypes.c_size_t(staging.numel() * staging.element_size()),
            ctypes.c_int32(dtype_code(in_host.dtype)),
            ctypes.c_int32(dtype_code(out_host.dtype)), ctypes.c_int64(Hq),
            ctypes.byref(cache.k.arc), ctypes.byref(cache.v.arc),
            ctypes.byref(cache.k.tail_desc), ctypes.byref(cache.v.tail_desc),
            ctypes.c_float(softmax_scale), ctypes.c_int32(num_splits),
            ctypes.c_int32(flags), ctypes.c_void_p(workspace.data_ptr()),
            ctypes.c_size_t(workspace.numel() * workspace.element_size()),
            _stream(stream, staging))
        self._keep = (in_host, out_host, staging, workspace)

    def __call__(self) -> None:
        st = self._fn(*self._args)
        if st != FC_OK:
            raise FcError(st, "fc_decode_step_host")


def fc_decode_step_staging_bytes(B: int, H: int, Hq: int, D: int,
                                 io_dtype: torch.dtype,
                                 out_dtype: torch.dtype) -> int:
    return int(load().fc_decode_step_staging_bytes(
        int(B), int(H), int(Hq), int(D), dtype_code(io_dtype),
        dtype_code(out_dtype)))


def fc_decode_step_layers(qs, k_news, v_news, kas, vas, kts, vts, outs,
                          workspaces, softmax_scale: float = 0.0,
                          num_splits: int = 0, fuse_combine: bool = True,
                          overlap: bool = False, q_final: bool = False,
                          stream=None) -> None:
    """One launch of the fused decode steps of len(qs) independent streams
    (per-layer tensors and descriptors in matching lists)."""
    n = len(qs)
    arr = (FcLayerStep * max(1, n))()
    for i in range(n):
        L = arr[i]
        L.q = qs[i].data_ptr()
        L.q_strides[:] = list(qs[i].stride())
        L.k_new, L.v_new = k_news[i].data_ptr(), v_news[i].data_ptr()
        L.k_strides[:] = list(k_news[i].stride())
        L.v_strides[:] = list(v_news[i].stride())
        L.ka = ctypes.addressof(kas[i])
        L.va = ctypes.addressof(vas[i])
        L.kt = ctypes.addressof(kts[i])
        L.vt = ctypes.addressof(vts[i])
        ws = workspaces[i]
        L.workspace = None if ws is None else ws.data_ptr()
        L.workspace_bytes = 0 if ws is None else ws.numel() * ws.element_size()
        L.out = outs[i].data_ptr()
        L.out_strides[:] = list(outs[i].stride())
    st = load().fc_decode_step_layers(
        n, arr, dtype_code(qs[0].dtype), dtype_code(k_news[0].dtype),
        dtype_code(outs[0].dtype), qs[0].shape[1], float(softmax_scale),
        int(num_splits), (FC_DECODE_FUSE_COMBINE if fuse_combine else 0) |
        (FC_DECODE_OVERLAP if overlap else 0) |
        (FC_DECODE_Q_FINAL if q_final else 0), _stream(stream, qs[0]))
    _check(st, "fc_decode_step_layers")


def fc_decode_attention_noalloc(q: torch.Tensor, ka: FcArchive, va: FcArchive,
                                kt: Optional[FcTail], vt: Optional[FcTail],
                                out: torch.Tensor, softmax_scale: float = 0.0,
                                num_splits: int = 0, stream=None) -> None:
    """Decode attention with the library's static scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    st = load().fc_decode_attention_noalloc(
        _ptr(q), dtype_code(q.dtype), _strides4(q), q.shape[1],
        ctypes.byref(ka), ctypes.byref(va), _ref(kt), _ref(vt),
        float(softmax_scale), int(num_splits), _ptr(out),
        dtype_code(out.dtype), _strides4(out), _stream(stream, q))
    _check(st, "fc_decode_attention_noalloc")


def fc_combine(workspace: torch.Tensor, B: int, Hq: int, D: int,
               num_splits: int, out: torch.Tensor, stream=None) -> None:
    st = load().fc_combine(_ptr(workspace),
                           workspace.numel() * workspace.element_size(),
                           int(B), int(Hq), int(D), int(num_splits),
                           _ptr(out), dtype_code(out.dtype), _strides4(out),
                           _stream(stream, out))
    _check(st, "fc_combine")


def fc_workspace_status(workspace: torch.Tensor, stream=None) -> int:
    v = ctypes.c_uint32(0)
    st = load().fc_workspace_status(
        _ptr(workspace), workspace.numel() * workspace.element_size(),
        ctypes.byref(v), _stream(stream, workspace))
    if st not in (FC_OK, FC_ERR_DEVICE):
        _check(st, "fc_workspace_status")
    return int(v.value)


def fc_noalloc_status(stream=None, device=None) -> int:
    """Status word of fc_decode_attention_noalloc's static scratch on the
    current device (0 = no error reported); reading clears it."""
    v = ctypes.c_uint32(0)
    s = _stream(stream) if stream is not None or device is None else \
        ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    st = load().fc_noalloc_status(ctypes.byref(v), s)
    if st not in (FC_OK, FC_ERR_DEVICE):
        _check(st, "fc_noalloc_status")
    return int(v.value)


def fc_storage_bytes(arc: FcArchive, tail: Optional[FcTail] = None) -> int:
    n = int(load().fc_storage_bytes(ctypes.byref(arc), _ref(tail)))
    if n < 0:
        raise FcError(FC_ERR_INVALID, "fc_storage_bytes")
    return n


# ------------------------------------------------- save / restore (state)

def fc_state_bytes(arc: FcArchive, tail: Optional[FcTail] = None) -> int:
    n = int(load().fc_state_bytes(ctypes.byref(arc), _ref(tail)))
    if n == 0:
        raise FcError(FC_ERR_INVALID, "fc_state_bytes")
    return n


def fc_state_save(arc: FcArchive, tail: Optional[FcTail], dst: torch.Tensor,
                  stream=None, device=None) -> None:
    """Write the stream's image into the CPU uint8 tensor ``dst`` (pinned
    for an asynchronous copy); complete once the stream reaches the copies."""
    if dst.device.type != "cpu" or dst.dtype != torch.uint8 or \
            not dst.is_contiguous():
        raise ValueError("dst must be a contiguous CPU uint8 tensor")
    s = _stream(stream) if stream is not None or device is None else \
        ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    st = load().fc_state_save(ctypes.byref(arc), _ref(tail), _ptr(dst),
                              dst.numel(), s)
    _check(st, "fc_state_save")


def fc_state_header(src: torch.Tensor) -> FcStateHeader:
    """The header of an image held in a CPU uint8 tensor."""
    if src.numel() < ctypes.sizeof(FcStateHeader):
        raise ValueError("image shorter than its header")
    if src.device.type != "cpu" or src.dtype != torch.uint8 or \
            not src.is_contiguous():
        raise ValueError("src must be a contiguous CPU uint8 tensor")
    hd = FcStateHeader()
    ctypes.memmove(ctypes.byref(hd), src.data_ptr(),
                   ctypes.sizeof(FcStateHeader))
    return hd


def fc_state_restore(src: torch.Tensor, arc: FcArchive,
                     tail: Optional[FcTail], stream=None,
                     device=None) -> None:
    """Load an image (CPU uint8 tensor) into the stream; sets n_blocks and
    the tail length on success."""
    if src.device.type != "cpu" or src.dtype != torch.uint8 or \
            not src.is_contiguous():
        raise ValueError("src must be a contiguous CPU uint8 tensor")
    s = _stream(stream) if stream is not None or device is None else \
        ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    st = load().fc_state_restore(_ptr(src), src.numel(), ctypes.byref(arc),
                                 _ref(tail), s)
    _check(st, "fc_state_restore")


# --------------------------------------------------- stream structure (view)

def fc_read_view(arc: FcArchive, tail: Optional[FcTail], first_block: int,
                 out: torch.Tensor, stream=None) -> None:
    """Decode archived blocks [first_block, n_blocks) and copy the live tail
    rows into ``out`` (B, H, T_out, D) at their token positions."""
    st = load().fc_read_view(ctypes.byref(arc), _ref(tail), int(first_block),
                             _ptr(out), dtype_code(out.dtype),
                             _strides4(out), int(out.shape[2]),
                             _stream(stream, out))
    _check(st, "fc_read_view")


def fc_crop(arc: FcArchive, tail: FcTail, tokens_to_remove: int,
            stream=None, device=None) -> None:
    """Remove the last ``-tokens_to_remove`` tokens (a negative count)."""
    s = _stream(stream) if stream is not None or device is None else \
        ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    st = load().fc_crop(ctypes.byref(arc), ctypes.byref(tail),
                        int(tokens_to_remove), s)
    _check(st, "fc_crop")


def fc_select_batch(src: FcArchive, src_tail: Optional[FcTail], idx,
                    dst: FcArchive, dst_tail: Optional[FcTail],
                    stream=None, device=None) -> None:
    """Batch row i of ``dst`` := batch row ``idx[i]`` of ``src`` (archive
    live blocks and tail rows). ``idx`` is a host sequence of ints."""
    idx = [int(i) for i in idx]
    arr = (ctypes.c_int64 * max(1, len(idx)))(*idx)
    s = _stream(stream) if stream is not None or device is None else \
        ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    st = load().fc_select_batch(ctypes.byref(src), _ref(src_tail), arr,
                                len(idx), ctypes.byref(dst), _ref(dst_tail),
                                s)
    _check(st, "fc_select_batch")
