"""Device archive of one layer's K and V streams and its decode attention.

Host bookkeeping around libfc (flashcodec/cache.py, ``_CodecStream`` and
``CodecKVCache``): each stream keeps a raw tail of at most R-1 tokens at the
input precision and a compressed archive whose capacity starts at 16 blocks
and doubles when full, the live prefix being copied by libfc's copy kernel.
The structural operations of the pages' cache are here too: the memoised
reconstructed view (``read``), exact ``crop``, batch gather
(``select_batch`` / ``reorder_cache``) and ``reset``.
Device memory comes from torch; every byte of codec and attention arithmetic
runs in libfc's kernels.
"""

from __future__ import annotations

import math
from typing import Optional

import torch

from . import _lib

INITIAL_BLOCKS = 16

_COEFF = {"i8": torch.int8, "bf16": torch.bfloat16, "f32": torch.float32}


def grown_capacity(capacity: int, need: int) -> int:
    """Geometric growth: unchanged if ``need`` fits, else the smallest
    16 * 2^k >= need (flashcodec/cache.py, ``_CodecStream._grow``)."""
    if need <= capacity:
        return capacity
    cap = INITIAL_BLOCKS
    while cap < need:
        cap *= 2
    return cap


class CodecStream:
    """One (B, H, T, D) K or V stream on the device. ``codec`` is "dct" (the
    block DCT, S kept rows) or "png" (the lossless tier: anchor and fp32
    first differences, S = R, coeff "f32")."""

    def __init__(self, B: int, H: int, D: int, R: int, S: int, coeff: str,
                 token_dtype: torch.dtype, device, capacity: int = 0,
                 codec: str = "dct"):
        self.B, self.H, self.D, self.R, self.S = B, H, D, R, S
        self.coeff = coeff
        self.token_dtype = token_dtype
        self.device = torch.device(device)
        self.coeffs: Optional[torch.Tensor] = None
        self.scales: Optional[torch.Tensor] = None
        self.tail = torch.zeros((B, H, R, D), dtype=token_dtype,
                                device=self.device)
        self.arc = _lib.FcArchive()
        self.arc.coeff_dtype = _lib.dtype_code(_COEFF[coeff])
        self.arc.R, self.arc.S = R, S
        self.codec = codec
        self.arc.codec = {"dct": _lib.FC_CODEC_DCT,
                          "png": _lib.FC_CODEC_PNG}[codec]
        self.arc.B, self.arc.H, self.arc.D = B, H, D
        self.tail_desc = _lib.FcTail()
        self.tail_desc.data = self.tail.data_ptr()
        self.tail_desc.dtype = _lib.dtype_code(token_dtype)
        self.tail_desc.len = 0
        self.tail_desc.stride_b, self.tail_desc.stride_h = \
            self.tail.stride(0), self.tail.stride(1)
        self._rec: Optional[torch.Tensor] = None   # reconstructed view
        self._rec_blocks = 0                       # blocks decoded into it
        self._alloc(grown_capacity(0, max(capacity, 1)))

    # -- storage -----------------------------------------------------------
    def _storage(self, B: int, cap: int):
        """Fresh (coeffs, scales, descriptor with n_blocks = 0) for B rows."""
        coeffs = torch.empty((B, self.H, cap, self.S, self.D),
                             dtype=_COEFF[self.coeff], device=self.device)
        scales = None
        if self.coeff == "i8":
            scales = torch.empty((B, self.H, cap, self.S),
                                 dtype=torch.float32, device=self.device)
        new = _lib.FcArchive()
        ctypes_copy(new, self.arc)
        new.B = B
        new.coeffs = coeffs.data_ptr()
        new.scales = None if scales is None else scales.data_ptr()
        new.capacity = cap
        new.n_blocks = 0
        new.coeff_stride_b, new.coeff_stride_h = coeffs.stride(0), \
            coeffs.stride(1)
        if scales is not None:
            new.scale_stride_b, new.scale_stride_h = scales.stride(0), \
                scales.stride(1)
        else:
            new.scale_stride_b = new.scale_stride_h = 0
        return coeffs, scales, new

    def _alloc(self, cap: int):
        coeffs, scales, new = self._storage(self.B, cap)
        if self.coeffs is not None and self.arc.n_blocks:
            _lib.fc_archive_copy_prefix(self.arc, new, device=self.device)
        else:
            new.n_blocks = self.arc.n_blocks if self.coeffs is not None else 0
        self.coeffs, self.scales, self.arc = coeffs, scales, new

    def ensure_capacity(self, need_blocks: int) -> bool:
        cap = grown_capacity(int(self.arc.capacity), int(need_blocks))
        if cap != self.arc.capacity:
            self._alloc(cap)
            return True
        return False

    # -- views ---------------------------------------------------------------
    @property
    def n_blocks(self) -> int:
        return int(self.arc.n_blocks)

    @property
    def tail_len(self) -> int:
        return int(self.tail_desc.len)

    @property
    def capacity(self) -> int:
        return int(self.arc.capacity)

    @property
    def seq_len(self) -> int:
        return self.n_blocks * self.R + self.tail_len

    def live_coeffs(self) -> torch.Tensor:
        return self.coeffs[:, :, : self.n_blocks]

    def live_scales(self) -> Optional[torch.Tensor]:
        return None if self.scales is None else \
            self.scales[:, :, : self.n_blocks]

    def live_tail(self) -> torch.Tensor:
        return self.tail[:, :, : self.tail_len]

    def storage_bytes(self) -> int:
        return _lib.fc_storage_bytes(self.arc, self.tail_desc)

    # -- structure (flashcodec/cache.py, _CodecStream) -------------------------
    def read(self) -> Optional[torch.Tensor]:
        """Reconstructed (B, H, seq_len, D) view in the token dtype
        (``_CodecStream.read``): archived blocks decompressed by libfc, then
        the raw tail. Each archived block is decoded once into a persistent
        buffer (append-only memoisation); ``None`` for an empty stream, the
        tail itself when nothing is archived. Without raw tokens the returned
        tensor aliases that buffer (its rows keep their values until a crop,
        batch gather or reset); with raw tokens it is a fresh tensor (the
        decoded prefix copied, the tail rows written by libfc), so a tensor
        handed out earlier never changes when a later read archives those
        tail tokens."""
        T = self.seq_len
        if T == 0:
            return None
        if self.n_blocks == 0:
            return self.live_tail()
        nb = self.n_blocks
        need = nb * self.R
        if self._rec is None or self._rec.shape[2] < need:
            old = 0 if self._rec is None else self._rec.shape[2]
            rows = max(need, 2 * old, INITIAL_BLOCKS * self.R)
            self._rec = torch.empty((self.B, self.H, rows, self.D),
                                    dtype=self.token_dtype,
                                    device=self.device)
            self._rec_blocks = 0   # a new buffer is decoded from block 0
        if self._rec_blocks < nb:
            _lib.fc_read_view(self.arc, None, self._rec_blocks, self._rec)
        self._rec_blocks = nb
        if self.tail_len == 0:
            return self._rec[:, :, :T]
        out = torch.empty((self.B, self.H, T, self.D), dtype=self.token_dtype,
                          device=self.device)
        out[:, :, :need].copy_(self._rec[:, :, :need])
        _lib.fc_read_view(self.arc, self.tail_desc, nb, out)
        return out

    def discard_view(self):
        """Free the reconstructed view (rebuilt by the next ``read``)."""
        self._rec = None
        self._rec_blocks = 0

    def crop(self, tokens_to_remove: int):
        """Remove the last ``-tokens_to_remove`` tokens exactly: archived
        blocks below the new end stay verbatim, a partial boundary block
        returns to the raw tail from its reconstruction
        (``_CodecStream.crop``; a negative count, zero does nothing)."""
        if tokens_to_remove > 0:
            raise ValueError("crop takes a negative count of tokens to remove")
        _lib.fc_crop(self.arc, self.tail_desc, int(tokens_to_remove),
                     device=self.device)
        self._rec_blocks = min(self._rec_blocks, self.n_blocks)

    def select_batch(self, idx):
        """Batch row i becomes row ``idx[i]`` (``_CodecStream.select_batch``):
        the archive and the raw tail are gathered by libfc into new storage
        of the same capacity; the view is rebuilt by the next ``read``."""
        self._adopt(self._gathered(host_indices(idx)))

    def _gathered(self, idx):
        """New storage holding batch rows ``idx`` of this stream, filled by
        libfc; the stream itself is not changed."""
        coeffs, scales, arc = self._storage(len(idx), self.capacity)
        tail = torch.zeros((len(idx), self.H, self.R, self.D),
                           dtype=self.token_dtype, device=self.device)
        td = _lib.FcTail()
        ctypes_copy(td, self.tail_desc)
        td.data = tail.data_ptr()
        td.len = 0
        td.stride_b, td.stride_h = tail.stride(0), tail.stride(1)
        _lib.fc_select_batch(self.arc, self.tail_desc, idx, arc, td,
                             device=self.device)
        return len(idx), coeffs, scales, arc, tail, td

    def _adopt(self, gathered):
        (self.B, self.coeffs, self.scales, self.arc, self.tail,
         self.tail_desc) = gathered
        self.discard_view()

    def save_state(self) -> torch.Tensor:
        """Exact image of the stream (header, live coefficients, scales and
        raw tail rows) in a pinned CPU uint8 tensor; the call waits for the
        copies."""
        n = _lib.fc_state_bytes(self.arc, self.tail_desc)
        pin = self.device.type == "cuda"
        buf = torch.empty(n, dtype=torch.uint8, pin_memory=pin)
        _lib.fc_state_save(self.arc, self.tail_desc, buf, device=self.device)
        if pin:
            torch.cuda.current_stream(self.device).synchronize()
        return buf

    def restore_state(self, buf: torch.Tensor):
        """Replace the stream's content with a saved image (bitwise); the
        archive grows first when the image holds more blocks than fit."""
        hd = _lib.fc_state_header(buf)
        self.ensure_capacity(int(hd.n_blocks))
        _lib.fc_state_restore(buf, self.arc, self.tail_desc,
                              device=self.device)
        self.discard_view()

    def reset(self):
        """Empty the stream; capacity and buffers are kept
        (``_CodecStream.reset``)."""
        self.arc.n_blocks = 0
        self.tail_desc.len = 0
        self._rec_blocks = 0


def host_indices(idx):
    """Batch indices as a list of Python ints (a tensor is read back)."""
    if isinstance(idx, torch.Tensor):
        idx = idx.tolist()
    return [int(i) for i in idx]


def ctypes_copy(dst, src):
    for name, _ in src._fields_:
        setattr(dst, name, getattr(src, name))


class CodecKVCache:
    """K and V streams of one attention layer plus decode attention.

    ``coeff_k`` / ``coeff_v`` choose the archive storage: "i8" (int8 codes
    with one fp32 scale per (block, frequency)), "bf16" or "f32".
    ``codec="png"`` selects the lossless PNG tier (anchor + fp32 first
    differences, flashcodec-kv README "Math"): S becomes R and both streams
    store fp32 rows.
    """

    def __init__(self, B: int, Hk: int, D: int, R: int = 8, S: int = 2,
                 coeff_k: str = "i8", coeff_v: str = "i8",
                 token_dtype: torch.dtype = torch.bfloat16, device="cuda",
                 capacity: int = 0, codec: str = "dct"):
        if codec == "png":
            S, coeff_k, coeff_v = R, "f32", "f32"
        self.B, self.Hk, self.D, self.R, self.S = B, Hk, D, R, S
        self.codec = codec
        self.k = CodecStream(B, Hk, D, R, S, coeff_k, token_dtype, device,
                             capacity, codec)
        self.v = CodecStream(B, Hk, D, R, S, coeff_v, token_dtype, device,
                             capacity, codec)
        self.device = self.k.device
        self._ws: Optional[torch.Tensor] = None
        self._plans: dict = {}      # (Hq, n_blocks) -> split count
        self._ws_need: dict = {}    # (Hq, splits) -> workspace bytes

    @property
    def seq_len(self) -> int:
        return self.k.seq_len

    def _grow_to(self, need_blocks: int) -> bool:
        """Grow both streams to hold need_blocks; True when they moved."""
        grew = self.k.ensure_capacity(need_blocks)
        return self.v.ensure_capacity(need_blocks) or grew

    # -- writes ------------------------------------------------------------
    def prefill(self, k: torch.Tensor, v: torch.Tensor):
        """Append a (B, Hk, T, D) prefill: complete blocks are compressed in
        one launch per stream, the remainder becomes the raw tail."""
        if k.shape != v.shape or k.shape[0] != self.B or \
                k.shape[1] != self.Hk or k.shape[3] != self.D:
            raise ValueError("prefill shape mismatch")
        t0 = 0
        # top up a partial tail token by token first (append semantics)
        while self.k.tail_len and t0 < k.shape[2]:
            self.append(k[:, :, t0:t0 + 1], v[:, :, t0:t0 + 1])
            t0 += 1
        if t0 >= k.shape[2]:
            return
        kk, vv = k[:, :, t0:], v[:, :, t0:]
        self._grow_to(self.k.n_blocks + kk.shape[2] // self.R)
        _lib.fc_compress_blocks(kk, self.k.arc, self.k.tail_desc)
        _lib.fc_compress_blocks(vv, self.v.arc, self.v.tail_desc)

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor):
        """decode_step: append one (B, Hk, 1, D) token to both streams."""
        if self.k.tail_len + 1 == self.R:
            self._grow_to(self.k.n_blocks + 1)
        _lib.fc_append_step(k_new, v_new, self.k.arc, self.v.arc,
                            self.k.tail_desc, self.v.tail_desc)

    def step(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
             out: Optional[torch.Tensor] = None,
             softmax_scale: Optional[float] = None, num_splits: int = 0,
             fuse_combine: bool = True, portable: bool = False,
             out_dtype: torch.dtype = torch.float32, overlap: bool = False,
             q_final: bool = False) -> torch.Tensor:
        """One decode step: append the (B, Hk, 1, D) token to both streams,
        then attend q over the updated cache (fc_decode_step: one launch on
        the tensor-core path). Flags as in ``attention``; a step that first
        grows the archive (a copy kernel writes every block) runs without
        the overlap flags, whose precondition that copy would break."""
        if self.k.tail_len + 1 == self.R and self._grow_to(self.k.n_blocks + 1):
            overlap = q_final = False
        Hq = q.shape[1]
        if out is None:
            out = torch.empty((self.B, Hq, 1, self.D), dtype=out_dtype,
                              device=q.device)
        ns = num_splits or self.num_splits(Hq)
        ws = self.workspace(Hq, ns)
        _lib.fc_decode_step(
            q, k_new, v_new, self.k.arc, self.v.arc, self.k.tail_desc,
            self.v.tail_desc, out, ws, softmax_scale=0.0 if softmax_scale is
            None else float(softmax_scale), num_splits=num_splits,
            fuse_combine=fuse_combine, portable=portable, overlap=overlap,
            q_final=q_final)
        if not fuse_combine:
            _lib.fc_combine(ws, self.B, Hq, self.D, ns, out)
        return out

    # -- attention -----------------------------------------------------------
    def num_splits(self, Hq: int) -> int:
        key = (Hq, self.k.n_blocks)     # the plan depends on nothing else
        ns = self._plans.get(key)
        if ns is None:
            ns = _lib.fc_decode_plan(self.k.arc, self.k.tail_desc, Hq)
            self._plans[key] = ns
        return ns

    def tensor_core_path(self, Hq: int, portable: bool = False) -> bool:
        """Whether decode attention runs on the tensor-core kernel."""
        return _lib.fc_decode_kernel(self.k.arc, self.v.arc, Hq, portable) \
            == _lib.FC_KERNEL_TENSOR_CORE

    def workspace(self, Hq: int, num_splits: int) -> torch.Tensor:
        key = (Hq, num_splits)
        need = self._ws_need.get(key)
        if need is None:
            need = _lib.fc_decode_workspace_bytes(self.B, Hq, self.D,
                                                  num_splits)
            self._ws_need[key] = need
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(need, dtype=torch.uint8,
                                   device=self.device)
        return self._ws

    def attention(self, q: torch.Tensor, out: Optional[torch.Tensor] = None,
                  softmax_scale: Optional[float] = None, num_splits: int = 0,
                  fuse_combine: bool = True, portable: bool = False,
                  out_dtype: torch.dtype = torch.float32,
                  overlap: bool = False, q_final: bool = False) -> torch.Tensor:
        """Decode attention of q (B, Hq, 1, D) over archive + tail.
        ``portable`` forces the CUDA-core kernel where the tensor-core kernel
        would apply. ``overlap`` launches it as a programmatic dependent of
        the preceding stream work (FC_DECODE_OVERLAP): valid in a decode loop
        where that work is an append or another attention, not right after a
        prefill of this cache. ``q_final`` (FC_DECODE_Q_FINAL, with
        ``overlap``) states that q was final before that preceding kernel
        started, which lets the kernel compute before it completes."""
        Hq = q.shape[1]
        if out is None:
            out = torch.empty((self.B, Hq, 1, self.D), dtype=out_dtype,
                              device=q.device)
        ns = num_splits or self.num_splits(Hq)
        ws = self.workspace(Hq, ns)
        _lib.fc_decode_attention(
            q, self.k.arc, self.v.arc, self.k.tail_desc, self.v.tail_desc,
            out, ws, softmax_scale=0.0 if softmax_scale is None else
            float(softmax_scale), num_splits=num_splits,
            fuse_combine=fuse_combine,
            portable=portable, overlap=overlap, q_final=q_final)
        if not fuse_combine:
            _lib.fc_combine(ws, self.B, Hq, self.D, ns, out)
        return out

    def storage_bytes(self) -> int:
        return self.k.storage_bytes() + self.v.storage_bytes()

    # -- the pages' cache interface (flashcodec/cache.py, CodecKVCache) --------
    def update(self, k_states: torch.Tensor, v_states: torch.Tensor):
        """Append (B, Hk, m, D) tokens to both streams, archiving across block
        boundaries, and return the reconstructed (key_view, value_view)."""
        self.prefill(k_states, v_states)
        return self.read()

    def read(self):
        """(key_view, value_view): each stream's reconstructed view."""
        return self.k.read(), self.v.read()

    def get_seq_length(self) -> int:
        return self.seq_len

    def crop(self, tokens_to_remove: int):
        """Exact removal of trailing tokens from both streams (negative count,
        e.g. rejected speculative tokens). If the V crop fails, K is put back
        as it was (descriptors and raw tail rows), so the two streams never
        disagree on length."""
        if tokens_to_remove > 0:
            raise ValueError("crop takes a negative count of tokens to remove")
        if (self.k.n_blocks, self.k.tail_len) != \
                (self.v.n_blocks, self.v.tail_len):
            raise RuntimeError("K and V streams disagree on length")
        saved = (self.k.arc.n_blocks, self.k.tail_desc.len,
                 self.k._rec_blocks, self.k.tail.clone())
        self.k.crop(tokens_to_remove)
        try:
            self.v.crop(tokens_to_remove)
        except Exception:
            (self.k.arc.n_blocks, self.k.tail_desc.len, self.k._rec_blocks,
             tail) = saved
            self.k.tail.copy_(tail)
            raise

    def select_batch(self, idx):
        """Gather batch rows of both streams (archives and raw tails); both
        are gathered before either is replaced, so a failure leaves the
        cache as it was."""
        idx = host_indices(idx)
        gk = self.k._gathered(idx)
        gv = self.v._gathered(idx)
        self.k._adopt(gk)
        self.v._adopt(gv)
        self.B = self.k.B
        self._plans.clear()
        self._ws_need.clear()

    reorder_cache = select_batch   # beam search

    def batch_repeat_interleave(self, repeats: int):
        """Replicate every batch row ``repeats`` times (contrastive search)."""
        self.select_batch([b for b in range(self.B) for _ in range(repeats)])

    def batch_select_indices(self, indices):
        """Keep only the given batch rows."""
        self.select_batch(indices)

    def discard_view(self):
        self.k.discard_view()
        self.v.discard_view()

    # -- save / restore ------------------------------------------------------
    def save_state(self) -> dict:
        """Exact images of both streams (``CodecStream.save_state``)."""
        return {"k": self.k.save_state(), "v": self.v.save_state()}

    def restore_state(self, state: dict):
        """Load images written by ``save_state``: the archives and raw tails
        become bitwise the saved ones (same B, Hk, D, R, S and dtypes)."""
        hk = _lib.fc_state_header(state["k"])
        hv = _lib.fc_state_header(state["v"])
        if (hk.n_blocks, hk.tail_len) != (hv.n_blocks, hv.tail_len):
            raise ValueError("K and V images disagree on length")
        self.k.restore_state(state["k"])
        self.v.restore_state(state["v"])

    def to_legacy(self):
        """The pages' legacy export (``FlashCodecCache.to_legacy_cache`` for
        one layer): the reconstructed (keys, values) views."""
        return self.read()

    @classmethod
    def from_legacy(cls, keys: torch.Tensor, values: torch.Tensor, **cfg):
        """The pages' legacy import (``from_legacy_cache`` for one layer):
        a new cache whose streams take the full views through the codec
        once more (lossy again, unlike ``restore_state``)."""
        B, Hk, _, D = keys.shape
        cache = cls(B, Hk, D, token_dtype=keys.dtype, device=keys.device,
                    **cfg)
        cache.prefill(keys, values)
        return cache

    def reset(self):
        """Empty both streams, keeping their capacity."""
        self.k.reset()
        self.v.reset()


def decode_step_layers(caches, qs, k_news, v_news, outs=None,
                       softmax_scale: Optional[float] = None,
                       out_dtype: torch.dtype = torch.float32,
                       overlap: bool = False, q_final: bool = False):
    """One decode step (append + attention) of every cache in ``caches`` in
    one launch (fc_decode_step_layers): cache i appends (k_news[i],
    v_news[i]) and attends qs[i]. The caches are independent streams of the
    same shape (the layers of a step whose queries are all known, or the
    sequences of a serving batch). ``overlap`` / ``q_final`` as in
    ``CodecKVCache.attention``, for a loop of such steps. Returns the
    outputs."""
    n = len(caches)
    for c in caches:
        if c.k.tail_len + 1 == c.R and c._grow_to(c.k.n_blocks + 1):
            overlap = q_final = False   # a growth copy precedes the launch
    Hq = qs[0].shape[1]
    if outs is None:
        outs = [torch.empty((c.B, Hq, 1, c.D), dtype=out_dtype,
                            device=qs[0].device) for c in caches]
    wss = [c.workspace(Hq, c.num_splits(Hq)) for c in caches]
    _lib.fc_decode_step_layers(
        qs, k_news, v_news, [c.k.arc for c in caches],
        [c.v.arc for c in caches], [c.k.tail_desc for c in caches],
        [c.v.tail_desc for c in caches], outs, wss,
        softmax_scale=0.0 if softmax_scale is None else float(softmax_scale),
        overlap=overlap, q_final=q_final)
    return outs


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
