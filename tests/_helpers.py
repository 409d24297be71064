"""Shared helpers of the test suite: build a device cache from synthetic
inputs, bring its archive back for the fp64 oracle, and the tolerance checks.

Tolerances (the parity bar of this hot path):
* int8 codes bit-exact, except +-1 where the oracle's pre-rounding value lies
  within 1e-5 of a half-integer;
* scales within 1e-6 relative;
* bf16 coefficients within 1 bf16 ulp, f32 coefficients within 1e-6 of the
  row's magnitude;
* attention output within 2e-3 max abs and 1e-3 relative L2 of fp64.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle

ATOL_OUT = 2e-3
RTOL_L2_OUT = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_codes(gpu_codes: np.ndarray, y: np.ndarray):
    """GPU int8 codes against the oracle's pre-rounding values y."""
    ref = np.clip(np.rint(y), -127, 127).astype(np.int64)
    got = gpu_codes.astype(np.int64)
    diff = got - ref
    near_half = np.abs(np.abs(y - np.floor(y)) - 0.5) < 1e-5
    bad = (diff != 0) & ~(near_half & (np.abs(diff) <= 1))
    assert not bad.any(), "code mismatch at %d positions (first %s)" % (
        int(bad.sum()), tuple(np.argwhere(bad)[0]))
    return int((diff != 0).sum())


def check_scales(gpu_scales: np.ndarray, ref_scales: np.ndarray):
    ref = np.asarray(ref_scales, dtype=np.float64)
    got = np.asarray(gpu_scales, dtype=np.float64)
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    ok = (rel <= 1e-6) | ((ref == 0) & (got == 0))
    assert ok.all(), "scale mismatch: max rel %.3g" % float(rel[~ok].max())


def check_coeffs(gpu: np.ndarray, C: np.ndarray, coeff: str):
    """Unquantised coefficients (..., nb, S, D) against the exact ones:
    bf16 within one bf16 ulp, f32 within 1e-6 of the block's largest
    coefficient. A coefficient whose exact value vanishes (its block's
    tokens cancel) is rounding noise of the fp64 sum on both sides, so bf16
    differences below 1e-12 of the block's largest coefficient also pass."""
    if coeff == "bf16":
        ref = oracle.round_to_dtype(C, "bf16")
        mag = np.maximum(np.abs(ref), np.abs(gpu)) + 1e-300
        ulp = np.ldexp(1.0, np.frexp(mag)[1] - 8)
        floor = 1e-12 * np.max(np.abs(C), axis=(-2, -1), keepdims=True)
        bad = np.abs(gpu - ref) > np.maximum(ulp, floor)
        if bad.any():
            k = tuple(np.argwhere(bad)[0])
            raise AssertionError(
                "bf16 coefficient mismatch at %d positions; first %s: gpu %r "
                "ref %r exact %r (max %.3g ulp)" % (
                    int(bad.sum()), k, float(gpu[k]), float(ref[k]),
                    float(C[k]), float(np.max(np.abs(gpu - ref) / ulp))))
    else:
        scale = np.max(np.abs(C), axis=(-2, -1), keepdims=True)
        err = np.abs(gpu - C)
        assert np.all(err <= 1e-6 * scale + 1e-30), \
            "f32 coefficient mismatch: %.3g" % float((err / (scale + 1e-30)).max())


def check_out(got: np.ndarray, ref: np.ndarray, what: str = ""):
    err = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert err <= ATOL_OUT and rel <= RTOL_L2_OUT, \
        "%s: max abs %.3g, rel L2 %.3g" % (what, err, rel)
    return err, rel


def _head_archive(stream, b: int, h: int) -> np.ndarray:
    """Live archived coefficients of one (b, h) of a device stream as float64
    (1, 1, nb, S, D): code * fp32 scale when quantised."""
    nb = stream.n_blocks
    c = stream.coeffs[b:b + 1, h:h + 1, :nb]
    if stream.coeff == "i8":
        s = stream.scales[b:b + 1, h:h + 1, :nb]
        return oracle.dequantize(c.cpu().numpy(), s.cpu().numpy())
    return f64(c)


def oracle_on_gpu_archive(cache, q: torch.Tensor, heads=None,
                          scale=None):
    """fp64 reference attention over the GPU's own archive bytes and tail,
    one kv head at a time. Returns (B, Hq, 1, D), or a dict (b, hq) -> (D,)
    when ``heads`` lists the query heads to check."""
    qq = f64(q)
    B, Hq = qq.shape[0], qq.shape[1]
    G = Hq // cache.Hk
    want = None if heads is None else {}
    groups = {}
    for b, hq in (heads if heads is not None else
                  [(b, hq) for b in range(B) for hq in range(Hq)]):
        groups.setdefault((b, hq // G), []).append(hq)
    out = np.empty(qq.shape) if heads is None else None
    for (b, h), hqs in sorted(groups.items()):
        ck = _head_archive(cache.k, b, h)
        cv = _head_archive(cache.v, b, h)
        tk = f64(cache.k.live_tail()[b:b + 1, h:h + 1])
        tv = f64(cache.v.live_tail()[b:b + 1, h:h + 1])
        o = oracle.decode_attention_reference(
            qq[b:b + 1, h * G:(h + 1) * G], ck, cv, tk, tv, cache.R, scale)
        for hq in hqs:
            if out is not None:
                out[b, hq] = o[0, hq - h * G]
            else:
                want[(b, hq)] = o[0, hq - h * G, 0]
    return out if heads is None else want
