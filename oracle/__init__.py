"""ctypes wrapper of the plain C oracle (``ffd_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg and CPU reference arm are the only callers.  The product path never imports this
package, and this package imports nothing from the product.

All arrays are numpy: bf16 tensors are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ffd_oracle.c")
_LIB = os.path.join(_HERE, "libffd_oracle.so")
_lock = threading.Lock()
_lib = None

OK, BAD_ARG, BAD_LENGTH = 0, 1, 2

# Reference maximum of the Top-delta filter (ffd_oracle.c, select_ref):
RUNNING_MAX = 0        # running maximum inside each split (R5)
PSEUDO_MAX_SEEDED = 1  # running maximum started at the sink/local pseudo-max (R15)
PSEUDO_MAX_FIXED = 2   # the pages' rule: s_j >= pseudo-max - delta, fixed threshold (R15, R19)


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (strict IEEE fp32: no contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-fno-unsafe-math-optimizations", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i, p = ctypes.c_int, ctypes.c_void_p
            lib.ffdo_quantize_keys.argtypes = [i, i, i, i, i, p, p, i, p, p]
            lib.ffdo_fold_query.argtypes = [i, p, p, p, p]
            lib.ffdo_fold_query.restype = None
            lib.ffdo_block_scores.argtypes = [i, i, i, i, i, i, p, p, p, p, p]
            lib.ffdo_select.argtypes = [i, i, i, i, i, i, p, p, ctypes.c_float, p, p]
            lib.ffdo_attend.argtypes = [i, i, i, i, i, i, p, p, p, p, p, p, p]
            lib.ffdo_decode.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p,
                                        ctypes.c_float, p, p, p]
            lib.ffdo_decode_pseudo_max.argtypes = lib.ffdo_decode.argtypes
            lib.ffdo_select_pseudo_max.argtypes = lib.ffdo_select.argtypes
            lib.ffdo_select_pseudo_max_fixed.argtypes = lib.ffdo_select.argtypes
            lib.ffdo_decode_ref.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p,
                                            ctypes.c_float, i, p, p, p]
            lib.ffdo_quantize_keys_tr.argtypes = [i, i, i, i, i, p, p, i, p, p, p]
            lib.ffdo_fold_query_tr.argtypes = [i, p, p, p, p]
            lib.ffdo_fold_query_tr.restype = None
            lib.ffdo_block_scores_tr.argtypes = [i, i, i, i, i, i, p, p, p, p, p]
            lib.ffdo_reconstruct_keys_tr.argtypes = [i, i, i, i, i, p, p, p, p, p]
            lib.ffdo_attend_tr.argtypes = [i, i, i, i, i, i, p, p, p, p, p, p, p, p, p]
            lib.ffdo_decode_tr.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p,
                                           ctypes.c_float, i, p, p, p]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc):
    if rc != OK:
        raise OracleError({BAD_ARG: "invalid argument", BAD_LENGTH: "length out of range"}.get(rc, rc))


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def mask_words(capacity: int, block_size: int) -> int:
    return (capacity // block_size + 31) // 32


def quantize_keys(k, lengths, block_size, block_begin=0, packed=None, scales=None):
    """int4 copy of bf16 keys ``k`` [B,Hkv,cap,D]; updates ``packed``/``scales`` in place."""
    k = _c(k, np.uint16)
    lengths = _c(lengths, np.int32)
    B, Hkv, cap, D = k.shape
    if packed is None:
        packed = np.zeros((B, Hkv, cap, D // 2), dtype=np.uint8)
    if scales is None:
        scales = np.zeros((B, Hkv, cap // block_size, D), dtype=np.uint16)
    assert packed.flags.c_contiguous and scales.flags.c_contiguous
    _check(_load().ffdo_quantize_keys(B, Hkv, cap, D, block_size, _ptr(k), _ptr(lengths),
                                      int(block_begin), _ptr(packed), _ptr(scales)))
    return packed, scales


def fold_query(q_head, scale_block):
    q_head = _c(q_head, np.uint16)
    scale_block = _c(scale_block, np.uint16)
    qi = np.zeros(q_head.shape[0], dtype=np.int8)
    c = np.zeros(1, dtype=np.float32)
    _load().ffdo_fold_query(q_head.shape[0], _ptr(q_head), _ptr(scale_block), _ptr(qi), _ptr(c))
    return qi, float(c[0])


def block_scores(q, packed, scales, lengths, block_size):
    q = _c(q, np.uint16)
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint16)
    lengths = _c(lengths, np.int32)
    B, Hq, D = q.shape
    _, Hkv, cap, _ = packed.shape
    out = np.empty((B, Hq, cap // block_size), dtype=np.float32)
    _check(_load().ffdo_block_scores(B, Hq, Hkv, cap, D, block_size, _ptr(q), _ptr(packed),
                                     _ptr(scales), _ptr(lengths), _ptr(out)))
    return out


def _reference(pseudo_max, reference):
    if reference is None:
        return PSEUDO_MAX_SEEDED if pseudo_max else RUNNING_MAX
    if reference not in (RUNNING_MAX, PSEUDO_MAX_SEEDED, PSEUDO_MAX_FIXED):
        raise OracleError(f"unknown reference {reference!r}")
    return reference


def select(scores, lengths, num_kv_heads, capacity, block_size, split_blocks, delta,
           pseudo_max=False, reference=None):
    """Returns (keep [B,Hq,nblk] uint8, mask [B,Hkv,words] uint32).  pseudo_max
    selects the seeded sink/local reference maximum instead of starting each
    split's running maximum at minus infinity; ``reference`` (RUNNING_MAX,
    PSEUDO_MAX_SEEDED, PSEUDO_MAX_FIXED) overrides it."""
    ref = _reference(pseudo_max, reference)
    scores = _c(scores, np.float32)
    lengths = _c(lengths, np.int32)
    B, Hq, nblk = scores.shape
    keep = np.zeros((B, Hq, nblk), dtype=np.uint8)
    mask = np.zeros((B, num_kv_heads, mask_words(capacity, block_size)), dtype=np.uint32)
    fn = {RUNNING_MAX: _load().ffdo_select, PSEUDO_MAX_SEEDED: _load().ffdo_select_pseudo_max,
          PSEUDO_MAX_FIXED: _load().ffdo_select_pseudo_max_fixed}[ref]
    _check(fn(B, Hq, num_kv_heads, capacity, block_size, split_blocks, _ptr(scores), _ptr(lengths),
              float(delta), _ptr(keep), _ptr(mask)))
    return keep, mask


def attend(q, k, v, lengths, mask, block_size):
    """fp64 attention over the selected blocks.  Returns (out [B,Hq,D] f64, lse [B,Hq])."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    lengths = _c(lengths, np.int32)
    mask = _c(mask, np.uint32)
    B, Hq, D = q.shape
    _, Hkv, cap, _ = k.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    _check(_load().ffdo_attend(B, Hq, Hkv, cap, D, block_size, _ptr(q), _ptr(k), _ptr(v),
                               _ptr(lengths), _ptr(mask), _ptr(out), _ptr(lse)))
    return out, lse


def decode(q, k, v, packed, scales, lengths, block_size, split_blocks, delta, pseudo_max=False,
           reference=None):
    """The whole step.  Returns (out [B,Hq,D] f64, mask [B,Hkv,words] u32, scores).
    Reference maximum as ``select``."""
    ref = _reference(pseudo_max, reference)
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    lengths = _c(lengths, np.int32)
    packed = None if packed is None else _c(packed, np.uint8)
    scales = None if scales is None else _c(scales, np.uint16)
    B, Hq, D = q.shape
    _, Hkv, cap, _ = k.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    mask = np.zeros((B, Hkv, mask_words(cap, block_size)), dtype=np.uint32)
    scores = np.zeros((B, Hq, cap // block_size), dtype=np.float32)
    _check(_load().ffdo_decode_ref(B, Hq, Hkv, cap, D, block_size, split_blocks, _ptr(q), _ptr(k),
                                   _ptr(v), _ptr(packed), _ptr(scales), _ptr(lengths), float(delta),
                                   ref, _ptr(out), _ptr(mask), _ptr(scores)))
    return out, mask, scores


def mask_to_blocks(mask_row, nblk):
    """Expand one [words] uint32 mask row into a bool array of nblk blocks."""
    bits = np.unpackbits(np.asarray(mask_row, dtype="<u4").view(np.uint8), bitorder="little")
    return bits[:nblk].astype(bool)


# ---- thumbnail + residual key format (2-bit thumbnails, 8-bit residuals) ----

def quantize_keys_tr(k, lengths, block_size, block_begin=0, thumb=None, resid=None, scales=None):
    """Thumbnail + residual copy of bf16 keys ``k`` [B,Hkv,cap,D]: returns
    (thumb [B,Hkv,cap,D/4] u8, resid [B,Hkv,cap,D] u8, scales [B,Hkv,nblk,D]
    bf16 bits), updated in place when given."""
    k = _c(k, np.uint16)
    lengths = _c(lengths, np.int32)
    B, Hkv, cap, D = k.shape
    if thumb is None:
        thumb = np.zeros((B, Hkv, cap, D // 4), dtype=np.uint8)
    if resid is None:
        resid = np.zeros((B, Hkv, cap, D), dtype=np.uint8)
    if scales is None:
        scales = np.zeros((B, Hkv, cap // block_size, D), dtype=np.uint16)
    assert thumb.flags.c_contiguous and resid.flags.c_contiguous and scales.flags.c_contiguous
    _check(_load().ffdo_quantize_keys_tr(B, Hkv, cap, D, block_size, _ptr(k), _ptr(lengths),
                                         int(block_begin), _ptr(thumb), _ptr(resid),
                                         _ptr(scales)))
    return thumb, resid, scales


def fold_query_tr(q_head, scale_block):
    q_head = _c(q_head, np.uint16)
    scale_block = _c(scale_block, np.uint16)
    qi = np.zeros(q_head.shape[0], dtype=np.int8)
    c = np.zeros(1, dtype=np.float32)
    _load().ffdo_fold_query_tr(q_head.shape[0], _ptr(q_head), _ptr(scale_block), _ptr(qi), _ptr(c))
    return qi, float(c[0])


def block_scores_tr(q, thumb, scales, lengths, block_size):
    q = _c(q, np.uint16)
    thumb = _c(thumb, np.uint8)
    scales = _c(scales, np.uint16)
    lengths = _c(lengths, np.int32)
    B, Hq, D = q.shape
    _, Hkv, cap, _ = thumb.shape
    out = np.empty((B, Hq, cap // block_size), dtype=np.float32)
    _check(_load().ffdo_block_scores_tr(B, Hq, Hkv, cap, D, block_size, _ptr(q), _ptr(thumb),
                                        _ptr(scales), _ptr(lengths), _ptr(out)))
    return out


def reconstruct_keys_tr(thumb, resid, scales, lengths, block_size):
    """The computer's keys k_hat [B,Hkv,cap,D] (float64; zero past the length)."""
    thumb = _c(thumb, np.uint8)
    resid = _c(resid, np.uint8)
    scales = _c(scales, np.uint16)
    lengths = _c(lengths, np.int32)
    B, Hkv, cap, D = resid.shape
    out = np.zeros((B, Hkv, cap, D), dtype=np.float64)
    _check(_load().ffdo_reconstruct_keys_tr(B, Hkv, cap, D, block_size, _ptr(thumb), _ptr(resid),
                                            _ptr(scales), _ptr(lengths), _ptr(out)))
    return out


def attend_tr(q, thumb, resid, scales, v, lengths, mask, block_size):
    """fp64 attention over the selected blocks with reconstructed keys."""
    q = _c(q, np.uint16)
    thumb = _c(thumb, np.uint8)
    resid = _c(resid, np.uint8)
    scales = _c(scales, np.uint16)
    v = _c(v, np.uint16)
    lengths = _c(lengths, np.int32)
    mask = _c(mask, np.uint32)
    B, Hq, D = q.shape
    _, Hkv, cap, _ = v.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    _check(_load().ffdo_attend_tr(B, Hq, Hkv, cap, D, block_size, _ptr(q), _ptr(thumb),
                                  _ptr(resid), _ptr(scales), _ptr(v), _ptr(lengths), _ptr(mask),
                                  _ptr(out), _ptr(lse)))
    return out, lse


def decode_tr(q, v, thumb, resid, scales, lengths, block_size, split_blocks, delta,
              pseudo_max=False, reference=None):
    """The whole step on the thumbnail + residual format.  Returns
    (out [B,Hq,D] f64, mask [B,Hkv,words] u32, scores).  Reference maximum as
    ``select``."""
    ref = _reference(pseudo_max, reference)
    q = _c(q, np.uint16)
    v = _c(v, np.uint16)
    thumb = _c(thumb, np.uint8)
    resid = _c(resid, np.uint8)
    scales = _c(scales, np.uint16)
    lengths = _c(lengths, np.int32)
    B, Hq, D = q.shape
    _, Hkv, cap, _ = v.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    mask = np.zeros((B, Hkv, mask_words(cap, block_size)), dtype=np.uint32)
    scores = np.zeros((B, Hq, cap // block_size), dtype=np.float32)
    _check(_load().ffdo_decode_tr(B, Hq, Hkv, cap, D, block_size, split_blocks, _ptr(q), _ptr(v),
                                  _ptr(thumb), _ptr(resid), _ptr(scales), _ptr(lengths),
                                  float(delta), ref, _ptr(out), _ptr(mask),
                                  _ptr(scores)))
    return out, mask, scores
