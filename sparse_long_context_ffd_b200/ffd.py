"""Thin ctypes binding of the C ABI in include/ffd.h (argument marshalling only).

Every step of the decode path runs in the CUDA library; this module only turns
torch tensors into pointers, picks the current CUDA stream and maps status
codes to exceptions.  There is no fallback: if the library is missing and
cannot be built, importing a function raises.
"""
from __future__ import annotations

import ctypes
import math
import threading
from typing import Optional

from . import build as _build

FFD_OK = 0
FFD_ERR_INVALID_ARG = 1
FFD_ERR_UNSUPPORTED = 2
FFD_ERR_WORKSPACE = 3
FFD_ERR_CUDA = 4
FFD_ERR_DEVICE_CHECK = 5
FFD_ERR_TIMEOUT = 6

FFD_DEVICE_FLAG_BAD_LENGTH = 0x1
FFD_DEVICE_FLAG_TIMEOUT = 0x2
FFD_DEVICE_FLAG_BOUNDS = 0x4  # debug build only (use_debug_library())
FFD_LAST_BLOCK = -1
FFD_MAX_SPLIT_BLOCKS = 512

# Every function the header declares; the library must export all of them.
EXPORTED = (
    "ffd_packed_bytes", "ffd_scale_bytes", "ffd_mask_words", "ffd_decode_workspace_bytes",
    "ffd_workspace_init", "ffd_quantize_keys", "ffd_decode", "ffd_check_device_status",
    "ffd_status_string", "ffd_abi_version", "ffd_decode_no_alloc", "ffd_decode_step",
    "ffd_decode_ex", "ffd_decode_partials", "ffd_partials_region", "ffd_merge_partials",
    "ffd_thumb_bytes", "ffd_residual_bytes", "ffd_quantize_keys_tr", "ffd_decode_tr",
    "ffd_decode_partials_tr", "ffd_decode_append", "ffd_decode_append_tr",
    "ffd_step_graph_create", "ffd_step_graph_run", "ffd_step_graph_destroy",
    "ffd_read_probe", "ffd_no_alloc_device_status",
)

FFD_REFERENCE_RUNNING_MAX = 0
FFD_REFERENCE_SINK_LOCAL = 1        # running maximum started at the sink/local pseudo-max
FFD_REFERENCE_SINK_LOCAL_FIXED = 2  # the sink/local pseudo-max as a fixed threshold

# Size of the library's built-in scratch array used by ffd_decode_no_alloc.
FFD_NO_ALLOC_SCRATCH_BYTES = 16 << 20


class FFDError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class DecodeOptions(ctypes.Structure):
    _fields_ = [("reference", ctypes.c_int32), ("requant_last", ctypes.c_int32),
                ("wait_limit_us", ctypes.c_int32)]


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("split_blocks", ctypes.c_int32)]

    def __repr__(self):
        return "Shape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def make_shape(batch, num_q_heads, num_kv_heads, capacity, block_size, split_blocks,
               head_dim=128) -> Shape:
    return Shape(batch, num_q_heads, num_kv_heads, head_dim, capacity, block_size, split_blocks)


_lock = threading.Lock()
_lib = None


_use_debug = False


def use_debug_library() -> None:
    """Load the bounds-checking debug build (libffd_b200_debug.so: FFD_DEBUG,
    FFD_DEVICE_FLAG_BOUNDS) instead of the product library.  For tests; call
    it before the process's first library call."""
    global _use_debug
    with _lock:
        if _lib is not None and not _use_debug:
            raise RuntimeError("the product library is already loaded in this process")
        _use_debug = True


def _debug_requested() -> bool:
    return _use_debug


def library_path() -> str:
    """The library this process loads: libffd_b200.so, or after
    use_debug_library() the bounds-checking debug build."""
    return _build.DEBUG_LIB if _debug_requested() else _build.LIB


def load_library() -> ctypes.CDLL:
    """Load the library, building it with nvcc first if it is missing or stale."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if _build.is_stale(path):
                _build.build(debug=_debug_requested())
            lib = ctypes.CDLL(path)
            sp = ctypes.POINTER(Shape)
            p, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
            for name in ("ffd_packed_bytes", "ffd_scale_bytes", "ffd_mask_words",
                         "ffd_decode_workspace_bytes", "ffd_thumb_bytes", "ffd_residual_bytes"):
                getattr(lib, name).argtypes = [sp]
                getattr(lib, name).restype = sz
            lib.ffd_workspace_init.argtypes = [sp, p, sz, p]
            lib.ffd_workspace_init.restype = st
            lib.ffd_quantize_keys.argtypes = [sp, p, p, ctypes.c_int32, p, p, p]
            lib.ffd_quantize_keys.restype = st
            lib.ffd_quantize_keys_tr.argtypes = [sp, p, p, ctypes.c_int32, p, p, p, p]
            lib.ffd_quantize_keys_tr.restype = st
            lib.ffd_decode_tr.argtypes = [sp, ctypes.POINTER(DecodeOptions), p, p, p, p, p, p, p,
                                          ctypes.c_float, p, p, p, sz, p]
            lib.ffd_decode_tr.restype = st
            lib.ffd_decode_partials_tr.argtypes = [sp, ctypes.POINTER(DecodeOptions), p, p, p, p,
                                                   p, p, p, ctypes.c_float, p, sz, p]
            lib.ffd_decode_partials_tr.restype = st
            i32 = ctypes.c_int32
            lib.ffd_decode_append.argtypes = [sp, i32, p, p, p, p, p, p, p, p, ctypes.c_float, p,
                                              p, p, sz, p]
            lib.ffd_decode_append.restype = st
            lib.ffd_decode_append_tr.argtypes = [sp, i32, p, p, p, p, p, p, p, p, p,
                                                 ctypes.c_float, p, p, p, sz, p]
            lib.ffd_decode_append_tr.restype = st
            lib.ffd_step_graph_create.argtypes = [sp, i32, i32, ctypes.c_float, i32, p, p, p, p,
                                                  p, p, p, p, p, p, sz, p, sz,
                                                  ctypes.POINTER(ctypes.c_void_p)]
            lib.ffd_step_graph_create.restype = st
            lib.ffd_step_graph_run.argtypes = [p]
            lib.ffd_step_graph_run.restype = st
            lib.ffd_step_graph_destroy.argtypes = [p]
            lib.ffd_step_graph_destroy.restype = None
            lib.ffd_decode.argtypes = [sp, p, p, p, p, p, p, ctypes.c_float, p, p, p, sz, p]
            lib.ffd_decode.restype = st
            lib.ffd_decode_ex.argtypes = [sp, ctypes.POINTER(DecodeOptions), p, p, p, p, p, p,
                                          ctypes.c_float, p, p, p, sz, p]
            lib.ffd_decode_ex.restype = st
            lib.ffd_decode_partials.argtypes = [sp, ctypes.POINTER(DecodeOptions), p, p, p, p, p,
                                                p, ctypes.c_float, p, sz, p]
            lib.ffd_decode_partials.restype = st
            lib.ffd_partials_region.argtypes = [sp, ctypes.POINTER(sz), ctypes.POINTER(sz)]
            lib.ffd_partials_region.restype = st
            lib.ffd_merge_partials.argtypes = [sp, ctypes.c_int32, p, sz, p, p, p, p]
            lib.ffd_merge_partials.restype = st
            lib.ffd_decode_step.argtypes = [sp, p, p, p, p, p, p, ctypes.c_float, p, p, p, sz, p]
            lib.ffd_decode_step.restype = st
            lib.ffd_decode_no_alloc.argtypes = [sp, p, p, p, p, p, p, ctypes.c_float, p, p, p]
            lib.ffd_decode_no_alloc.restype = st
            lib.ffd_no_alloc_device_status.argtypes = [p, p]
            lib.ffd_no_alloc_device_status.restype = st
            lib.ffd_check_device_status.argtypes = [p, ctypes.POINTER(ctypes.c_uint32), p]
            lib.ffd_check_device_status.restype = st
            lib.ffd_read_probe.argtypes = [p, sz, p, p]
            lib.ffd_read_probe.restype = st
            lib.ffd_status_string.argtypes = [st]
            lib.ffd_status_string.restype = ctypes.c_char_p
            lib.ffd_abi_version.argtypes = []
            lib.ffd_abi_version.restype = ctypes.c_int32
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load_library().ffd_status_string(int(status)).decode()


def abi_version() -> int:
    return int(load_library().ffd_abi_version())


def _check(status: int, what: str) -> None:
    if status != FFD_OK:
        raise FFDError(status, what)


def _ptr(t) -> Optional[int]:
    """Device pointer of a CUDA tensor (None passes a null pointer)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("FFD entry points take CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("FFD entry points take contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def packed_bytes(shape: Shape) -> int:
    return int(load_library().ffd_packed_bytes(ctypes.byref(shape)))


def scale_bytes(shape: Shape) -> int:
    return int(load_library().ffd_scale_bytes(ctypes.byref(shape)))


def thumb_bytes(shape: Shape) -> int:
    return int(load_library().ffd_thumb_bytes(ctypes.byref(shape)))


def residual_bytes(shape: Shape) -> int:
    return int(load_library().ffd_residual_bytes(ctypes.byref(shape)))


def mask_words(shape: Shape) -> int:
    return int(load_library().ffd_mask_words(ctypes.byref(shape)))


def decode_workspace_bytes(shape: Shape) -> int:
    return int(load_library().ffd_decode_workspace_bytes(ctypes.byref(shape)))


def workspace_init(shape: Shape, workspace, stream=None) -> None:
    _check(load_library().ffd_workspace_init(ctypes.byref(shape), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(),
                                             _stream(stream)), "ffd_workspace_init")


def quantize_keys(shape: Shape, k, lengths, block_begin: int, k_packed, k_scales,
                  stream=None) -> None:
    _check(load_library().ffd_quantize_keys(ctypes.byref(shape), _ptr(k), _ptr(lengths),
                                            int(block_begin), _ptr(k_packed), _ptr(k_scales),
                                            _stream(stream)), "ffd_quantize_keys")


def quantize_keys_tr(shape: Shape, k, lengths, block_begin: int, k_thumb, k_resid, k_scales,
                     stream=None) -> None:
    """2-bit thumbnails + 8-bit residuals (+ bf16 scales) of the keys."""
    _check(load_library().ffd_quantize_keys_tr(ctypes.byref(shape), _ptr(k), _ptr(lengths),
                                               int(block_begin), _ptr(k_thumb), _ptr(k_resid),
                                               _ptr(k_scales), _stream(stream)),
           "ffd_quantize_keys_tr")


def decode_tr(shape: Shape, q, k, v, k_thumb, k_resid, k_scales, lengths, delta: float, out,
              mask, workspace, reference: int = FFD_REFERENCE_RUNNING_MAX,
              requant_last: bool = False, stream=None, wait_limit_us: int = 0) -> None:
    """Decode step on the thumbnail + residual key format (k is read only when
    requant_last re-quantises the last block; it may be None otherwise)."""
    opts = DecodeOptions(int(reference), 1 if requant_last else 0, int(wait_limit_us))
    _check(load_library().ffd_decode_tr(ctypes.byref(shape), ctypes.byref(opts), _ptr(q), _ptr(k),
                                         _ptr(v), _ptr(k_thumb), _ptr(k_resid), _ptr(k_scales),
                                         _ptr(lengths), float(delta), _ptr(out), _ptr(mask),
                                         _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)), "ffd_decode_tr")


def decode_append(shape: Shape, q, k_new, v_new, k, v, k_packed, k_scales, lengths,
                  delta: float, out, mask, workspace,
                  reference: int = FFD_REFERENCE_RUNNING_MAX, stream=None) -> None:
    """One launch per step: write the new token's K/V rows (k_new, v_new
    [B,Hkv,D]) at position lengths-1, re-quantise the last block, decode."""
    _check(load_library().ffd_decode_append(ctypes.byref(shape), int(reference), _ptr(q),
                                             _ptr(k_new), _ptr(v_new), _ptr(k), _ptr(v),
                                             _ptr(k_packed), _ptr(k_scales), _ptr(lengths),
                                             float(delta), _ptr(out), _ptr(mask), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(),
                                             _stream(stream)), "ffd_decode_append")


def decode_append_tr(shape: Shape, q, k_new, v_new, k, v, k_thumb, k_resid, k_scales, lengths,
                     delta: float, out, mask, workspace,
                     reference: int = FFD_REFERENCE_RUNNING_MAX, stream=None) -> None:
    """decode_append on the thumbnail + residual key format."""
    _check(load_library().ffd_decode_append_tr(ctypes.byref(shape), int(reference), _ptr(q),
                                                _ptr(k_new), _ptr(v_new), _ptr(k), _ptr(v),
                                                _ptr(k_thumb), _ptr(k_resid), _ptr(k_scales),
                                                _ptr(lengths), float(delta), _ptr(out), _ptr(mask),
                                                _ptr(workspace),
                                                workspace.numel() * workspace.element_size(),
                                                _stream(stream)), "ffd_decode_append_tr")


def decode_partials_tr(local_shape: Shape, q, k, v, k_thumb, k_resid, k_scales, local_lengths,
                       delta: float, workspace, requant_last: bool = False, stream=None) -> None:
    """Context shard on the thumbnail + residual format (see decode_partials)."""
    opts = DecodeOptions(FFD_REFERENCE_RUNNING_MAX, 1 if requant_last else 0)
    _check(load_library().ffd_decode_partials_tr(ctypes.byref(local_shape), ctypes.byref(opts),
                                                  _ptr(q), _ptr(k), _ptr(v), _ptr(k_thumb),
                                                  _ptr(k_resid), _ptr(k_scales),
                                                  _ptr(local_lengths), float(delta),
                                                  _ptr(workspace),
                                                  workspace.numel() * workspace.element_size(),
                                                  _stream(stream)), "ffd_decode_partials_tr")


def decode(shape: Shape, q, k, v, k_packed, k_scales, lengths, delta: float, out, mask,
           workspace, stream=None) -> None:
    _check(load_library().ffd_decode(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(k_packed), _ptr(k_scales), _ptr(lengths),
                                      float(delta), _ptr(out), _ptr(mask), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream)), "ffd_decode")


def decode_step(shape: Shape, q, k, v, k_packed, k_scales, lengths, delta: float, out, mask,
                workspace, stream=None) -> None:
    """Re-quantise each sequence's last key block and decode, in one launch."""
    _check(load_library().ffd_decode_step(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(k_packed), _ptr(k_scales), _ptr(lengths),
                                           float(delta), _ptr(out), _ptr(mask), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream)), "ffd_decode_step")


def decode_ex(shape: Shape, q, k, v, k_packed, k_scales, lengths, delta: float, out, mask,
              workspace, reference: int = FFD_REFERENCE_RUNNING_MAX, requant_last: bool = False,
              stream=None, wait_limit_us: int = 0) -> None:
    """ffd_decode / ffd_decode_step with the reference-maximum mode and the
    kernel's wait limit (0: the default 2 s; see ffd_decode_options)."""
    opts = DecodeOptions(int(reference), 1 if requant_last else 0, int(wait_limit_us))
    _check(load_library().ffd_decode_ex(ctypes.byref(shape), ctypes.byref(opts), _ptr(q), _ptr(k),
                                         _ptr(v), _ptr(k_packed), _ptr(k_scales), _ptr(lengths),
                                         float(delta), _ptr(out), _ptr(mask), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)), "ffd_decode_ex")


def decode_partials(local_shape: Shape, q, k, v, k_packed, k_scales, local_lengths,
                    delta: float, workspace, requant_last: bool = False, stream=None) -> None:
    """Context shard: split partials and bits into the workspace, no merge."""
    opts = DecodeOptions(FFD_REFERENCE_RUNNING_MAX, 1 if requant_last else 0)
    _check(load_library().ffd_decode_partials(ctypes.byref(local_shape), ctypes.byref(opts),
                                               _ptr(q), _ptr(k), _ptr(v), _ptr(k_packed),
                                               _ptr(k_scales), _ptr(local_lengths), float(delta),
                                               _ptr(workspace),
                                               workspace.numel() * workspace.element_size(),
                                               _stream(stream)), "ffd_decode_partials")


def partials_region(local_shape: Shape):
    """(offset, bytes) of the workspace region the shards exchange."""
    off, nbytes = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(load_library().ffd_partials_region(ctypes.byref(local_shape), ctypes.byref(off),
                                               ctypes.byref(nbytes)), "ffd_partials_region")
    return int(off.value), int(nbytes.value)


def merge_partials(local_shape: Shape, num_shards: int, gathered, global_lengths, out, mask,
                   stream=None) -> None:
    """Merge the gathered shard regions into the output rows and global mask."""
    _check(load_library().ffd_merge_partials(ctypes.byref(local_shape), int(num_shards),
                                              _ptr(gathered),
                                              gathered.numel() * gathered.element_size(),
                                              _ptr(global_lengths), _ptr(out), _ptr(mask),
                                              _stream(stream)), "ffd_merge_partials")


def decode_no_alloc(shape: Shape, q, k, v, k_packed, k_scales, lengths, delta: float, out,
                    mask, stream=None) -> None:
    """ffd_decode without a workspace: for callers that cannot allocate device
    memory.  Uses the library's built-in 16 MiB scratch array; calls on one
    device must not overlap on the GPU.  The first call on a device should
    come before any stream capture.  Device-side flags: no_alloc_device_status."""
    _check(load_library().ffd_decode_no_alloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                              _ptr(k_packed), _ptr(k_scales), _ptr(lengths),
                                              float(delta), _ptr(out), _ptr(mask),
                                              _stream(stream)), "ffd_decode_no_alloc")


def no_alloc_device_status(stream=None) -> int:
    """Synchronise, read and clear the flags the last decode_no_alloc call on
    the current device left in the library's built-in array; returns
    FFD_DEVICE_FLAG_* bits."""
    flags = ctypes.c_uint32(0)
    st = load_library().ffd_no_alloc_device_status(ctypes.byref(flags), _stream(stream))
    if st not in (FFD_OK, FFD_ERR_DEVICE_CHECK, FFD_ERR_TIMEOUT):
        raise FFDError(st, "ffd_no_alloc_device_status")
    return int(flags.value)


def read_probe(buf, sink, stream=None) -> None:
    """ffd_read_probe: read the whole (16-byte aligned) device tensor `buf`
    once; `sink` is a device int32/uint32 tensor of at least one element."""
    _check(load_library().ffd_read_probe(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink),
                                         _stream(stream)), "ffd_read_probe")


def check_device_status(workspace, stream=None) -> int:
    """Synchronise, read and clear the device flags; returns FFD_DEVICE_FLAG_* bits."""
    flags = ctypes.c_uint32(0)
    st = load_library().ffd_check_device_status(_ptr(workspace), ctypes.byref(flags),
                                                _stream(stream))
    if st not in (FFD_OK, FFD_ERR_DEVICE_CHECK, FFD_ERR_TIMEOUT):
        raise FFDError(st, "ffd_check_device_status")
    return int(flags.value)


class DecodeBuffers:
    """Device buffers one decode step needs besides the caller's KV cache.

    Allocation is PyTorch's job (caching allocator); the library only
    receives pointers.
    """

    def __init__(self, shape: Shape, device="cuda"):
        import torch
        self.shape = shape
        B, Hq, Hkv = shape.batch, shape.num_q_heads, shape.num_kv_heads
        cap, T, D = shape.capacity, shape.block_size, shape.head_dim
        self.k_packed = torch.empty((B, Hkv, cap, D // 2), dtype=torch.uint8, device=device)
        self.k_scales = torch.empty((B, Hkv, cap // T, D), dtype=torch.bfloat16, device=device)
        self.out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=device)
        self.mask = torch.empty((B, Hkv, math.ceil(cap // T / 32)), dtype=torch.int32,
                                device=device)
        ws = decode_workspace_bytes(shape)
        self.workspace = torch.empty((max(ws, 256) + 15) // 16 * 16, dtype=torch.uint8,
                                     device=device)
        workspace_init(shape, self.workspace)


class ThumbResidBuffers(DecodeBuffers):
    """DecodeBuffers plus the thumbnail + residual key copy (k_packed unused)."""

    def __init__(self, shape: Shape, device="cuda"):
        import torch
        super().__init__(shape, device)
        B, Hkv, cap, D = shape.batch, shape.num_kv_heads, shape.capacity, shape.head_dim
        self.k_packed = None
        self.k_thumb = torch.empty((B, Hkv, cap, D // 4), dtype=torch.uint8, device=device)
        self.k_resid = torch.empty((B, Hkv, cap, D), dtype=torch.uint8, device=device)


class StepGraph:
    """Owner of a native decode-step graph (ffd_step_graph_*): one call runs
    H2D of the inputs, the fused append + decode and D2H of the results."""

    def __init__(self, shape: Shape, fmt: int, reference: int, delta: float, advance: bool,
                 host_in, dev_in, k, v, k_copy, k_resid, k_scales, lengths, dev_result,
                 host_result, mask_offset: int, workspace):
        self._lib = load_library()
        handle = ctypes.c_void_p(None)
        _check(self._lib.ffd_step_graph_create(
            ctypes.byref(shape), int(fmt), int(reference), float(delta), 1 if advance else 0,
            host_in.data_ptr(), _ptr(dev_in), _ptr(k), _ptr(v), _ptr(k_copy), _ptr(k_resid),
            _ptr(k_scales), _ptr(lengths), _ptr(dev_result), host_result.data_ptr(),
            int(mask_offset), _ptr(workspace), workspace.numel() * workspace.element_size(),
            ctypes.byref(handle)), "ffd_step_graph_create")
        self._handle = handle

    def run(self) -> None:
        _check(self._lib.ffd_step_graph_run(self._handle), "ffd_step_graph_run")

    def close(self) -> None:
        if self._handle is not None and self._handle.value:
            self._lib.ffd_step_graph_destroy(self._handle)
        self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown
            pass
