"""ctypes binding of libtpla (argument marshalling only).

Every step of the decode path runs in libtpla's CUDA kernels; this module
only turns torch tensors into ``tpla_tensor`` descriptors, allocates outputs
and workspace with torch when the caller did not, and raises on non-zero
status.  There is no CPU or PyTorch fallback: if the library cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libtpla.so")

TPLA_BF16, TPLA_F32, TPLA_I32 = 1, 2, 3
ROPE_MODES = {"replicate": 0, "split": 1}
KERNELS = {"auto": 0, "generic": 1, "sm100": 2}
STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported", -3: "CUDA error",
          -4: "workspace", -5: "device timeout", -6: "device bounds"}


class TplaError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        msg = f"{fn} failed: {STATUS.get(status, status)} ({status})"
        if status == -3:
            msg += f", cudaError {cuda_error}"
        super().__init__(msg)


class TplaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("ndim", ctypes.c_int32), ("shape", ctypes.c_int64 * 4),
                ("stride", ctypes.c_int64 * 4)]


class TplaDecodeOpts(ctypes.Structure):
    _fields_ = [("num_splits", ctypes.c_int32), ("shard", ctypes.c_int32),
                ("kernel", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


_lib = None
_lock = threading.Lock()
_P = ctypes.POINTER


def lib() -> ctypes.CDLL:
    """Load libtpla.so (building it in-tree with nvcc first if it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                from . import build as _build
                _build.build()
            L = ctypes.CDLL(_LIB_PATH)
            T = _P(TplaTensor)
            L.tpla_decode_ex.argtypes = [T, T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                         T, T, _P(TplaDecodeOpts), ctypes.c_void_p]
            L.tpla_decode.argtypes = [T, T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                      T, T, ctypes.c_void_p]
            L.tpla_decode_workspace_size.argtypes = [T, T, T, T, ctypes.c_int, ctypes.c_int, T,
                                                     _P(TplaDecodeOpts), _P(ctypes.c_size_t)]
            L.tpla_lse_merge.argtypes = [T, T, T, T, ctypes.c_void_p]
            L.tpla_hadamard_apply.argtypes = [T, ctypes.c_int, ctypes.c_void_p]
            L.tpla_vup_combine.argtypes = [T, T, T, ctypes.c_void_p]
            L.tpla_error_string.argtypes = [ctypes.c_int]
            L.tpla_error_string.restype = ctypes.c_char_p
            L.tpla_get_device_status.argtypes = [ctypes.c_void_p, _P(ctypes.c_int)]
            L.tpla_selftest_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_void_p]
            L.tpla_latent_covariance.argtypes = [T, T, T, ctypes.c_void_p]
            L.tpla_covariance_finalize.argtypes = [T, T, ctypes.c_int64, T, T, ctypes.c_void_p]
            L.tpla_rotate_apply.argtypes = [T, T, ctypes.c_void_p, ctypes.c_size_t,
                                            ctypes.c_void_p]
            L.tpla_cache_append.argtypes = [T, T, T, T, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_float, ctypes.c_void_p]
            L.tpla_prefill.argtypes = [T, T, ctypes.c_int, T, T, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_float, ctypes.c_float, T, T, ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_void_p]
            L.tpla_prefill_workspace_size.argtypes = [T, _P(ctypes.c_size_t)]
            for f in ("tpla_decode_ex", "tpla_decode", "tpla_decode_workspace_size",
                      "tpla_lse_merge", "tpla_hadamard_apply", "tpla_vup_combine",
                      "tpla_last_cuda_error", "tpla_get_device_status", "tpla_version",
                      "tpla_selftest_wait_timeout", "tpla_latent_covariance",
                      "tpla_covariance_finalize", "tpla_rotate_apply", "tpla_cache_append",
                      "tpla_prefill", "tpla_prefill_workspace_size"):
                getattr(L, f).restype = ctypes.c_int
            L.tpla_launch_count.restype = ctypes.c_int64
            _lib = L
    return _lib


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise TplaError(fn, rc, lib().tpla_last_cuda_error() if rc == -3 else 0)


_DT = {torch.bfloat16: TPLA_BF16, torch.float32: TPLA_F32, torch.int32: TPLA_I32}


def desc(t: torch.Tensor | None):
    """tpla_tensor descriptor of a torch tensor (None -> NULL)."""
    if t is None:
        return None
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}")
    if t.dim() > 4:
        raise ValueError("at most 4 dimensions")
    d = TplaTensor()
    d.data = t.data_ptr() if t.numel() else None
    d.dtype = _DT[t.dtype]
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _ref(d):
    return ctypes.byref(d) if d is not None else None


def _on_current_device(*tensors) -> None:
    """libtpla receives raw device addresses and launches on the current
    device, so every tensor must be a CUDA tensor on that device: a host
    tensor or one on another GPU would be read at a wrong address."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"libtpla takes CUDA tensors; got one on {t.device}")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on different devices: {dev} and {t.device}")
    if dev is not None and dev.index is not None and dev.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {dev} but the current device is "
                         f"cuda:{torch.cuda.current_device()}")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _opts(num_splits, shard, kernel, ws=None, ws_bytes=0) -> TplaDecodeOpts:
    o = TplaDecodeOpts()
    o.num_splits = int(num_splits)
    o.shard = -1 if shard is None else int(shard)
    o.kernel = KERNELS[kernel] if isinstance(kernel, str) else int(kernel)
    o.reserved = 0
    o.workspace = ws
    o.workspace_bytes = ws_bytes
    return o


def decode_workspace_size(q, kv_cache, seq_lens, page_table, G, rope_mode, out, *,
                          num_splits=0, shard=None, kernel="auto") -> int:
    _on_current_device(q, kv_cache, seq_lens, page_table, out)
    n = ctypes.c_size_t(0)
    o = _opts(num_splits, shard, kernel)
    rc = lib().tpla_decode_workspace_size(
        _ref(desc(q)), _ref(desc(kv_cache)), _ref(desc(seq_lens)), _ref(desc(page_table)),
        int(G), ROPE_MODES[rope_mode], _ref(desc(out)), ctypes.byref(o), ctypes.byref(n))
    _check("tpla_decode_workspace_size", rc)
    return int(n.value)


def decode(q, kv_cache, seq_lens, page_table, G=1, rope_mode="replicate", scale=None,
           out=None, lse=None, *, num_splits=0, shard=None, kernel="auto",
           workspace=None, out_dtype=torch.float32, want_lse=True, stream=None):
    """MLA (G=1) / TPLA (G>1) latent-KV decode through ``tpla_decode_ex``.

    Returns (out, lse).  See include/tpla.h for layouts.
    """
    if scale is None:
        raise ValueError("scale is required")
    _on_current_device(q, kv_cache, seq_lens, page_table, out, lse, workspace)
    B, H = q.shape[0], q.shape[1]
    width = 512 if shard is None else 512 // G
    n_sh = G if shard is None else 1
    if out is None:
        out = torch.empty((B, H, width), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, n_sh), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(q, kv_cache, seq_lens, page_table, G, rope_mode, out,
                                 num_splits=num_splits, shard=shard, kernel=kernel)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty((need + 15) // 16 * 16, dtype=torch.uint8, device=q.device)
    o = _opts(num_splits, shard, kernel, workspace.data_ptr() if need else None,
              workspace.numel() * workspace.element_size() if need else 0)
    rc = lib().tpla_decode_ex(
        _ref(desc(q)), _ref(desc(kv_cache)), _ref(desc(seq_lens)), _ref(desc(page_table)),
        int(G), ROPE_MODES[rope_mode], ctypes.c_float(scale), _ref(desc(out)), _ref(desc(lse)),
        ctypes.byref(o), _stream(stream))
    _check("tpla_decode_ex", rc)
    return out, lse


def decode_simple(q, kv_cache, seq_lens, page_table, G, rope_mode, scale, out, lse=None,
                  stream=None):
    """``tpla_decode`` (default options, library-managed workspace)."""
    _on_current_device(q, kv_cache, seq_lens, page_table, out, lse)
    rc = lib().tpla_decode(
        _ref(desc(q)), _ref(desc(kv_cache)), _ref(desc(seq_lens)), _ref(desc(page_table)),
        int(G), ROPE_MODES[rope_mode], ctypes.c_float(scale), _ref(desc(out)), _ref(desc(lse)),
        _stream(stream))
    _check("tpla_decode", rc)
    return out, lse


def lse_merge(o_parts, lse_parts, out=None, lse=None, stream=None):
    _on_current_device(o_parts, lse_parts, out, lse)
    S, B, H, Wd = o_parts.shape
    if out is None:
        out = torch.empty((B, H, Wd), dtype=torch.float32, device=o_parts.device)
    if lse is None:
        lse = torch.empty((B, H, lse_parts.shape[3]), dtype=torch.float32, device=o_parts.device)
    rc = lib().tpla_lse_merge(_ref(desc(o_parts)), _ref(desc(lse_parts)), _ref(desc(out)),
                              _ref(desc(lse)), _stream(stream))
    _check("tpla_lse_merge", rc)
    return out, lse


def hadamard_apply(buf, dim=512, stream=None):
    """In-place orthonormal Walsh-Hadamard transform of buf[..., :dim]."""
    _on_current_device(buf)
    rc = lib().tpla_hadamard_apply(_ref(desc(buf)), int(dim), _stream(stream))
    _check("tpla_hadamard_apply", rc)
    return buf


def vup_combine(out_latent, W_uv, y=None, stream=None):
    _on_current_device(out_latent, W_uv, y)
    B, H = out_latent.shape[0], out_latent.shape[1]
    if y is None:
        y = torch.empty((B, H, W_uv.shape[2]), dtype=torch.float32, device=out_latent.device)
    rc = lib().tpla_vup_combine(_ref(desc(out_latent)), _ref(desc(W_uv)), _ref(desc(y)),
                                _stream(stream))
    _check("tpla_vup_combine", rc)
    return y


def latent_covariance(rows, stream=None):
    """(mean [512], covariance [512, 512]) f32 of the first 512 columns of
    the calibration rows ([N, >= 512] or [B, H, >= 512] bf16), computed by
    tpla_latent_covariance + tpla_covariance_finalize."""
    _on_current_device(rows)
    dev = rows.device
    C = torch.zeros((512, 512), dtype=torch.float32, device=dev)
    ssum = torch.zeros((512,), dtype=torch.float32, device=dev)
    st = _stream(stream)
    _check("tpla_latent_covariance",
           lib().tpla_latent_covariance(_ref(desc(rows)), _ref(desc(C)), _ref(desc(ssum)), st))
    n = rows.shape[0] * (rows.shape[1] if rows.dim() == 3 else 1)
    cov = torch.empty_like(C)
    mean = torch.empty_like(ssum)
    _check("tpla_covariance_finalize",
           lib().tpla_covariance_finalize(_ref(desc(C)), _ref(desc(ssum)), int(n),
                                          _ref(desc(cov)), _ref(desc(mean)), st))
    return mean, cov


def rotate_apply(buf, U, scratch=None, stream=None):
    """In place x <- x U on the first 512 columns of every row of ``buf``
    (bf16), U [512, 512] bf16 (tpla_rotate_apply).  ``scratch`` (a device
    tensor of at least H * 512 f32) is allocated when not given."""
    _on_current_device(buf, U, scratch)
    if scratch is None:
        lead = buf.shape[0]
        per = (buf.shape[1] if buf.dim() == 3 else 1) * 512
        scratch = torch.empty((max(1, min(lead, max(1, (1 << 24) // per))) * per,),
                              dtype=torch.float32, device=buf.device)
    rc = lib().tpla_rotate_apply(_ref(desc(buf)), _ref(desc(U)), scratch.data_ptr(),
                                 scratch.numel() * scratch.element_size(), _stream(stream))
    _check("tpla_rotate_apply", rc)
    return buf


def cache_append(kv_new, positions, page_table, kv_cache, norm_groups=1, hadamard=False,
                 eps=1e-6, stream=None):
    """Store each request's new token row (``kv_new`` [B, 576]: latent before
    its RMS normalisation, then the rope key) into ``kv_cache`` at token
    ``positions[b]``, normalised over ``norm_groups`` shards, optionally
    rotated first (tpla_cache_append).  In place on ``kv_cache``."""
    _on_current_device(kv_new, positions, page_table, kv_cache)
    rc = lib().tpla_cache_append(_ref(desc(kv_new)), _ref(desc(positions)),
                                 _ref(desc(page_table)) if page_table is not None else None,
                                 _ref(desc(kv_cache)), int(norm_groups), 1 if hadamard else 0,
                                 ctypes.c_float(eps), _stream(stream))
    _check("tpla_cache_append", rc)
    return kv_cache


def prefill(q, kv_new, start, page_row, kv_cache, norm_groups=1, hadamard=False, eps=1e-6,
            scale=None, out=None, lse=None, *, workspace=None, out_dtype=torch.float32,
            want_lse=True, stream=None):
    """Prefill of one request (tpla_prefill): store the prompt rows ``kv_new``
    [T, 576] at positions start .. start + T - 1 through the request's page
    row ``page_row`` [max_pages] (as ``cache_append`` stores a row), then exact
    MLA of every prompt token (``q`` [T, H, 576]) over its causal prefix.
    Returns (out [T, H, 512], lse [T, H, 1]); ``kv_cache`` is updated in
    place."""
    if scale is None:
        raise ValueError("scale is required")
    _on_current_device(q, kv_new, page_row, kv_cache, out, lse, workspace)
    T, H = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty((T, H, 512), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, H, 1), dtype=torch.float32, device=q.device)
    n = ctypes.c_size_t(0)
    _check("tpla_prefill_workspace_size",
           lib().tpla_prefill_workspace_size(_ref(desc(q)), ctypes.byref(n)))
    need = int(n.value)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty((need + 15) // 16 * 16, dtype=torch.uint8, device=q.device)
    rc = lib().tpla_prefill(
        _ref(desc(q)), _ref(desc(kv_new)), int(start), _ref(desc(page_row)), _ref(desc(kv_cache)),
        int(norm_groups), 1 if hadamard else 0, ctypes.c_float(eps), ctypes.c_float(scale),
        _ref(desc(out)), _ref(desc(lse)), workspace.data_ptr() if need else None,
        workspace.numel() * workspace.element_size() if need else 0, _stream(stream))
    _check("tpla_prefill", rc)
    return out, lse


def device_status(stream=None) -> int:
    v = ctypes.c_int(0)
    _check("tpla_get_device_status", lib().tpla_get_device_status(_stream(stream), ctypes.byref(v)))
    return int(v.value)


def error_string(code: int) -> str:
    return lib().tpla_error_string(int(code)).decode()


def launch_count() -> int:
    """Kernels libtpla has launched in this process so far."""
    return int(lib().tpla_launch_count())


def selftest_wait_timeout(microseconds: int = 1000, stream=None) -> None:
    """Run one bounded barrier wait that nothing completes; the device status
    then reads TPLA_ERR_DEVICE_TIMEOUT (see tpla_selftest_wait_timeout)."""
    _check("tpla_selftest_wait_timeout",
           lib().tpla_selftest_wait_timeout(int(microseconds), _stream(stream)))


def version() -> int:
    return int(lib().tpla_version())
