"""Python binding of libmla_b200.so (include/mla.h): argument marshalling only.

Every function keeps the name of the C entry point it calls. Torch is used for device
memory and streams; all arithmetic runs in the library's CUDA kernels. If the library
is missing the import fails loudly: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libmla_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "mla.h")

MLA_OK = 0
MLA_ERR_INVALID_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_CUDA = -3
MLA_ERR_WORKSPACE_TOO_SMALL = -4
MLA_ERR_DEVICE_TIMEOUT = -5
MLA_ERR_DEVICE_BAD_INPUT = -6
MLA_NOALLOC_SCRATCH_BYTES = 64 << 20
MLA_MAX_PARTS = 1024
MLA_FP8_ROW_BYTES = 656


class MlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m mla_paged_kv_06_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    sig = {
        "mla_status_string": (ctypes.c_char_p, [i32]),
        "mla_metadata_ints": (sz, [i32]),
        "mla_num_splits_len": (sz, [i32, i32, i32]),
        "mla_workspace_bytes": (sz, [i32, i32, i32, i32]),
        "mla_num_work_units": (i32, [i32, i32, i32]),
        "mla_test_set_stall": (i32, [i32, ctypes.c_ulonglong]),
        "mla_get_metadata": (i32, [vp, i32, i32, i32, i32, vp, vp, vp]),
        "mla_decode_fwd": (i32, [vp, vp, i32, vp, i32, vp, i32, i32, i32, f32, i32,
                                 vp, vp, vp, sz, vp, vp, vp]),
        "mla_decode_fwd_simt": (i32, [vp, vp, i32, vp, i32, vp, i32, i32, i32, f32, i32,
                                      vp, vp, vp, sz, vp, vp, vp]),
        "mla_decode_fwd_noalloc": (i32, [vp, vp, i32, vp, i32, vp, i32, i32, i32, f32, i32,
                                         vp, vp, vp, vp, vp]),
        "mla_decode_fwd_partial": (i32, [vp, vp, i32, vp, i32, vp, i32, i32, i32, f32, i32,
                                         vp, vp, vp, sz, vp, vp, vp]),
        "mla_decode_fwd_fp8": (i32, [vp, vp, i32, vp, i32, vp, i32, i32, i32, f32, i32,
                                     vp, vp, vp, sz, vp, vp, vp]),
        "mla_combine_partials": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp]),
        "mla_kv_append": (i32, [vp, i32, vp, i32, vp, i32, vp, i32, vp]),
        "mla_kv_append_fp8": (i32, [vp, i32, vp, i32, vp, i32, vp, i32, vp]),
        "mla_get_last_device_error": (i32, [vp, ctypes.POINTER(ctypes.c_uint32)]),
        "mla_plan_host": (i32, [vp, i32, i32, i32, i32, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def header_functions() -> list[str]:
    """Names of the functions include/mla.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def library():
    return _lib


def status_string(status: int) -> str:
    return _lib.mla_status_string(status).decode()


def _check(status: int, what: str):
    if status != MLA_OK:
        raise MlaError(status, what)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return ctypes.c_void_p(handle)


def mla_metadata_ints(num_sms: int) -> int:
    return _lib.mla_metadata_ints(num_sms)


def mla_num_splits_len(batch: int, h_q: int, s_q: int) -> int:
    return _lib.mla_num_splits_len(batch, h_q, s_q)


def mla_workspace_bytes(batch: int, h_q: int, s_q: int, num_sms: int) -> int:
    return _lib.mla_workspace_bytes(batch, h_q, s_q, num_sms)


def mla_num_work_units(num_sms: int, h_q: int = 128, s_q: int = 1) -> int:
    n = _lib.mla_num_work_units(num_sms, h_q, s_q)
    if n < 0:
        raise MlaError(n, "mla_num_work_units")
    return n


def mla_test_set_stall(stall: bool, wait_limit_ns: int = 0):
    """Test hook: make every decode kernel launched afterwards stall before its first copy
    (each wait then gives up after wait_limit_ns); stall=False restores normal decoding."""
    _check(_lib.mla_test_set_stall(1 if stall else 0, wait_limit_ns), "mla_test_set_stall")


def default_num_sms(device=None) -> int:
    return torch.cuda.get_device_properties(device or torch.cuda.current_device()).multi_processor_count


def mla_get_metadata(seqlens: torch.Tensor, h_q: int, s_q: int, num_sms: int | None = None,
                     metadata: torch.Tensor | None = None, num_splits: torch.Tensor | None = None,
                     stream=None):
    """Split-KV schedule for `seqlens` (device int32 [batch]). Returns (metadata, num_splits)."""
    assert seqlens.is_cuda and seqlens.dtype == torch.int32 and seqlens.is_contiguous()
    batch = seqlens.numel()
    num_sms = default_num_sms(seqlens.device) if num_sms is None else num_sms
    if metadata is None:
        metadata = torch.empty(mla_metadata_ints(num_sms), dtype=torch.int32, device=seqlens.device)
    if num_splits is None:
        n = mla_num_splits_len(batch, h_q, s_q)
        if n == 0:
            raise MlaError(MLA_ERR_UNSUPPORTED, "mla_num_splits_len")
        num_splits = torch.empty(n, dtype=torch.int32, device=seqlens.device)
    _check(_lib.mla_get_metadata(_ptr(seqlens), batch, h_q, s_q, num_sms, _ptr(metadata),
                                 _ptr(num_splits), _stream(stream)), "mla_get_metadata")
    return metadata, num_splits


def _decode(fn_name, q, kcache, block_table, seqlens, scale, causal, metadata, num_splits,
            workspace=None, out=None, lse=None, stream=None, num_sms=None,
            out_dtype=torch.bfloat16):
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.dim() == 4 and q.is_contiguous()
    if fn_name == "mla_decode_fwd_fp8":
        assert kcache.dtype == torch.uint8 and kcache.dim() == 3 and kcache.shape[2] == MLA_FP8_ROW_BYTES
    else:
        assert kcache.dtype == torch.bfloat16
    assert kcache.is_contiguous()
    assert block_table.dtype == torch.int32 and block_table.is_contiguous()
    batch, s_q, h_q, _ = q.shape
    num_blocks = kcache.shape[0]
    max_blocks = block_table.shape[1]
    if out is None:
        out = torch.empty((batch, s_q, h_q, 512), dtype=out_dtype, device=q.device)
    assert out.dtype == out_dtype and out.is_contiguous()
    if lse is None:
        lse = torch.empty((batch, h_q, s_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        nsm = default_num_sms(q.device) if num_sms is None else num_sms
        workspace = torch.empty(mla_workspace_bytes(batch, h_q, s_q, nsm), dtype=torch.uint8,
                                device=q.device)
    fn = getattr(_lib, fn_name)
    _check(fn(_ptr(q), _ptr(kcache), num_blocks, _ptr(block_table), max_blocks,
              _ptr(seqlens), batch, s_q, h_q, float(scale), int(bool(causal)),
              _ptr(metadata), _ptr(num_splits), _ptr(workspace), workspace.numel(),
              _ptr(out), _ptr(lse), _stream(stream)), fn_name)
    return out, lse


def mla_decode_fwd(q, kcache, block_table, seqlens, scale, causal, metadata, num_splits,
                   workspace=None, out=None, lse=None, stream=None, num_sms=None):
    """Paged MLA decode on the tensor-core kernel. Returns (out bf16 [b,s_q,h_q,512],
    lse fp32 [b,h_q,s_q])."""
    return _decode("mla_decode_fwd", q, kcache, block_table, seqlens, scale, causal, metadata,
                   num_splits, workspace, out, lse, stream, num_sms)


def mla_decode_fwd_fp8(q, kcache_fp8, block_table, seqlens, scale, causal, metadata,
                       num_splits, workspace=None, out=None, lse=None, stream=None,
                       num_sms=None):
    """Paged MLA decode over an FP8 latent cache (uint8 [num_blocks, 64, 656], the row
    format of mla_kv_append_fp8). Returns (out bf16 [b,s_q,h_q,512], lse fp32 [b,h_q,s_q])."""
    return _decode("mla_decode_fwd_fp8", q, kcache_fp8, block_table, seqlens, scale, causal,
                   metadata, num_splits, workspace, out, lse, stream, num_sms)


def mla_decode_fwd_partial(q, kcache, block_table, seqlens, scale, causal, metadata,
                           num_splits, workspace=None, out=None, lse=None, stream=None,
                           num_sms=None):
    """mla_decode_fwd with an unrounded fp32 output (the per-device partial of a split
    across devices). Returns (out fp32 [b,s_q,h_q,512], lse fp32 [b,h_q,s_q])."""
    return _decode("mla_decode_fwd_partial", q, kcache, block_table, seqlens, scale, causal,
                   metadata, num_splits, workspace, out, lse, stream, num_sms,
                   out_dtype=torch.float32)


def mla_combine_partials(o_parts, lse_parts, out=None, lse=None, stream=None):
    """Merge per-device partials: o_parts fp32 [parts, b, s_q, h_q, 512] and lse_parts
    fp32 [parts, b, h_q, s_q] -> (out bf16 [b, s_q, h_q, 512], lse fp32 [b, h_q, s_q])."""
    assert o_parts.is_cuda and o_parts.dtype == torch.float32 and o_parts.dim() == 5
    assert lse_parts.dtype == torch.float32 and lse_parts.dim() == 4
    assert o_parts.is_contiguous() and lse_parts.is_contiguous()
    parts, batch, s_q, h_q, dv = o_parts.shape
    assert dv == 512 and tuple(lse_parts.shape) == (parts, batch, h_q, s_q)
    if out is None:
        out = torch.empty((batch, s_q, h_q, 512), dtype=torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty((batch, h_q, s_q), dtype=torch.float32, device=o_parts.device)
    _check(_lib.mla_combine_partials(_ptr(o_parts), _ptr(lse_parts), parts, batch, s_q, h_q,
                                     _ptr(out), _ptr(lse), _stream(stream)),
           "mla_combine_partials")
    return out, lse


def mla_decode_fwd_simt(q, kcache, block_table, seqlens, scale, causal, metadata, num_splits,
                        workspace=None, out=None, lse=None, stream=None, num_sms=None):
    """Same as mla_decode_fwd on the CUDA-core kernel."""
    return _decode("mla_decode_fwd_simt", q, kcache, block_table, seqlens, scale, causal,
                   metadata, num_splits, workspace, out, lse, stream, num_sms)


def mla_decode_fwd_noalloc(q, kcache, block_table, seqlens, scale, causal, metadata,
                           num_splits, out=None, lse=None, stream=None):
    """mla_decode_fwd with the library's built-in scratch instead of a workspace (the C
    call allocates nothing; `out` and `lse` are created here when not given)."""
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.dim() == 4 and q.is_contiguous()
    assert kcache.dtype == torch.bfloat16 and kcache.is_contiguous()
    assert block_table.dtype == torch.int32 and block_table.is_contiguous()
    batch, s_q, h_q, _ = q.shape
    if out is None:
        out = torch.empty((batch, s_q, h_q, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((batch, h_q, s_q), dtype=torch.float32, device=q.device)
    _check(_lib.mla_decode_fwd_noalloc(
        _ptr(q), _ptr(kcache), kcache.shape[0], _ptr(block_table), block_table.shape[1],
        _ptr(seqlens), batch, s_q, h_q, float(scale), int(bool(causal)), _ptr(metadata),
        _ptr(num_splits), _ptr(out), _ptr(lse), _stream(stream)), "mla_decode_fwd_noalloc")
    return out, lse


def mla_kv_append(kv_new, block_table, seqlens, kcache, stream=None):
    """Write kv_new (bf16 [batch, s_new, 576]) at positions seqlens[b] + j of each
    sequence's pages in kcache (in place). The lengths are not advanced."""
    assert kv_new.is_cuda and kv_new.dtype == torch.bfloat16 and kv_new.dim() == 3
    assert kv_new.is_contiguous() and kcache.is_contiguous() and kcache.dtype == torch.bfloat16
    assert block_table.dtype == torch.int32 and block_table.is_contiguous()
    assert seqlens.dtype == torch.int32 and seqlens.is_contiguous()
    batch, s_new, _ = kv_new.shape
    _check(_lib.mla_kv_append(_ptr(kv_new), s_new, _ptr(block_table), block_table.shape[1],
                              _ptr(seqlens), batch, _ptr(kcache), kcache.shape[0],
                              _stream(stream)), "mla_kv_append")
    return kcache


def mla_kv_append_fp8(kv_new, block_table, seqlens, kcache_fp8, stream=None):
    """Quantize kv_new (bf16 [batch, s_new, 576]) into the FP8 cache kcache_fp8 (uint8
    [num_blocks, 64, 656]) at positions seqlens[b] + j (in place; lengths not advanced)."""
    assert kv_new.is_cuda and kv_new.dtype == torch.bfloat16 and kv_new.dim() == 3
    assert kv_new.is_contiguous() and kcache_fp8.is_contiguous()
    assert kcache_fp8.dtype == torch.uint8 and kcache_fp8.shape[1:] == (64, MLA_FP8_ROW_BYTES)
    assert block_table.dtype == torch.int32 and block_table.is_contiguous()
    assert seqlens.dtype == torch.int32 and seqlens.is_contiguous()
    batch, s_new, _ = kv_new.shape
    _check(_lib.mla_kv_append_fp8(_ptr(kv_new), s_new, _ptr(block_table), block_table.shape[1],
                                  _ptr(seqlens), batch, _ptr(kcache_fp8), kcache_fp8.shape[0],
                                  _stream(stream)), "mla_kv_append_fp8")
    return kcache_fp8


def mla_get_last_device_error(stream=None):
    """(status, raw word) of the device error word; reading clears it."""
    detail = ctypes.c_uint32(0)
    st = _lib.mla_get_last_device_error(_stream(stream), ctypes.byref(detail))
    return st, detail.value


def mla_plan_host(seqlens, h_q: int, s_q: int, num_units: int):
    """Host copy of the scheduler. Returns (metadata, num_splits) as numpy int32."""
    lens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    batch = lens.size
    n = mla_num_splits_len(batch, h_q, s_q)
    if n == 0:
        raise MlaError(MLA_ERR_UNSUPPORTED, "mla_num_splits_len")
    meta = np.zeros(8 * (num_units + 1), dtype=np.int32)
    ns = np.zeros(n, dtype=np.int32)
    _check(_lib.mla_plan_host(lens.ctypes.data, batch, h_q, s_q, num_units, meta.ctypes.data,
                              ns.ctypes.data), "mla_plan_host")
    return meta, ns
