"""ctypes binding of libart (include/art.h): argument marshalling only.

Every step of the attention walk runs in the CUDA library; this module turns
torch tensors into ``art_tensor_t`` descriptors, passes the current CUDA
stream, and raises ``ArtError`` on a non-zero status.  There is no CPU
fallback: importing fails when ``libart.so`` has not been built, and calls
with tensors that are not on a CUDA device are refused.
"""
from __future__ import annotations

import ctypes
import os
import struct
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libart.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libart.so is not built ({LIB_PATH}); run `python -m kv_cache_early_art_b200.build` "
                      "or __graft_entry__.build()")

_lib = ctypes.CDLL(LIB_PATH)

F32, BF16, I32 = 0, 1, 2
_DTYPE = {torch.float32: F32, torch.bfloat16: BF16, torch.int32: I32}

STATUS = {
    0: "ART_OK", -1: "ART_ERR_NULL", -2: "ART_ERR_SHAPE", -3: "ART_ERR_DTYPE", -4: "ART_ERR_UNSUPPORTED",
    -5: "ART_ERR_PARAM", -6: "ART_ERR_LAUNCH", -7: "ART_ERR_DEVICE_TIMEOUT", -8: "ART_ERR_BAD_INDEX",
    -9: "ART_ERR_SCRATCH_SIZE",
}
ENGINE_AUTO, ENGINE_CUDA, ENGINE_MMA = 0, 1, 2


class ArtTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class ArtLaunchInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("engine", "cluster_size", "grid", "threads", "stages",
                                               "compute_warps", "window", "smem_bytes", "prefetch", "merge_cta",
                                               "ring_slots")]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


class ArtParams(ctypes.Structure):
    _fields_ = [(n, ArtTensor) for n in ("q", "k_cache", "v_cache", "page_table", "block_order", "seq_lens",
                                         "out", "stop_block")] + [
        ("eps_m", ctypes.c_float), ("eps_d", ctypes.c_float), ("P", ctypes.c_int32),
        ("min_blocks", ctypes.c_int32), ("sm_scale", ctypes.c_float),
        ("eps_m_per_seq", ctypes.c_void_p), ("eps_d_per_seq", ctypes.c_void_p),
        ("P_per_seq", ctypes.c_void_p), ("min_blocks_per_seq", ctypes.c_void_p),
        ("blocks_fetched", ctypes.c_void_p), ("device_status", ctypes.c_void_p),
        ("engine", ctypes.c_int32), ("cluster_size", ctypes.c_int32), ("stages", ctypes.c_int32),
        ("compute_warps", ctypes.c_int32), ("window", ctypes.c_int32), ("timeout_ns", ctypes.c_int64),
        ("debug_flags", ctypes.c_int32), ("info", ctypes.POINTER(ArtLaunchInfo)), ("prefetch", ctypes.c_int32),
        ("detector_off", ctypes.c_int32), ("merge_cta", ctypes.c_int32), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_int64)]


def _struct_format(cls) -> str:
    """struct-module format of a ctypes Structure, padding included, read
    from the structure's own field offsets (so it always matches art.h as the
    ctypes declaration does)."""
    codes = {ctypes.c_void_p: "Q", ctypes.c_int32: "i", ctypes.c_int64: "q", ctypes.c_float: "f"}
    parts, off = [], 0
    for name, ty in cls._fields_:
        fo = getattr(cls, name).offset
        if fo > off:
            parts.append(f"{fo - off}x")
            off = fo
        if isinstance(ty, type) and issubclass(ty, ctypes.Structure):
            parts.append(_struct_format(ty))
        elif isinstance(ty, type) and issubclass(ty, ctypes.Array):
            parts.append(f"{ty._length_}{codes[ty._type_]}")
        else:
            parts.append(codes.get(ty, "Q"))  # pointers are 8-byte addresses
        off += ctypes.sizeof(ty)
    if ctypes.sizeof(cls) > off:
        parts.append(f"{ctypes.sizeof(cls) - off}x")
    return "".join(parts)


# art_params_t packed in one call: building the nested ctypes structures field
# by field cost ~23 us of host time per call, packing them ~10 us
_PARAMS = struct.Struct("<" + _struct_format(ArtParams))
assert _PARAMS.size == ctypes.sizeof(ArtParams)


_P = ctypes.POINTER
_lib.art_decode_attention.argtypes = [_P(ArtTensor)] * 6 + [ctypes.c_float, ctypes.c_float, ctypes.c_int32,
                                                            ctypes.c_int32, _P(ArtTensor), _P(ArtTensor),
                                                            ctypes.c_void_p]
_lib.art_decode_attention.restype = ctypes.c_int
_lib.art_decode_attention_ex.argtypes = [_P(ArtParams), ctypes.c_void_p]
_lib.art_decode_attention_ex.restype = ctypes.c_int
_lib.art_decode_attention_multi.argtypes = [_P(ArtParams), ctypes.c_int32, ctypes.c_void_p]
_lib.art_decode_attention_multi.restype = ctypes.c_int
_lib.art_build_order_sink_recency.argtypes = [_P(ArtTensor), ctypes.c_int32, _P(ArtTensor), ctypes.c_void_p]
_lib.art_build_order_sink_recency.restype = ctypes.c_int
_lib.art_page_summary.argtypes = [_P(ArtTensor)] * 4 + [ctypes.c_void_p, ctypes.c_void_p]
_lib.art_page_summary.restype = ctypes.c_int
_lib.art_build_order_importance.argtypes = [_P(ArtTensor)] * 4 + [ctypes.c_int32, ctypes.c_float] + [
    _P(ArtTensor)] * 2 + [ctypes.c_void_p, ctypes.c_void_p]
_lib.art_build_order_importance.restype = ctypes.c_int
_lib.art_workspace_bytes.argtypes = [_P(ArtParams)]
_lib.art_workspace_bytes.restype = ctypes.c_int64
_lib.art_decode_attention_no_alloc.argtypes = [_P(ArtParams), ctypes.c_void_p]
_lib.art_decode_attention_no_alloc.restype = ctypes.c_int
_lib.art_strerror.argtypes = [ctypes.c_int]
_lib.art_strerror.restype = ctypes.c_char_p
_lib.art_version.argtypes = []
_lib.art_version.restype = ctypes.c_int32


class ArtError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({art_strerror(status)})")


def art_strerror(status: int) -> str:
    return _lib.art_strerror(int(status)).decode()


def art_version() -> int:
    return int(_lib.art_version())


def _tensor_fields(t):
    """The eleven art_tensor_t values of a tensor (all zero for None)."""
    if t is None:
        return (0,) * 11
    n = t.dim()
    sh, sd = tuple(t.shape), t.stride()
    if n < 4:
        pad = (0,) * (4 - n)
        sh, sd = sh + pad, sd + pad
    return (t.data_ptr() if t.numel() else 0, _DTYPE.get(t.dtype, -1), n) + sh + sd


def _addr(t):
    return t.data_ptr() if t is not None else 0


def descriptor(t: torch.Tensor) -> ArtTensor:
    """art_tensor_t over a tensor's storage (no copy)."""
    d = ArtTensor()
    d.data = t.data_ptr() if t.numel() else None
    d.dtype = _DTYPE.get(t.dtype, -1)
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libart runs on the GPU only: every tensor must be on a CUDA device")


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, device=None) -> Optional[int]:
    if stream is None:
        if _raw_stream is not None and device is not None and device.index is not None:
            return _raw_stream(device.index)  # the same handle, without building a Stream object
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str):
    if status != 0:
        raise ArtError(status, where)


def art_decode_attention(q, k_cache, v_cache, page_table, block_order, seq_lens, eps_m, eps_d, P, min_blocks,
                         out=None, stop_block=None, stream=None):
    """One ART decode-attention step (art_decode_attention in art.h).
    block_order=None walks the default order (sink block, then newest first).
    Returns (out [B,Hq,d] fp32, stop_block [B,Hkv] int32)."""
    _need_cuda(q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block)
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    if stop_block is None:
        stop_block = torch.empty(B, k_cache.shape[1], dtype=torch.int32, device=q.device)
    ds = [descriptor(t) if t is not None else None
          for t in (q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block)]
    refs = [ctypes.byref(x) if x is not None else None for x in ds]
    st = _lib.art_decode_attention(*refs[:6], float(eps_m), float(eps_d), int(P), int(min_blocks), refs[6],
                                   refs[7], _stream(stream, q.device))
    _check(st, "art_decode_attention")
    return out, stop_block


def _params(q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block, eps_m, eps_d, P, min_blocks,
            sm_scale, eps_m_per_seq, eps_d_per_seq, P_per_seq, min_blocks_per_seq, blocks_fetched, device_status,
            engine, cluster_size, stages, compute_warps, window, timeout_ns, debug_flags, prefetch, detector_off=0,
            merge_cta=0, want_info=True):
    """Fill art_params_t (argument marshalling only); returns (params, info)."""
    per = [eps_m_per_seq, eps_d_per_seq, P_per_seq, min_blocks_per_seq, blocks_fetched, device_status]
    _need_cuda(q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block, *per)
    for t, dt in zip(per, (torch.float32, torch.float32, torch.int32, torch.int32, torch.int32, torch.int32)):
        if t is not None and (t.dtype != dt or not t.is_contiguous()):
            raise ValueError(f"per-sequence/accounting arrays must be contiguous {dt}")
    p = ArtParams.from_buffer_copy(_PARAMS.pack(
        *_tensor_fields(q), *_tensor_fields(k_cache), *_tensor_fields(v_cache), *_tensor_fields(page_table),
        *_tensor_fields(block_order), *_tensor_fields(seq_lens), *_tensor_fields(out), *_tensor_fields(stop_block),
        float(eps_m), float(eps_d), int(P), int(min_blocks), float(sm_scale),
        _addr(eps_m_per_seq), _addr(eps_d_per_seq), _addr(P_per_seq), _addr(min_blocks_per_seq),
        _addr(blocks_fetched), _addr(device_status), int(engine), int(cluster_size), int(stages),
        int(compute_warps), int(window), int(timeout_ns), int(debug_flags), 0, int(prefetch), int(detector_off),
        int(merge_cta), 0, 0))
    info = None
    if want_info:
        info = ArtLaunchInfo()
        p.info = ctypes.pointer(info)
    return p, info


def art_decode_attention_ex(q, k_cache, v_cache, page_table, block_order, seq_lens, *, eps_m=0.0, eps_d=0.0,
                            P=0, min_blocks=0, sm_scale=0.0, eps_m_per_seq=None, eps_d_per_seq=None,
                            P_per_seq=None, min_blocks_per_seq=None, blocks_fetched=None, device_status=None,
                            engine=0, cluster_size=0, stages=0, compute_warps=0, window=0, timeout_ns=0,
                            debug_flags=0, prefetch=0, detector_off=0, merge_cta=0, workspace=None, out=None,
                            stop_block=None, stream=None, want_info=False):
    """art_decode_attention_ex in art.h.  Per-sequence arrays are device
    tensors of length B (float32 thresholds, int32 P / min_blocks);
    workspace a device tensor (any dtype, 256-byte aligned) or None.
    Returns (out, stop_block) or (out, stop_block, launch_info_dict)."""
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    if stop_block is None:
        stop_block = torch.empty(B, k_cache.shape[1], dtype=torch.int32, device=q.device)
    p, info = _params(q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block, eps_m, eps_d, P,
                      min_blocks, sm_scale, eps_m_per_seq, eps_d_per_seq, P_per_seq, min_blocks_per_seq,
                      blocks_fetched, device_status, engine, cluster_size, stages, compute_warps, window,
                      timeout_ns, debug_flags, prefetch, detector_off, merge_cta, want_info=want_info)
    if workspace is not None:
        _need_cuda(workspace)
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel() * workspace.element_size()
    st = _lib.art_decode_attention_ex(ctypes.byref(p), _stream(stream, q.device))
    _check(st, "art_decode_attention_ex")
    if want_info:
        return out, stop_block, info.as_dict()
    return out, stop_block


def art_decode_attention_multi(q, k_cache, v_cache, page_table, block_order, seq_lens, *, eps_m=0.0, eps_d=0.0,
                               P=0, min_blocks=0, sm_scale=0.0, eps_m_per_seq=None, eps_d_per_seq=None,
                               P_per_seq=None, min_blocks_per_seq=None, blocks_fetched=None, device_status=None,
                               engine=0, cluster_size=0, stages=0, compute_warps=0, window=0, timeout_ns=0,
                               debug_flags=0, prefetch=0, detector_off=0, merge_cta=0, out=None, stop_block=None,
                               stream=None, want_info=False):
    """art_decode_attention_multi in art.h: q [B, T, Hq, d], T query tokens
    per sequence sharing one walk.  Returns (out [B, T, Hq, d],
    stop_block [B, T, Hkv]) or those plus the launch info dict."""
    B, T, Hq, d = q.shape
    if out is None:
        out = torch.empty(B, T, Hq, d, dtype=torch.float32, device=q.device)
    if stop_block is None:
        stop_block = torch.empty(B, T, k_cache.shape[1], dtype=torch.int32, device=q.device)
    p, info = _params(q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block, eps_m, eps_d, P,
                      min_blocks, sm_scale, eps_m_per_seq, eps_d_per_seq, P_per_seq, min_blocks_per_seq,
                      blocks_fetched, device_status, engine, cluster_size, stages, compute_warps, window,
                      timeout_ns, debug_flags, prefetch, detector_off, merge_cta, want_info=want_info)
    st = _lib.art_decode_attention_multi(ctypes.byref(p), int(T), _stream(stream, q.device))
    _check(st, "art_decode_attention_multi")
    if want_info:
        return out, stop_block, info.as_dict()
    return out, stop_block


def art_workspace_bytes(q, k_cache, v_cache, page_table, block_order, seq_lens, **options):
    """art_workspace_bytes in art.h: the workspace art_decode_attention_ex can
    use for this problem (0 when its workspace walk does not apply)."""
    B, Hq, d = q.shape
    out = options.pop("out", None)
    stop_block = options.pop("stop_block", None)
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    if stop_block is None:
        stop_block = torch.empty(B, k_cache.shape[1], dtype=torch.int32, device=q.device)
    kw = dict(eps_m=0.0, eps_d=0.0, P=0, min_blocks=0, sm_scale=0.0, eps_m_per_seq=None, eps_d_per_seq=None,
              P_per_seq=None, min_blocks_per_seq=None, blocks_fetched=None, device_status=None, engine=0,
              cluster_size=0, stages=0, compute_warps=0, window=0, timeout_ns=0, debug_flags=0, prefetch=0,
              detector_off=0, merge_cta=0)
    kw.update(options)
    p, _ = _params(q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block, want_info=False, **kw)
    n = int(_lib.art_workspace_bytes(ctypes.byref(p)))
    if n < 0:
        raise ArtError(n, "art_workspace_bytes")
    return n


def art_decode_attention_no_alloc(q, k_cache, v_cache, page_table, block_order, seq_lens, *, eps_m=0.0, eps_d=0.0,
                                  P=0, min_blocks=0, sm_scale=0.0, eps_m_per_seq=None, eps_d_per_seq=None,
                                  P_per_seq=None, min_blocks_per_seq=None, blocks_fetched=None, device_status=None,
                                  engine=0, cluster_size=0, stages=0, compute_warps=0, window=0, timeout_ns=0,
                                  prefetch=0, detector_off=0, out=None, stop_block=None, stream=None,
                                  want_info=False):
    """art_decode_attention_no_alloc in art.h: the workspace walk with the
    library's own fixed scratch array, for callers that cannot allocate
    device memory (pass out and stop_block to allocate nothing here either).
    Returns (out, stop_block) or those plus the launch info dict."""
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    if stop_block is None:
        stop_block = torch.empty(B, k_cache.shape[1], dtype=torch.int32, device=q.device)
    p, info = _params(q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block, eps_m, eps_d, P,
                      min_blocks, sm_scale, eps_m_per_seq, eps_d_per_seq, P_per_seq, min_blocks_per_seq,
                      blocks_fetched, device_status, engine, cluster_size, stages, compute_warps, window,
                      timeout_ns, 0, prefetch, detector_off, 0, want_info=want_info)
    st = _lib.art_decode_attention_no_alloc(ctypes.byref(p), _stream(stream, q.device))
    _check(st, "art_decode_attention_no_alloc")
    if want_info:
        return out, stop_block, info.as_dict()
    return out, stop_block


def art_build_order_sink_recency(seq_lens, page, block_order=None, max_blocks=None, stream=None):
    """Default walk order [0, N-1, ..., 1] (-1 padded) on the device."""
    _need_cuda(seq_lens, block_order)
    if block_order is None:
        if max_blocks is None:
            raise ValueError("give block_order or max_blocks")
        block_order = torch.empty(seq_lens.shape[0], int(max_blocks), dtype=torch.int32, device=seq_lens.device)
    a, b = descriptor(seq_lens), descriptor(block_order)
    st = _lib.art_build_order_sink_recency(ctypes.byref(a), int(page), ctypes.byref(b), _stream(stream))
    _check(st, "art_build_order_sink_recency")
    return block_order


def _status_ptr(device_status):
    if device_status is None:
        return None
    _need_cuda(device_status)
    if device_status.dtype != torch.int32 or device_status.numel() < 1:
        raise ValueError("device_status must be an int32 device tensor")
    return device_status.data_ptr()


def art_page_summary(k_cache, page_table, seq_lens, summary=None, *, dtype=torch.float32, device_status=None,
                     stream=None):
    """Mean key of every referenced page, per kv-head (art_page_summary in
    art.h).  Returns summary [num_pages, Hkv, d] (float32 or bfloat16)."""
    _need_cuda(k_cache, page_table, seq_lens, summary)
    if summary is None:
        NP, Hkv, _, d = k_cache.shape
        summary = torch.zeros(NP, Hkv, d, dtype=dtype, device=k_cache.device)
    ds = [descriptor(t) for t in (k_cache, page_table, seq_lens, summary)]
    st = _lib.art_page_summary(*[ctypes.byref(x) for x in ds], _status_ptr(device_status), _stream(stream))
    _check(st, "art_page_summary")
    return summary


def art_build_order_importance(q, summary, page_table, seq_lens, page, *, sm_scale=0.0, block_scores=None,
                               block_order=None, device_status=None, stream=None):
    """Importance-first walk order (art_build_order_importance in art.h).
    Returns (block_order [B, max_blocks] int32, block_scores [B, max_blocks] float32)."""
    _need_cuda(q, summary, page_table, seq_lens, block_scores, block_order)
    B, mb = page_table.shape
    if block_scores is None:
        block_scores = torch.empty(B, mb, dtype=torch.float32, device=q.device)
    if block_order is None:
        block_order = torch.empty(B, mb, dtype=torch.int32, device=q.device)
    ds = [descriptor(t) for t in (q, summary, page_table, seq_lens, block_scores, block_order)]
    r = [ctypes.byref(x) for x in ds]
    st = _lib.art_build_order_importance(*r[:4], int(page), float(sm_scale), r[4], r[5],
                                         _status_ptr(device_status), _stream(stream))
    _check(st, "art_build_order_importance")
    return block_order, block_scores


def raw_library():
    """The loaded ctypes library (for ABI tests)."""
    return _lib
