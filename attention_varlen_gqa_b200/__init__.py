"""Python binding of ``libattn.so``, the sm_100a fused attention-forward library.

Argument marshalling only: every function below checks tensor dtypes and
devices, derives sizes from tensor shapes, allocates outputs with torch when
the caller did not pass them, and calls the C entry point of the same name
(declared in ``include/attn.h``).  All arithmetic runs in the CUDA kernels of
the library; there is no CPU path.  Importing this package fails when the
library has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python attention_varlen_gqa_b200/build.py` "
        "(the CUDA library is required; there is no fallback)")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t

EXPORTS = {
    "attn_get_config": (_I, [_P]),
    "attn_status_string": (ctypes.c_char_p, [_I]),
    "attn_varlen_fwd": (_I, [_P, _P, _P, _P, _P] + [_I] * 9 + [_F, _P, _P, _P]),
    "attn_varlen_fwd_ex": (_I, [_P, _P, _P, _P, _P] + [_I] * 9 + [_F, _F, _P, _P, _P, _P, _P]),
    "attn_paged_prefill": (_I, [_P] * 6 + [_I] * 11 + [_F, _F, _P, _P, _P, _P, _P]),
    "attn_paged_decode_workspace_size": (_S, [_I, _I, _I]),
    "attn_paged_decode": (_I, [_P] * 5 + [_I] * 7 + [_F, _F, _P, _P, _P, _S, _P]),
    "attn_paged_decode_ex": (_I, [_P] * 5 + [_I] * 7 + [_F, _F, _P, _P, _P, _P, _P, _S, _P]),
    "attn_paged_decode_static": (_I, [_P] * 5 + [_I] * 7 + [_F, _F, _P, _P, _P]),
    "attn_paged_decode_qdq_workspace_size": (_S, [_I, _I, _I, _I]),
    "attn_paged_decode_qdq": (_I, [_P] * 5 + [_I] * 7 + [_F, _F, _I, _F, _I, _F] + [_P] * 5 + [_S, _P]),
    "attn_paged_decode_workspace_size_ex": (_S, [_I, _I, _I, _I, _F]),
    "attn_smallseq_fwd": (_I, [_P] * 4 + [_I] * 5 + [_F, _P, _P, _P]),
    "attn_smallseq_bwd": (_I, [_P] * 6 + [_I] * 5 + [_F, _P, _P, _P, _P]),
    "attn_varlen_bwd_workspace_size": (_S, [_I, _I]),
    "attn_varlen_bwd": (_I, [_P] * 8 + [_I] * 9 + [_F] + [_P] * 4 + [_S, _P]),
    "attn_get_last_device_error": (_I, [_P]),
}
for _name, (_res, _args) in EXPORTS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

DEVERR = {1: "CU_SEQLENS", 2: "SEQ_LEN", 4: "BLOCK_TABLE", 8: "SMALLSEQ_LEN", 16: "TIMEOUT", 32: "BUSY"}


class AttnError(RuntimeError):
    """A negative status returned by the C library."""

    def __init__(self, fn, status):
        self.status = status
        name = lib.attn_status_string(status).decode()
        super().__init__(f"{fn} failed: {name} ({status})")


class AttnConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "prefill_block_m", "prefill_block_n", "skip_tile", "decode_splits", "decode_split_tile",
        "decode_page_size", "smallseq_max_s_kv")]


def _check(fn, rc):
    if rc != 0:
        raise AttnError(fn, rc)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t, name, dtype, dims=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dims, got {tuple(t.shape)}")


def attn_get_config():
    cfg = AttnConfig()
    _check("attn_get_config", lib.attn_get_config(ctypes.byref(cfg)))
    return {n: getattr(cfg, n) for n, _ in AttnConfig._fields_}


def attn_get_last_device_error(stream=None):
    """Synchronise ``stream`` and return (and clear) the device error bits."""
    rc = lib.attn_get_last_device_error(_stream(stream))
    if rc < 0:
        raise AttnError("attn_get_last_device_error", rc)
    return rc


def attn_varlen_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_q, max_k, causal=True, scale=None,
                    out=None, lse=None, skip_threshold=0.0, skip_mask=None, skip_counts=None,
                    want_lse=True, stream=None):
    """Packed varlen GQA forward. q [Tq, h_q, d], k/v [Tk, h_kv, d] bf16;
    cu_seqlens_* int32 [B + 1].  Returns (out, lse)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    total_q, h_q, d = q.shape
    total_k, h_kv, _ = k.shape
    batch = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((total_q, h_q), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if skip_threshold == 0.0 and skip_mask is None and skip_counts is None:
        # the plain entry point when nothing of the skip-softmax extension is asked for
        rc = lib.attn_varlen_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), batch, total_q, total_k,
            int(max_q), int(max_k), h_q, h_kv, d, int(bool(causal)), scale, _ptr(out), _ptr(lse), _stream(stream))
    else:
        rc = lib.attn_varlen_fwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), batch, total_q, total_k,
            int(max_q), int(max_k), h_q, h_kv, d, int(bool(causal)), scale, float(skip_threshold),
            _ptr(skip_mask), _ptr(skip_counts), _ptr(out), _ptr(lse), _stream(stream))
    _check("attn_varlen_fwd", rc)
    return out, lse


def attn_paged_prefill(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k, max_q, max_k,
                       causal=True, scale=None, page_size=16, out=None, lse=None, skip_threshold=0.0,
                       skip_mask=None, skip_counts=None, want_lse=True, stream=None):
    """Varlen GQA forward with K/V in a paged cache. q [Tq, h_q, d]; caches
    [pages, page_size, h_kv, d]; block_table int32 [B, max_pages];
    cu_seqlens_q int32 [B + 1]; seq_lens_k int32 [B].  Returns (out, lse)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _need(seq_lens_k, "seq_lens_k", torch.int32, 1)
    if k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape")
    total_q, h_q, d = q.shape
    num_pages, ps, h_kv, _ = k_cache.shape
    if ps != page_size:
        raise ValueError(f"cache page dimension {ps} != page_size {page_size}")
    batch = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((total_q, h_q), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib.attn_paged_prefill(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(cu_seqlens_q), _ptr(seq_lens_k),
        batch, total_q, int(max_q), int(max_k), num_pages, block_table.shape[1], page_size, h_q, h_kv, d,
        int(bool(causal)), scale, float(skip_threshold), _ptr(skip_mask), _ptr(skip_counts), _ptr(out),
        _ptr(lse), _stream(stream))
    _check("attn_paged_prefill", rc)
    return out, lse


def prefill_skip_mask_words(batch, max_q, max_k, h_q, block_m=128, skip_tile=32):
    qb = -(-max_q // block_m)
    kt = -(-max_k // skip_tile)
    return -(-(batch * qb * h_q * kt) // 32), qb, kt


def attn_varlen_bwd(q, k, v, out, dout, lse, cu_seqlens_q, cu_seqlens_k, max_q, max_k, causal=True, scale=None,
                    dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of attn_varlen_fwd from its output and log-sum-exp.  dout like
    out; returns (dq [Tq, h_q, d], dk, dv [Tk, h_kv, d])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, n, torch.bfloat16, 3)
    _need(lse, "lse", torch.float32, 2)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    total_q, h_q, d = q.shape
    total_k, h_kv, _ = k.shape
    if dq is None:
        dq = torch.empty_like(q)
    if dk is None:
        dk = torch.empty_like(k)
    if dv is None:
        dv = torch.empty_like(v)
    need = int(lib.attn_varlen_bwd_workspace_size(total_q, h_q))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib.attn_varlen_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(cu_seqlens_q),
                             _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, total_q, total_k, int(max_q), int(max_k),
                             h_q, h_kv, d, 1 if causal else 0, scale, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_varlen_bwd", rc)
    return dq, dk, dv


def attn_paged_decode_workspace_size(batch, h_q, d, max_pages_per_seq=0, skip_threshold=0.0):
    if skip_threshold > 0.0:
        return int(lib.attn_paged_decode_workspace_size_ex(batch, h_q, d, max_pages_per_seq, float(skip_threshold)))
    return int(lib.attn_paged_decode_workspace_size(batch, h_q, d))


QDQ_FORMATS = {None: 0, "none": 0, "nvfp4": 1}


def attn_paged_decode(q, k_cache, v_cache, block_table, seq_lens, page_size=16, skip_threshold=0.0,
                      scale=None, out=None, lse=None, workspace=None, skip_mask=None,
                      skip_counts=None, want_lse=True, skip_schedule="split", p_qdq=None, p_qdq_amax=1.0,
                      v_qdq=None, v_qdq_amax=1.0, stream=None):
    """One-token paged decode. q [B, h_q, d]; caches [pages, page_size, h_kv, d];
    block_table int32 [B, max_pages]; seq_lens int32 [B].  Returns (out, lse).
    skip_schedule (skip_threshold > 0, or P / V quantised): "split" -- two
    passes over the split schedule with a workspace (allocated here when not
    given); "sequential" -- one split per (sequence, kv-head), no workspace.
    p_qdq / v_qdq: None or "nvfp4" (NVFP4 quantise-dequantise of P / V before
    their product, with the operand's amax)."""
    if p_qdq not in QDQ_FORMATS or v_qdq not in QDQ_FORMATS:
        raise ValueError(f"p_qdq / v_qdq must be one of {sorted(k for k in QDQ_FORMATS if k)} or None")
    if QDQ_FORMATS[p_qdq] or QDQ_FORMATS[v_qdq]:
        return _paged_decode_qdq(q, k_cache, v_cache, block_table, seq_lens, page_size, skip_threshold, scale,
                                 out, lse, workspace, skip_mask, skip_counts, want_lse, skip_schedule,
                                 QDQ_FORMATS[p_qdq], p_qdq_amax, QDQ_FORMATS[v_qdq], v_qdq_amax, stream)
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    batch, h_q, d = q.shape
    num_pages, ps, h_kv, _ = k_cache.shape
    if ps != page_size:
        raise ValueError(f"cache page dimension {ps} != page_size {page_size}")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((batch, h_q), dtype=torch.float32, device=q.device)
    ws_bytes = 0
    if skip_threshold > 0.0 and skip_schedule == "sequential":
        workspace = None
    elif skip_schedule not in ("split", "sequential"):
        raise ValueError(f"skip_schedule must be 'split' or 'sequential', got {skip_schedule!r}")
    else:
        need = attn_paged_decode_workspace_size(batch, h_q, d, block_table.shape[1], skip_threshold)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if skip_mask is None and skip_counts is None:
        # the plain entry point when no skip reporting is asked for
        rc = lib.attn_paged_decode(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), batch, num_pages,
            block_table.shape[1], page_size, h_q, h_kv, d, float(skip_threshold), scale, _ptr(out), _ptr(lse),
            _ptr(workspace), ws_bytes, _stream(stream))
    else:
        rc = lib.attn_paged_decode_ex(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), batch, num_pages,
            block_table.shape[1], page_size, h_q, h_kv, d, float(skip_threshold), scale,
            _ptr(skip_mask), _ptr(skip_counts), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
            _stream(stream))
    _check("attn_paged_decode", rc)
    return out, lse


def _paged_decode_qdq(q, k_cache, v_cache, block_table, seq_lens, page_size, skip_threshold, scale, out, lse,
                      workspace, skip_mask, skip_counts, want_lse, skip_schedule, p_fmt, p_amax, v_fmt, v_amax,
                      stream):
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    batch, h_q, d = q.shape
    num_pages, ps, h_kv, _ = k_cache.shape
    if ps != page_size:
        raise ValueError(f"cache page dimension {ps} != page_size {page_size}")
    if skip_schedule not in ("split", "sequential"):
        raise ValueError(f"skip_schedule must be 'split' or 'sequential', got {skip_schedule!r}")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((batch, h_q), dtype=torch.float32, device=q.device)
    ws_bytes = 0
    if skip_schedule == "sequential":
        workspace = None
    else:
        need = int(lib.attn_paged_decode_qdq_workspace_size(batch, h_q, d, block_table.shape[1]))
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib.attn_paged_decode_qdq(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), batch, num_pages,
        block_table.shape[1], page_size, h_q, h_kv, d, float(skip_threshold), scale, p_fmt, float(p_amax), v_fmt,
        float(v_amax), _ptr(skip_mask), _ptr(skip_counts), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
        _stream(stream))
    _check("attn_paged_decode_qdq", rc)
    return out, lse


STATIC_WORKSPACE_BYTES = 48 << 20


def attn_paged_decode_static(q, k_cache, v_cache, block_table, seq_lens, page_size=16,
                             skip_threshold=0.0, scale=None, out=None, lse=None, want_lse=True,
                             stream=None):
    """attn_paged_decode without a workspace argument, for callers that cannot
    allocate device memory: the split partials live in the library's own
    48 MiB device scratch array, shared by every call (calls that overlap on
    the GPU race).  Output tensors may still be allocated here when not given."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    batch, h_q, d = q.shape
    num_pages, ps, h_kv, _ = k_cache.shape
    if ps != page_size:
        raise ValueError(f"cache page dimension {ps} != page_size {page_size}")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((batch, h_q), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib.attn_paged_decode_static(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), batch, num_pages,
        block_table.shape[1], page_size, h_q, h_kv, d, float(skip_threshold), scale, _ptr(out),
        _ptr(lse), _stream(stream))
    _check("attn_paged_decode_static", rc)
    return out, lse


def attn_smallseq_fwd(q, k, v, cu_seqlens_kv, max_s_kv, scale=None, out=None, weights=None,
                      want_weights=True, stream=None):
    """s_q = 1 cross attention. q [B, h, d]; k/v [Tk, h, d]; cu_seqlens_kv int32
    [B + 1].  Returns (out, weights [B, h, 1, max_s_kv])."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(cu_seqlens_kv, "cu_seqlens_kv", torch.int32, 1)
    batch, h, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if weights is None and want_weights:
        weights = torch.empty((batch, h, 1, int(max_s_kv)), dtype=torch.bfloat16, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib.attn_smallseq_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_kv), batch, k.shape[0], h,
                               d, int(max_s_kv), scale, _ptr(out), _ptr(weights), _stream(stream))
    _check("attn_smallseq_fwd", rc)
    return out, weights


def attn_smallseq_bwd(q, k, v, dout, weights, cu_seqlens_kv, max_s_kv=None, scale=None, dq=None, dk=None,
                      dv=None, stream=None):
    """Gradients of attn_smallseq_fwd from its attention weights [B, h, 1, max_s_kv].
    dout [B, h, d].  Returns (dq [B, h, d], dk, dv [Tk, h, d])."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(dout, "dout", torch.bfloat16, 3)
    _need(weights, "weights", torch.bfloat16, 4)
    _need(cu_seqlens_kv, "cu_seqlens_kv", torch.int32, 1)
    batch, h, d = q.shape
    if max_s_kv is None:
        max_s_kv = weights.shape[3]
    if dq is None:
        dq = torch.empty_like(q)
    if dk is None:
        dk = torch.empty_like(k)
    if dv is None:
        dv = torch.empty_like(v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib.attn_smallseq_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(weights), _ptr(cu_seqlens_kv),
                               batch, k.shape[0], h, d, int(max_s_kv), scale, _ptr(dq), _ptr(dk), _ptr(dv),
                               _stream(stream))
    _check("attn_smallseq_bwd", rc)
    return dq, dk, dv
