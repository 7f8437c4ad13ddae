"""ctypes binding of libic_b200.so (include/ic.h), one Python function per C entry point.

Argument marshalling only: shapes are read off the torch tensors, pointers and
the current CUDA stream are handed to the library, and a non-zero status
raises ``ICError``.  Every step of the path runs in the library's kernels;
there is no fallback of any kind: if the library is missing the first call
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# IC_DEBUG_BOUNDS=1 in the environment selects the debug-bounds build of the same
# library (device-side index checks reported as IC_ERR_BOUNDS; see ic.h)
LIB_PATH = os.path.join(_PKG, "libic_b200_debug.so" if os.environ.get("IC_DEBUG_BOUNDS") == "1"
                        else "libic_b200.so")

IC_OK = 0
IC_ERR_INVALID_ARG = -1
IC_ERR_UNSUPPORTED = -2
IC_ERR_WORKSPACE = -3
IC_ERR_CUDA = -4
IC_ERR_TIMEOUT = -5
IC_ERR_BOUNDS = -6
IC_F32, IC_BF16, IC_E4M3 = 0, 1, 2

# names declared in include/ic.h (checked against the header by the tests)
EXPORTS = ("ic_last_error", "ic_version", "ic_device_status", "ic_trace_begin", "ic_trace_end",
           "ic_quant_e4m3_rows", "ic_pack_kv_e4m3",
           "ic_indexer_scores", "ic_indexer_topk", "ic_indexer_topk_workspace_size", "ic_topk",
           "ic_topk_varlen", "ic_sparse_attn",
           "ic_attn_workspace_size",
           "ic_layer_stack", "ic_decode_step", "ic_stack_workspace_size",
           "ic_sparse_attn_noalloc", "ic_layer_stack_rows", "ic_layer_stack_varlen")


class ICError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("ic status %d: %s" % (status, msg))
        self.status = status


class ic_layer_io(ctypes.Structure):
    _fields_ = [("q_idx", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("k_idx", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("q", ctypes.c_void_p), ("kv", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p)]


class ic_stack_desc(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int), ("batch", ctypes.c_int), ("decode", ctypes.c_int),
                ("k", ctypes.c_int), ("idx_dtype", ctypes.c_int), ("H", ctypes.c_int),
                ("D", ctypes.c_int), ("attn_dtype", ctypes.c_int), ("heads", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("ld_kv", ctypes.c_long),
                ("scale", ctypes.c_float), ("flags", ctypes.c_int)]


IC_STACK_FUSED_TOPK = 1


_lib = None


def lib() -> ctypes.CDLL:
    """Opens libic_b200.so (built in-tree by ``build.py``); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libic_b200.so is not built (%s); run "
                           "`python -m sparse_attention_indexer_sum_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P, I, Lg, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_float, ctypes.c_size_t
    L.ic_last_error.restype = ctypes.c_char_p
    L.ic_last_error.argtypes = []
    L.ic_version.restype = I
    L.ic_device_status.argtypes = [P]
    L.ic_trace_begin.argtypes = [P, I]
    L.ic_trace_begin.restype = I
    L.ic_trace_end.argtypes = [P, P, P, I]
    L.ic_trace_end.restype = Lg
    L.ic_quant_e4m3_rows.argtypes = [P, I, Lg, I, P, P, P]
    L.ic_pack_kv_e4m3.argtypes = [P, Lg, Lg, P, Lg, P]
    L.ic_indexer_scores.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Lg, P, Lg, P]
    L.ic_indexer_topk.argtypes = [P, P, P, P, P, I, I, I, I, I, Lg, I, P, P, S, P]
    L.ic_indexer_topk_workspace_size.argtypes = [I, I, Lg]
    L.ic_indexer_topk_workspace_size.restype = S
    L.ic_topk.argtypes = [P, Lg, I, Lg, Lg, I, P, P]
    L.ic_topk_varlen.argtypes = [P, Lg, I, Lg, P, I, P, P]
    L.ic_sparse_attn.argtypes = [P, P, Lg, P, P, I, I, I, I, I, I, I, I, F, P, P, P, S, P]
    L.ic_attn_workspace_size.argtypes = [I, I, I, I, I]
    L.ic_attn_workspace_size.restype = S
    L.ic_layer_stack.argtypes = [ctypes.c_char_p, ctypes.POINTER(ic_stack_desc),
                                 ctypes.POINTER(ic_layer_io), I, P, P, S, P]
    L.ic_decode_step.argtypes = L.ic_layer_stack.argtypes
    L.ic_layer_stack_rows.argtypes = [ctypes.c_char_p, ctypes.POINTER(ic_stack_desc),
                                      ctypes.POINTER(ic_layer_io), I, Lg, Lg, P, P, S, P]
    L.ic_layer_stack_varlen.argtypes = [ctypes.c_char_p, ctypes.POINTER(ic_stack_desc),
                                        ctypes.POINTER(ic_layer_io), I, ctypes.POINTER(Lg), I, P,
                                        P, S, P]
    L.ic_stack_workspace_size.argtypes = [ctypes.POINTER(ic_stack_desc)]
    L.ic_stack_workspace_size.restype = S
    L.ic_sparse_attn_noalloc.argtypes = [P, P, Lg, P, P, I, I, I, I, I, I, I, I, F, P, P, P]
    for name in ("ic_device_status", "ic_quant_e4m3_rows", "ic_pack_kv_e4m3", "ic_indexer_scores",
                 "ic_topk",
                 "ic_topk_varlen", "ic_indexer_topk",
                 "ic_sparse_attn", "ic_layer_stack", "ic_decode_step", "ic_sparse_attn_noalloc",
                 "ic_layer_stack_rows", "ic_layer_stack_varlen"):
        getattr(L, name).restype = I
    _lib = L
    return L


def ic_last_error() -> str:
    return lib().ic_last_error().decode()


def ic_version() -> int:
    return int(lib().ic_version())


def _check(st: int):
    if st != IC_OK:
        raise ICError(st, ic_last_error())


def _p(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return IC_F32
    if t.dtype == torch.bfloat16:
        return IC_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return IC_E4M3
    raise ValueError("unsupported dtype %s" % t.dtype)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def ic_device_status(stream=None):
    """Synchronises the stream; raises ICError(IC_ERR_TIMEOUT) if a device wait gave up
    (IC_ERR_BOUNDS if a debug-bounds check failed)."""
    _check(lib().ic_device_status(_stream(stream)))


KIND_NAMES = {1: "indexer_tc_bf16", 2: "indexer_tc_e4m3", 3: "indexer_f32", 4: "fill_masked",
              5: "topk", 6: "attn_mla", 7: "attn_combine", 8: "attn_f32", 9: "quant_e4m3",
              10: "topk_merge", 11: "indexer_topk_bf16", 12: "indexer_topk_e4m3",
              13: "attn_mla_kv8", 14: "pack_kv_e4m3", 15: "fill_valid"}


def ic_trace_begin(capacity: int = 4096, stream=None):
    """Starts per-launch event tracing on this thread (see ic.h)."""
    _check(lib().ic_trace_begin(_stream(stream), int(capacity)))
    return int(capacity)


def ic_trace_end(capacity: int = 4096):
    """Stops tracing; returns (launches, [(kind_name, ms, work), ...])."""
    import numpy as np
    ms = np.zeros(capacity, np.float32)
    kinds = np.zeros(capacity, np.int32)
    work = np.zeros(capacity, np.float64)
    n = lib().ic_trace_end(ms.ctypes.data_as(ctypes.c_void_p), kinds.ctypes.data_as(ctypes.c_void_p),
                           work.ctypes.data_as(ctypes.c_void_p), int(capacity))
    if n < 0:
        raise ICError(int(n), ic_last_error())
    m = min(int(n), capacity)
    return int(n), [(KIND_NAMES.get(int(kinds[i]), str(kinds[i])), float(ms[i]), float(work[i]))
                    for i in range(m)]


def ic_quant_e4m3_rows(x: torch.Tensor, codes=None, scales=None, stream=None):
    """Per-row e4m3 codes (uint8) and fp32 scales of x[..., n]."""
    _contig(x)
    n = x.shape[-1]
    rows = x.numel() // n
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _check(lib().ic_quant_e4m3_rows(_p(x), dtype_code(x), rows, n, _p(codes), _p(scales),
                                    _stream(stream)))
    return codes, scales


KV8_ROW_BYTES = 656


def ic_pack_kv_e4m3(kv: torch.Tensor, out=None, stream=None):
    """fp8 latent-KV cache rows [..., 656] uint8 of bf16 latent rows kv [..., 576]
    (512 e4m3 codes in four 128-dim groups, 4 fp32 group scales, 64 bf16 rope dims)."""
    if kv.dtype != torch.bfloat16 or kv.shape[-1] != 576 or kv.stride(-1) != 1:
        raise ValueError("kv must be bf16 [..., 576] with contiguous rows")
    rows = kv.numel() // 576
    if out is None:
        out = torch.empty(kv.shape[:-1] + (KV8_ROW_BYTES,), dtype=torch.uint8, device=kv.device)
    _contig(kv, out)
    _check(lib().ic_pack_kv_e4m3(_p(kv), rows, 576, _p(out), out.shape[-1], _stream(stream)))
    return out


def ic_indexer_scores(q, k, w, scores=None, *, pos0: int = 0, q_scale=None, k_scale=None,
                      stream=None):
    """Indexer scores [B, R, Lk] (or [R, Lk] without a batch axis) of q [B?,R,H,D],
    k [B?,Lk,D], w [B?,R,H]; e4m3 inputs (uint8 codes) take q_scale [B?,R,H], k_scale [B?,Lk]."""
    _contig(q, k, w, q_scale, k_scale)
    squeeze = q.dim() == 3
    B = 1 if squeeze else q.shape[0]
    R, H, D = q.shape[-3:]
    Lk = k.shape[-2]
    if scores is None:
        shape = (R, Lk) if squeeze else (B, R, Lk)
        scores = torch.empty(shape, dtype=torch.float32, device=q.device)
    ld = scores.stride(-2)
    _check(lib().ic_indexer_scores(_p(q), _p(q_scale), _p(k), _p(k_scale), _p(w), dtype_code(q),
                                   B, H, D, R, Lk, int(pos0), _p(scores), ld, _stream(stream)))
    return scores


def ic_indexer_topk_workspace_size(batch: int, Lk: int, pos0: int) -> int:
    return int(lib().ic_indexer_topk_workspace_size(int(batch), int(Lk), int(pos0)))


def ic_indexer_topk(q, k, w, k_top: int, workspace, *, pos0: int, q_scale=None, k_scale=None,
                    idx=None, stream=None):
    """Indexer and top-k in one pass for one query per sequence: q [B,1,H,D],
    k [B,Lk,D], w [B,1,H] (e4m3 codes take q_scale [B,1,H], k_scale [B,Lk]); returns
    idx [B, k_top] int32.  The scores are never written."""
    _contig(q, k, w, q_scale, k_scale)
    if q.dim() != 4 or q.shape[1] != 1:
        raise ValueError("q must be [B, 1, H, D]")
    B, _, H, D = q.shape
    Lk = k.shape[-2]
    if idx is None:
        idx = torch.empty((B, k_top), dtype=torch.int32, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().ic_indexer_topk(_p(q), _p(q_scale), _p(k), _p(k_scale), _p(w), dtype_code(q), B,
                                 H, D, Lk, int(pos0), int(k_top), _p(idx), _p(workspace),
                                 ws_bytes, _stream(stream)))
    return idx


def ic_topk(scores, k: int, *, n: int | None = None, pos0: int = -1, idx=None, stream=None):
    """Exact top-k indices [rows, k] (int32, ascending, -1 padded) of scores [rows, ld].
    pos0 >= 0 makes the rows causal: row r keeps columns s <= pos0 + r."""
    rows = scores.shape[0]
    n = scores.shape[1] if n is None else n
    if scores.stride(1) != 1:
        raise ValueError("scores rows must be contiguous")
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    _check(lib().ic_topk(_p(scores), rows, n, scores.stride(0), int(pos0), int(k), _p(idx),
                         _stream(stream)))
    return idx


def ic_topk_varlen(scores, k: int, valid_len, *, n: int | None = None, idx=None, stream=None):
    """Exact top-k indices [rows, k] of scores [rows, ld] with row r's candidates the
    columns s < valid_len[r] (device int32 [rows])."""
    rows = scores.shape[0]
    n = scores.shape[1] if n is None else n
    if scores.stride(1) != 1:
        raise ValueError("scores rows must be contiguous")
    if valid_len.dtype != torch.int32 or valid_len.numel() != rows:
        raise ValueError("valid_len must be int32 [rows]")
    _contig(valid_len)
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    _check(lib().ic_topk_varlen(_p(scores), rows, n, scores.stride(0), _p(valid_len), int(k),
                                _p(idx), _stream(stream)))
    return idx


def ic_attn_workspace_size(batch: int, rows: int, heads: int, dv: int, k: int) -> int:
    return int(lib().ic_attn_workspace_size(batch, rows, heads, dv, k))


def ic_sparse_attn(q, kv, idx, scale: float, *, v=None, dv: int | None = None, out=None, lse=None,
                   workspace=None, stream=None):
    """Sparse attention.  q [B?,R,heads,dk]; kv [B?,Lkv,ld_kv]; idx [B?,R,k];
    v [B?,Lkv,dv] for the MQA form (fp32), else absorbed MLA over kv[..., :dv]: a bf16
    cache, or an fp8 cache (uint8 rows of ic_pack_kv_e4m3) with q and out bf16."""
    _contig(q, idx, v)
    if kv.stride(-1) != 1:
        raise ValueError("kv rows must be contiguous")
    squeeze = q.dim() == 3
    B = 1 if squeeze else q.shape[0]
    R, heads, dk = q.shape[-3:]
    Lkv = kv.shape[-2]
    kk = idx.shape[-1]
    if v is not None:
        dv = v.shape[-1]
    elif dv is None:
        dv = 512
    if out is None:
        out = torch.empty(q.shape[:-1] + (dv,), dtype=q.dtype, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    dt = IC_E4M3 if (v is None and kv.dtype == torch.uint8) else dtype_code(q)
    _check(lib().ic_sparse_attn(_p(q), _p(kv), kv.stride(-2), _p(v), _p(idx), dt, B, R,
                                heads, dk, dv, Lkv, kk, float(scale), _p(out), _p(lse),
                                _p(workspace), ws_bytes, _stream(stream)))
    return out


def ic_sparse_attn_noalloc(q, kv, idx, scale: float, *, out, dv: int = 512, lse=None,
                           stream=None):
    """Absorbed-MLA sparse attention whose split scratch is the library's fixed device
    array rather than a workspace (for callers that cannot allocate; at most
    IC_NOALLOC_MAX_QUERIES = 64 queries).  q [B?,R,16,576] bf16; kv [B?,Lkv,ld_kv];
    idx [B?,R,k] int32.  The caller passes ``out`` [B?,R,16,dv] bf16 (and, if wanted,
    ``lse`` [B?,R,16] f32), both contiguous: this wrapper allocates nothing either.
    Calls that overlap on the GPU race on the shared array."""
    _contig(q, idx, out, lse)
    if kv.stride(-1) != 1:
        raise ValueError("kv rows must be contiguous")
    squeeze = q.dim() == 3
    B = 1 if squeeze else q.shape[0]
    R, heads, dk = q.shape[-3:]
    if idx.dtype != torch.int32 or tuple(idx.shape[:-1]) != tuple(q.shape[:-2]):
        raise ValueError("idx must be int32 [B?, R, k] matching q")
    if out is None or out.dtype != q.dtype or tuple(out.shape) != tuple(q.shape[:-1]) + (dv,):
        raise ValueError("out must be a %s tensor of shape %s" % (
            q.dtype, tuple(q.shape[:-1]) + (dv,)))
    if lse is not None and (lse.dtype != torch.float32 or
                            tuple(lse.shape) != tuple(q.shape[:-1])):
        raise ValueError("lse must be a float32 tensor of shape %s" % (tuple(q.shape[:-1]),))
    _check(lib().ic_sparse_attn_noalloc(_p(q), _p(kv), kv.stride(-2), None, _p(idx),
                                        dtype_code(q), B, R, heads, dk, dv, kv.shape[-2],
                                        idx.shape[-1], float(scale), _p(out), _p(lse),
                                        _stream(stream)))
    return out


def make_desc(*, L, k, H, D, idx_dtype, heads, dk, dv, attn_dtype, scale, ld_kv=None, batch=1,
              decode=False, flags=0) -> ic_stack_desc:
    return ic_stack_desc(L=L, batch=batch, decode=int(bool(decode)), k=k, idx_dtype=idx_dtype, H=H,
                         D=D, attn_dtype=attn_dtype, heads=heads, dk=dk, dv=dv,
                         ld_kv=dk if ld_kv is None else ld_kv, scale=scale, flags=flags)


def ic_stack_workspace_size(desc: ic_stack_desc) -> int:
    return int(lib().ic_stack_workspace_size(ctypes.byref(desc)))


def _layers(layers):
    arr = (ic_layer_io * len(layers))()
    for i, d in enumerate(layers):
        arr[i] = ic_layer_io(*[(d.get(f).data_ptr() if d.get(f) is not None else None)
                               for f, _ in ic_layer_io._fields_])
    return arr


def ic_layer_stack(pattern: str, desc: ic_stack_desc, layers: list[dict], t_cache, workspace,
                   stream=None):
    """Prefill layer stack; layers are dicts with the ic_layer_io field names."""
    arr = _layers(layers)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().ic_layer_stack(pattern.encode(), ctypes.byref(desc), arr, len(layers),
                                _p(t_cache), _p(workspace), ws_bytes, _stream(stream)))


def ic_layer_stack_rows(pattern: str, desc: ic_stack_desc, layers: list[dict], row0: int,
                        rows: int, t_cache, workspace, stream=None):
    """Prefill stack for query rows [row0, row0 + rows) of the desc.L-token sequence.
    Row-indexed layer tensors (q_idx, q_scale, w, q, out, lse) and t_cache hold just
    those rows; k_idx, k_scale and kv hold all desc.L keys."""
    arr = _layers(layers)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().ic_layer_stack_rows(pattern.encode(), ctypes.byref(desc), arr, len(layers),
                                     int(row0), int(rows), _p(t_cache), _p(workspace), ws_bytes,
                                     _stream(stream)))


def ic_layer_stack_varlen(pattern: str, desc: ic_stack_desc, layers: list[dict], cu_seqlens,
                          t_cache, workspace, stream=None):
    """Prefill stack over sequences packed along the row axis; cu_seqlens = [0, L_0,
    L_0 + L_1, ...] (host ints).  Every layer tensor holds the packed rows."""
    cu = (ctypes.c_long * len(cu_seqlens))(*[int(x) for x in cu_seqlens])
    arr = _layers(layers)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().ic_layer_stack_varlen(pattern.encode(), ctypes.byref(desc), arr, len(layers), cu,
                                       len(cu_seqlens) - 1, _p(t_cache), _p(workspace), ws_bytes,
                                       _stream(stream)))


def ic_decode_step(pattern: str, desc: ic_stack_desc, layers: list[dict], t_cache, workspace,
                   stream=None):
    """Decode step over the layer stack (desc.decode = 1)."""
    arr = _layers(layers)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().ic_decode_step(pattern.encode(), ctypes.byref(desc), arr, len(layers),
                                _p(t_cache), _p(workspace), ws_bytes, _stream(stream)))


def decode_step_graph(pattern: str, desc: ic_stack_desc, layers: list[dict], t_cache, workspace,
                      warmup: int = 1) -> torch.cuda.CUDAGraph:
    """One ic_decode_step captured into a CUDA graph over these buffers.

    ``graph.replay()`` reruns the whole step (its kernels and the programmatic
    launch edges between them) with one launch from the host, on the current
    stream.  Every replay reads the same input tensors and writes the same
    outputs: a caller updates the inputs in place between replays.  The step
    allocates nothing, so the graph holds no memory of its own."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warmup):  # first-call set-up (kernel attributes) outside the capture
            ic_decode_step(pattern, desc, layers, t_cache, workspace, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    # relaxed: the step's per-launch host calls (kernel attributes, device queries)
    # are not stream work and need not be refused while capturing
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        ic_decode_step(pattern, desc, layers, t_cache, workspace)
    return graph
