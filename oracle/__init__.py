"""CPU oracle for the IndexCache / DeepSeek Sparse Attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library never does, and this package imports nothing from
the product package: the two share only the seeded input generators, which hold
none of the method's arithmetic.

The arithmetic lives in ``ic_oracle.c`` (fp64, written out from the pages'
definitions); this module builds it with gcc, marshals numpy arrays, and holds
the layer loop of the routing pseudocode in "IndexCache: Wie DeepSeek
O(NL^2)-Kosten in Sparse Attention um 75% reduziert" (section "Einfache
Implementierung, enorme Effizienzgewinne"), which is plain control flow.

Every function here is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ic_oracle.c")
_LIB = os.path.join(_HERE, "libic_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ic_oracle.c with gcc (plain -O2, IEEE arithmetic, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            L = ctypes.c_long
            lib.ico_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.ico_e4m3_decode.restype = ctypes.c_double
            lib.ico_e4m3_encode.argtypes = [ctypes.c_double]
            lib.ico_e4m3_encode.restype = ctypes.c_uint8
            lib.ico_quant_rows_e4m3.argtypes = [P, L, I, P, P]
            lib.ico_indexer_scores.argtypes = [P, P, P, I, I, I, I, I, L, P, I, P, I]
            lib.ico_topk.argtypes = [P, L, I, L, P, I, P, I]
            lib.ico_sparse_attn.argtypes = [P, P, L, P, L, P, I, I, I, I, I, I, I,
                                            ctypes.c_double, P, P, I]
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


# ----------------------------------------------------------------------------- e4m3
def e4m3_decode(code: int) -> float:
    """Value of one OCP E4M3 code (bias 7, no infinities, S.1111.111 = NaN)."""
    return float(_load().ico_e4m3_decode(int(code) & 0xFF))


def e4m3_encode(x: float) -> int:
    """Nearest E4M3 code, ties to even, saturating at +-448."""
    return int(_load().ico_e4m3_encode(float(x)))


def e4m3_decode_array(codes: np.ndarray) -> np.ndarray:
    table = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def quant_rows_e4m3(x: np.ndarray):
    """Per-row e4m3 quantisation of x[..., n] (fp32): returns (codes uint8, scales f32).

    scale = amax/448 (1 for an all-zero row), code = E4M3(x / scale), both in fp32.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    n = x.shape[-1]
    rows = x.size // n if n else 0
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros(x.shape[:-1], dtype=np.float32)
    _load().ico_quant_rows_e4m3(_p(x), rows, n, _p(codes), _p(scales))
    return codes, scales


def dequant_rows_e4m3(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """codes [..., n] with scales [...] -> fp64 values code_value * scale."""
    return e4m3_decode_array(codes) * np.asarray(scales, dtype=np.float64)[..., None]


# ----------------------------------------------------------------------------- indexer
def indexer_scores(q, k, w, pos0: int = 0, rows_sel=None, nthreads: int | None = None):
    """Lightning-indexer scores in fp64.

    q [B, R, H, D], k [B, Lk, D], w [B, R, H] (a missing leading batch axis is
    added).  Returns I [B, nsel, Lk] (fp64) with
    I[b, j, s] = sum_h w[b, r, h] * max(0, q[b, r, h, :] . k[b, s, :]) for
    s <= pos0 + r (r = rows_sel[j], or j) and -inf for s > pos0 + r.
    """
    q, k, w = _f64(q), _f64(k), _f64(w)
    squeeze = q.ndim == 3
    if squeeze:
        q, k, w = q[None], k[None], w[None]
    B, R, H, D = q.shape
    Lk = k.shape[1]
    assert k.shape == (B, Lk, D) and w.shape == (B, R, H)
    assert np.isfinite(q).all() and np.isfinite(k).all() and np.isfinite(w).all()
    sel = None
    nsel = R
    if rows_sel is not None:
        sel = np.ascontiguousarray(np.asarray(rows_sel, dtype=np.int32))
        assert sel.ndim == 1 and (sel >= 0).all() and (sel < R).all()
        nsel = int(sel.size)
    out = np.empty((B, nsel, Lk), dtype=np.float64)
    _load().ico_indexer_scores(_p(q), _p(k), _p(w), B, R, H, D, Lk, int(pos0),
                               _p(sel) if sel is not None else None, nsel, _p(out),
                               nthreads or default_threads())
    return out[0] if squeeze else out


def indexer_scores_at(q_rows, k, w_rows, positions, nthreads: int | None = None):
    """Indexer scores of a few query rows at arbitrary positions (no batch axis).

    q_rows [n, H, D], w_rows [n, H], positions [n]; k [Lk, D].  Row j is scored at
    position positions[j] (keys s <= positions[j]).  One call of the same routine per
    row, spread over a thread pool (the C routine releases the GIL).
    Returns [n, Lk] fp64.
    """
    from concurrent.futures import ThreadPoolExecutor
    q_rows, k, w_rows = _f64(q_rows), _f64(k), _f64(w_rows)
    pos = [int(p) for p in positions]
    out = np.empty((len(pos), k.shape[0]), dtype=np.float64)

    def one(j):
        out[j] = indexer_scores(q_rows[j:j + 1], k, w_rows[j:j + 1], pos0=pos[j], nthreads=1)[0]

    with ThreadPoolExecutor(max_workers=nthreads or default_threads()) as ex:
        list(ex.map(one, range(len(pos))))
    return out


def indexer_scores_e4m3(q_codes, q_scale, k_codes, k_scale, w, pos0: int = 0, rows_sel=None,
                        nthreads: int | None = None):
    """The indexer on per-row e4m3 inputs: the same definition on the dequantised values
    q = code(q) * q_scale[token, head], k = code(k) * k_scale[token]."""
    q = dequant_rows_e4m3(q_codes, q_scale)
    k = dequant_rows_e4m3(k_codes, k_scale)
    return indexer_scores(q, k, w, pos0=pos0, rows_sel=rows_sel, nthreads=nthreads)


# ----------------------------------------------------------------------------- top-k
def topk(scores, k: int, valid=None, nthreads: int | None = None) -> np.ndarray:
    """Exact per-row top-k over fp32 scores [rows, n].

    Returns int32 [rows, k]: the min(k, valid[r]) indices s < valid[r] with the
    largest scores (ties to the lower index, -0 == +0), in ascending index
    order, padded with -1.
    """
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float32))
    squeeze = s.ndim == 1
    if squeeze:
        s = s[None]
    rows, n = s.shape
    v = None
    if valid is not None:
        v = np.ascontiguousarray(np.broadcast_to(np.asarray(valid, dtype=np.int32), (rows,)))
        assert (v >= 0).all() and (v <= n).all()
    lim = v if v is not None else np.full(rows, n)
    for r in range(rows):
        assert np.isfinite(s[r, :lim[r]]).all(), "the oracle supports finite scores only"
    out = np.empty((rows, k), dtype=np.int32)
    _load().ico_topk(_p(s), rows, n, n, _p(v) if v is not None else None, int(k), _p(out),
                     nthreads or default_threads())
    return out[0] if squeeze else out


def causal_valid(rows: int, pos0: int, n: int) -> np.ndarray:
    """Number of candidate keys of query rows 0..rows-1 at positions pos0 + r."""
    return np.minimum(np.arange(rows, dtype=np.int64) + pos0 + 1, n).astype(np.int32)


# ----------------------------------------------------------------------------- attention
def sparse_attn(q, kv, idx, scale: float, dv: int | None = None, v=None,
                nthreads: int | None = None):
    """Sparse attention of every query row over its index set, fp64.

    q [B, R, Hq, Dk]; kv [B, Lkv, >=Dk]; idx [B, R, k] (entries < 0 skipped).
    MLA absorbed form (v is None): values are kv[..., :dv] of the same latent rows.
    MQA form: separate v [B, Lkv, Dv].  Returns (out [B, R, Hq, Dv], lse [B, R, Hq]).
    """
    q = _f64(q)
    kv = _f64(kv)
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    squeeze = q.ndim == 3
    if squeeze:
        q, kv, idx = q[None], kv[None], idx[None]
        if v is not None:
            v = _f64(v)[None]
    elif v is not None:
        v = _f64(v)
    B, R, Hq, Dk = q.shape
    Lkv, ld_kv = kv.shape[1], kv.shape[2]
    assert ld_kv >= Dk
    kk = idx.shape[2]
    assert idx.shape == (B, R, kk)
    assert (idx < Lkv).all()
    if v is None:
        Dv = int(dv if dv is not None else Dk)
        assert Dv <= ld_kv
        ld_v = 0
    else:
        Dv = v.shape[2]
        ld_v = v.shape[2]
        assert v.shape[:2] == (B, Lkv)
    out = np.empty((B, R, Hq, Dv), dtype=np.float64)
    lse = np.empty((B, R, Hq), dtype=np.float64)
    _load().ico_sparse_attn(_p(q), _p(kv), ld_kv, _p(v) if v is not None else None, ld_v,
                            _p(idx), B, R, Hq, Dk, Dv, kk, Lkv, float(scale), _p(out), _p(lse),
                            nthreads or default_threads())
    if squeeze:
        return out[0], lse[0]
    return out, lse


# ----------------------------------------------------------------------------- fp8 latent KV
KV_GROUP = 128     # latent dims per e4m3 scale group
KV_LATENT = 512    # e4m3 latent dims of a 576-d row; the other 64 (rope) stay bf16


def kv_pack_e4m3(kv):
    """The fp8 latent-KV cache of bf16-valued rows kv [..., 576] (float arrays).

    The 512 latent dims are quantised in four groups of 128 with the per-row
    quantiser (scale = amax / 448 per group, code = E4M3(x / scale)); the 64
    rope dims are kept as they are.  Returns (codes uint8 [..., 512],
    scales f32 [..., 4], rope f32 [..., 64])."""
    kv = np.asarray(kv, dtype=np.float32)
    assert kv.shape[-1] == KV_LATENT + 64
    lead = kv.shape[:-1]
    lat = np.ascontiguousarray(kv[..., :KV_LATENT]).reshape(lead + (KV_LATENT // KV_GROUP, KV_GROUP))
    codes, scales = quant_rows_e4m3(lat)
    return codes.reshape(lead + (KV_LATENT,)), scales, np.ascontiguousarray(kv[..., KV_LATENT:])


def kv_dequant_e4m3(codes, scales, rope):
    """fp64 rows [..., 576] of an fp8 latent-KV cache: code value * its group's scale
    for the 512 latent dims, then the 64 rope dims."""
    codes = np.asarray(codes, dtype=np.uint8)
    lead = codes.shape[:-1]
    g = codes.reshape(lead + (KV_LATENT // KV_GROUP, KV_GROUP))
    lat = dequant_rows_e4m3(g, scales).reshape(lead + (KV_LATENT,))
    return np.concatenate([lat, np.asarray(rope, dtype=np.float64)], axis=-1)


def sparse_attn_kv_e4m3(q, codes, scales, rope, idx, scale: float, nthreads: int | None = None):
    """Absorbed-MLA sparse attention over an fp8 latent-KV cache: the same definition
    as sparse_attn on the dequantised rows (values = their first 512 dims)."""
    kv = kv_dequant_e4m3(codes, scales, rope)
    return sparse_attn(q, kv, idx, scale, dv=KV_LATENT, nthreads=nthreads)


# ----------------------------------------------------------------------------- F/S stack
def parse_pattern(pattern: str) -> list[str]:
    """Layer types from a pattern string such as "F,S,S,S" or "F S S S" or "FSSS".

    The first layer must be F, since only an F layer fills the index cache that
    later S layers read ("IndexCache: Wie DeepSeek O(NL^2)-Kosten in Sparse
    Attention um 75% reduziert", the F/S layer list).  Raises ValueError otherwise.
    """
    if not isinstance(pattern, str):
        raise ValueError("pattern must be a string")
    kinds = []
    for ch in pattern:
        if ch in ", ":
            continue
        if ch not in "FS":
            raise ValueError("bad character %r in layer pattern" % ch)
        kinds.append(ch)
    if not kinds:
        raise ValueError("empty layer pattern")
    if kinds[0] != "F":
        raise ValueError("the first layer must be F")
    return kinds


def layer_stack(pattern: str, layers: list[dict], k: int, scale: float, dv: int | None = None,
                nthreads: int | None = None, keep_scores: bool = False):
    """The routing loop of the pages, without FFN: for each layer l,
    F: I = Indexer_l, T = top-k(I), T_cache = T;  S: T = T_cache;  then
    out_l = SparseAttn_l(T).

    Each layer dict holds ``q_idx [L,H,D]``, ``k_idx [L,D]``, ``w [L,H]`` (needed on
    F layers) and ``q [L,Hq,Dk]``, ``kv [L,*]`` (and ``v`` for the MQA form).
    Positions are 0..L-1 (prefill).  Scores are rounded to fp32 before the top-k,
    the precision the top-k compares in.  Returns a list of per-layer dicts with
    ``T`` (int32 [L,k]), ``out``, ``lse`` and, if asked, ``scores``.
    """
    kinds = parse_pattern(pattern)
    if len(kinds) != len(layers):
        raise ValueError("pattern has %d layers, got %d inputs" % (len(kinds), len(layers)))
    t_cache = None
    res = []
    for kind, lay in zip(kinds, layers):
        entry = {"kind": kind}
        if kind == "F":
            I = indexer_scores(lay["q_idx"], lay["k_idx"], lay["w"], pos0=0, nthreads=nthreads)
            I32 = I.astype(np.float32)
            L = I32.shape[0]
            T = topk(I32, k, valid=causal_valid(L, 0, I32.shape[1]), nthreads=nthreads)
            t_cache = T
            if keep_scores:
                entry["scores"] = I
        else:
            T = t_cache
        out, lse = sparse_attn(lay["q"], lay["kv"], T, scale, dv=dv, v=lay.get("v"),
                               nthreads=nthreads)
        entry.update(T=T, out=out, lse=lse)
        res.append(entry)
    return res
