"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds random draws, shapes and dtype casts only: none of the
method's arithmetic.  It is the one piece shared by the CUDA path's tests and
bench and by the CPU oracle's tests (the oracle itself never imports it; the
tests pass it the same arrays).

Workloads (names used everywhere in this repository):

``tiny_stack``    4 layers "F,S,S,S", L=1024, fp32.  Indexer H=4, D=32, k=64,
                  q,k ~ N(0, std 1/sqrt(32)), w ~ U(0,1).  Attention in MQA form:
                  4 heads, d=64, one shared K and V, all N(0,1); scale 1/sqrt(64).
                  Indexer keys (and queries) follow K_{l+1} = 0.9 K_l + 0.436 noise.
``prefill_8k``    1 layer "F", L=8192, bf16, k=2048.  Indexer H=64, D=128,
                  q,k ~ N(0, std 1/sqrt(128)), w ~ U(0,1)/8, 64 heavy keys.
                  Absorbed MLA: 16 heads x 576 over a shared 576-d latent, 512-d out.
``stack_32k``     8 layers "F,S,S,S,F,S,S,S", L=32768, bf16, shapes of prefill_8k,
                  AR(1) indexer keys/queries across layers.
``prefill_200k``  4 layers "F,S,S,S" (vs "F,F,F,F"), L=200000, bf16 (and an
                  e4m3 indexer), shapes of prefill_8k.
``decode_200k``   64 sequences x 1 new token over a 200000-token context,
                  4 layers "F,S,S,S"; e4m3 indexer key cache with per-token
                  scales, bf16 latent KV cache.

Heavy keys: one seeded unit vector u in R^D and 64 distinct positions; those
keys get +3 sigma sqrt(D) u = +3u (3x a typical key's norm along u), the same
u and positions on every layer.
"""
from __future__ import annotations

import dataclasses
import math
import zlib

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    L: int                    # tokens (prefill) or context length (decode)
    pattern: str
    dtype: torch.dtype        # input dtype of indexer and attention tensors
    H: int                    # indexer heads
    D: int                    # indexer head dim
    k: int                    # top-k
    w_scale: float            # w ~ U(0,1) * w_scale
    heavy: int                # number of heavy key positions
    attn: str                 # "mqa" or "mla"
    Hq: int                   # attention heads
    Dk: int                   # attention key dim (576 latent+rope for MLA)
    Dv: int                   # attention value / output dim
    batch: int = 1            # sequences (decode)
    decode: bool = False
    ar1: bool = True          # AR(1) correlation of indexer inputs across layers

    @property
    def layers(self) -> int:
        return len([c for c in self.pattern if c in "FS"])

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.Dk)


WORKLOADS = {
    "tiny_stack": Workload("tiny_stack", 1024, "F,S,S,S", torch.float32, 4, 32, 64, 1.0, 0,
                           "mqa", 4, 64, 64),
    "prefill_8k": Workload("prefill_8k", 8192, "F", torch.bfloat16, 64, 128, 2048, 0.125, 64,
                           "mla", 16, 576, 512),
    "stack_32k": Workload("stack_32k", 32768, "F,S,S,S,F,S,S,S", torch.bfloat16, 64, 128, 2048,
                          0.125, 64, "mla", 16, 576, 512),
    "prefill_200k": Workload("prefill_200k", 200000, "F,S,S,S", torch.bfloat16, 64, 128, 2048,
                             0.125, 64, "mla", 16, 576, 512),
    "decode_200k": Workload("decode_200k", 200000, "F,S,S,S", torch.bfloat16, 64, 128, 2048,
                            0.125, 64, "mla", 16, 576, 512, batch=64, decode=True),
}


def variant(base: str, **changes) -> Workload:
    """A named workload with some fields replaced (smaller L for parity tests, etc.)."""
    return dataclasses.replace(WORKLOADS[base], **changes)


def _seed(*parts) -> int:
    return zlib.crc32("/".join(str(p) for p in parts).encode()) & 0x7FFFFFFF


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def _normal(shape, std, device, *parts) -> torch.Tensor:
    g = _gen(device, *parts)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def _uniform(shape, device, *parts) -> torch.Tensor:
    g = _gen(device, *parts)
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32)


def heavy_keys(wl: Workload, seed: int = 0):
    """(positions int64 [heavy], u float32 [D]) -- drawn on the CPU, tiny."""
    if wl.heavy == 0:
        return torch.zeros(0, dtype=torch.int64), torch.zeros(wl.D)
    g = _gen("cpu", seed, wl.name, "heavy_pos")
    pos = torch.randperm(wl.L, generator=g)[: wl.heavy]
    u = _normal((wl.D,), 1.0, "cpu", seed, wl.name, "heavy_dir")
    u = u / u.norm()
    return pos, u


def indexer_inputs(wl: Workload, layer: int, device="cpu", seed: int = 0, rows: int | None = None):
    """Indexer inputs of one layer: dict(q_idx [B?,R,H,D], k_idx [B?,Lk,D], w [B?,R,H]).

    Prefill: R = L query rows (or the first ``rows``), Lk = L.  Decode: a batch
    axis of wl.batch sequences, R = 1 new token, Lk = L keys.
    Layer l's keys (and queries) are AR(1) in l: X_l = 0.9 X_{l-1} + 0.436 N_l.
    """
    std = 1.0 / math.sqrt(wl.D)
    B = wl.batch
    R = 1 if wl.decode else (rows if rows is not None else wl.L)
    qshape = (B, R, wl.H, wl.D) if wl.decode else (R, wl.H, wl.D)
    kshape = (B, wl.L, wl.D) if wl.decode else (wl.L, wl.D)
    wshape = (B, R, wl.H) if wl.decode else (R, wl.H)

    def ar1(shape, tag):
        x = _normal(shape, std, device, seed, wl.name, tag, 0)
        if wl.ar1:
            for l in range(1, layer + 1):
                x.mul_(0.9).add_(_normal(shape, std, device, seed, wl.name, tag, l), alpha=0.436)
        return x

    q = ar1(qshape, "q_idx")
    k = ar1(kshape, "k_idx")
    if wl.heavy:
        pos, u = heavy_keys(wl, seed)
        u = u.to(device)
        if wl.decode:
            k[:, pos.to(device), :] += 3.0 * u
        else:
            k[pos.to(device), :] += 3.0 * u
    w = _uniform(wshape, device, seed, wl.name, "w") * wl.w_scale
    return {"q_idx": q.to(wl.dtype), "k_idx": k.to(wl.dtype), "w": w}


def attn_inputs(wl: Workload, layer: int, device="cpu", seed: int = 0, rows: int | None = None):
    """Attention inputs of one layer, all N(0,1), drawn fresh per layer.

    MLA: dict(q [R,Hq,Dk], kv [L,Dk]); MQA: dict(q [R,Hq,Dk], kv [L,Dk], v [L,Dv]).
    Decode adds a leading batch axis and R = 1.
    """
    B = wl.batch
    R = 1 if wl.decode else (rows if rows is not None else wl.L)
    lead_q = (B, R) if wl.decode else (R,)
    lead_kv = (B, wl.L) if wl.decode else (wl.L,)
    out = {
        "q": _normal(lead_q + (wl.Hq, wl.Dk), 1.0, device, seed, wl.name, "q", layer).to(wl.dtype),
        "kv": _normal(lead_kv + (wl.Dk,), 1.0, device, seed, wl.name, "kv", layer).to(wl.dtype),
    }
    if wl.attn == "mqa":
        out["v"] = _normal(lead_kv + (wl.Dv,), 1.0, device, seed, wl.name, "v", layer).to(wl.dtype)
    return out


def sample_rows(L: int, k: int, n: int, block: int, seed: int = 0) -> torch.Tensor:
    """A seeded, sorted sample of n query rows that covers the first rows (t < k),
    the last rows, the rows either side of every row-block boundary, and random rows."""
    pick = set()
    for t in (0, 1, 2, k - 2, k - 1, k, k + 1, L - 2, L - 1):
        if 0 <= t < L:
            pick.add(t)
    b = block
    while b < L and len(pick) < n // 2:
        for t in (b - 1, b):
            pick.add(t)
        b += block
    g = _gen("cpu", seed, "rows", L, k, n)
    for t in torch.randint(0, L, (4 * n,), generator=g).tolist():
        if len(pick) >= n:
            break
        pick.add(int(t))
    return torch.tensor(sorted(pick)[:n], dtype=torch.int64)
