"""Small, fixed cases of each hot kernel, for capturing them under a profiler.

    python -m sparse_attention_indexer_sum_b200.profile_cases indexer_longrows
    python -m sparse_attention_indexer_sum_b200.profile_cases indexer_longrows_e4m3
    python -m sparse_attention_indexer_sum_b200.profile_cases attn_tail4k
    python -m sparse_attention_indexer_sum_b200.profile_cases decode_indexer
    python -m sparse_attention_indexer_sum_b200.profile_cases decode_indexer_fused
    python -m sparse_attention_indexer_sum_b200.profile_cases decode_attn
    python -m sparse_attention_indexer_sum_b200.profile_cases decode_step

Each case builds its inputs once, on the GPU, with seeded generators. It runs the
kernels through the C ABI, 2 warm-up rounds then 3 traced rounds, and prints
each traced launch's time and throughput. With ncu, `-s 2 -c 1` on the kernel's
name captures a warm launch. Every case fits in a few GB of device memory.

  indexer_longrows  512 query rows at causal positions 100000..100511 against
                    100512 keys (bf16, H=64, d=128, w ~ U(0,1)/8): ic_indexer_scores,
                    then ic_topk (k = 2048) on the same rows.
  indexer_longrows_e4m3  the same rows with e4m3 inputs (per-row scales, quantised
                    on the GPU): ic_indexer_scores alone.
  attn_tail4k       the last 4096 query rows of the 200000-token prefill workload,
                    with index sets from the indexer + top-k on those rows, then
                    ic_sparse_attn over the full 200000-row latent KV.
  decode_indexer    64 sequences x 1 query at position 199999 over an e4m3 key
                    cache of 200000 keys (per-token scales), then ic_topk.
  decode_attn       one decode layer's attention: 64 sequences x 1 query, each
                    over 2048 random distinct rows of its own 20000-row latent KV
                    (1.5 GB in all, far beyond L2); split over the SMs, partials
                    merged by the combine kernel.
  decode_indexer_fused  the decode_indexer inputs through ic_indexer_topk (the
                    fused indexer -> top-k: indexer_tc_kernel's fused instance, then
                    topk_merge_kernel).
  decode_step       the whole F,S,S,S decode step of 64 sequences x 1 query over
                    200000 tokens (ic_decode_step: e4m3 indexer, top-k, four
                    attention layers with their merges).  The four layers share
                    one 14.7 GB latent cache and one key cache (each layer has its
                    own queries), ~17 GB in all; for a launch list only.
"""
from __future__ import annotations

import math
import sys

import torch

from . import binding as ic
from . import synth


def _report(trace):
    for name, ms, work in trace:
        unit = "TFLOP/s" if name.startswith("indexer") else "GB/s"
        rate = work / ms / 1e9 if unit == "TFLOP/s" else work / ms / 1e6
        print("%-18s %9.3f ms  %10.1f %s" % (name, ms, rate, unit))


def _rounds(fn, warm=2, timed=3):
    for _ in range(warm):
        fn()
    ic.ic_device_status()
    ic.ic_trace_begin(256)
    for _ in range(timed):
        fn()
    _, trace = ic.ic_trace_end(256)
    _report(trace)


def indexer_longrows():
    torch.manual_seed(0)
    dev = "cuda"
    R, P0 = 512, 100000
    Lk = P0 + R
    q = (torch.randn(R, 64, 128, device=dev) / math.sqrt(128)).to(torch.bfloat16)
    k = (torch.randn(Lk, 128, device=dev) / math.sqrt(128)).to(torch.bfloat16)
    w = torch.rand(R, 64, device=dev) / 8
    scores = torch.empty(R, Lk, device=dev)
    idx = torch.empty(R, 2048, dtype=torch.int32, device=dev)

    def rnd():
        ic.ic_indexer_scores(q, k, w, scores=scores, pos0=P0)
        ic.ic_topk(scores, 2048, pos0=P0, idx=idx)
    _rounds(rnd)


def indexer_longrows_e4m3():
    torch.manual_seed(0)
    dev = "cuda"
    R, P0 = 512, 100000
    Lk = P0 + R
    q = (torch.randn(R, 64, 128, device=dev) / math.sqrt(128)).to(torch.bfloat16)
    k = (torch.randn(Lk, 128, device=dev) / math.sqrt(128)).to(torch.bfloat16)
    q8, qs = ic.ic_quant_e4m3_rows(q)
    k8, ks = ic.ic_quant_e4m3_rows(k)
    w = torch.rand(R, 64, device=dev) / 8
    scores = torch.empty(R, Lk, device=dev)

    _rounds(lambda: ic.ic_indexer_scores(q8, k8, w, scores=scores, pos0=P0, q_scale=qs,
                                         k_scale=ks))


def attn_tail4k():
    dev = "cuda"
    wl = synth.WORKLOADS["prefill_200k"]
    L, R = wl.L, 4096
    P0 = L - R
    d = synth.indexer_inputs(wl, 0, device=dev)
    q_idx = d["q_idx"][P0:].clone()
    w = d["w"][P0:].clone()
    k_idx = d["k_idx"]
    del d
    torch.cuda.empty_cache()
    scores = torch.empty(R, L, device=dev)
    idx = torch.empty(R, wl.k, dtype=torch.int32, device=dev)
    ic.ic_indexer_scores(q_idx, k_idx, w, scores=scores, pos0=P0)
    ic.ic_topk(scores, wl.k, pos0=P0, idx=idx)
    ic.ic_device_status()
    del scores, q_idx, k_idx
    torch.cuda.empty_cache()
    a = synth.attn_inputs(wl, 0, device=dev)
    q = a["q"][P0:].clone()
    kv = a["kv"]
    del a
    torch.cuda.empty_cache()
    out = torch.empty(R, 16, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(R, 16, device=dev)
    _rounds(lambda: ic.ic_sparse_attn(q, kv, idx, wl.scale, out=out, lse=lse))


def decode_indexer():
    dev = "cuda"
    B, L = 64, 200000
    g = torch.Generator(device=dev).manual_seed(0)
    q = (torch.randn(B, 1, 64, 128, device=dev, generator=g) / math.sqrt(128)).to(torch.bfloat16)
    q8, qs = ic.ic_quant_e4m3_rows(q)
    k8 = torch.empty(B, L, 128, dtype=torch.uint8, device=dev)
    ks = torch.empty(B, L, dtype=torch.float32, device=dev)
    for b in range(B):
        kb = (torch.randn(L, 128, device=dev, generator=g) / math.sqrt(128)).to(torch.bfloat16)
        ic.ic_quant_e4m3_rows(kb, codes=k8[b], scales=ks[b])
    w = torch.rand(B, 1, 64, device=dev, generator=g) / 8
    scores = torch.empty(B, 1, L, device=dev)
    idx = torch.empty(B, 1, 2048, dtype=torch.int32, device=dev)

    def rnd():
        ic.ic_indexer_scores(q8, k8, w, scores=scores, pos0=L - 1, q_scale=qs, k_scale=ks)
        ic.ic_topk(scores.view(B, L), 2048, pos0=L - 1, idx=idx.view(B, 2048))
    _rounds(rnd)


def decode_indexer_fused():
    dev = "cuda"
    B, L = 64, 200000
    g = torch.Generator(device=dev).manual_seed(0)
    q = (torch.randn(B, 1, 64, 128, device=dev, generator=g) / math.sqrt(128)).to(torch.bfloat16)
    q8, qs = ic.ic_quant_e4m3_rows(q)
    k8 = torch.empty(B, L, 128, dtype=torch.uint8, device=dev)
    ks = torch.empty(B, L, dtype=torch.float32, device=dev)
    for b in range(B):
        kb = (torch.randn(L, 128, device=dev, generator=g) / math.sqrt(128)).to(torch.bfloat16)
        ic.ic_quant_e4m3_rows(kb, codes=k8[b], scales=ks[b])
    w = torch.rand(B, 1, 64, device=dev, generator=g) / 8
    ws = torch.empty(ic.ic_indexer_topk_workspace_size(B, L, L - 1) // 4 + 4, device=dev)
    _rounds(lambda: ic.ic_indexer_topk(q8, k8, w, 2048, ws, pos0=L - 1, q_scale=qs, k_scale=ks))


def decode_attn():
    dev = "cuda"
    wl = synth.variant("decode_200k", L=20000)
    B, L, k = wl.batch, wl.L, wl.k
    a = synth.attn_inputs(wl, 0, device=dev)
    q, kv = a["q"], a["kv"]
    g = torch.Generator(device=dev).manual_seed(0)
    idx = torch.empty(B, 1, k, dtype=torch.int32, device=dev)
    for b in range(B):
        idx[b, 0] = torch.sort(torch.randperm(L, device=dev, generator=g)[:k]).values.int()
    ws = torch.empty(ic.ic_attn_workspace_size(B, 1, wl.Hq, wl.Dv, k) // 4 + 1, device=dev)
    out = torch.empty(B, 1, wl.Hq, wl.Dv, dtype=torch.bfloat16, device=dev)
    _rounds(lambda: ic.ic_sparse_attn(q, kv, idx, wl.scale, out=out, workspace=ws))


def decode_step():
    dev = "cuda"
    wl = synth.WORKLOADS["decode_200k"]
    B, L, k = wl.batch, wl.L, wl.k
    d = synth.indexer_inputs(wl, 0, device=dev)
    q8, qs = ic.ic_quant_e4m3_rows(d["q_idx"])
    k8, ks = ic.ic_quant_e4m3_rows(d.pop("k_idx"))
    kv = synth.attn_inputs(wl, 0, device=dev)["kv"]
    torch.cuda.empty_cache()
    g = torch.Generator(device=dev).manual_seed(1)
    layers = []
    for _ in range(wl.layers):
        q = torch.randn(B, 1, wl.Hq, wl.Dk, device=dev, generator=g).to(torch.bfloat16)
        layers.append({"q_idx": q8, "q_scale": qs, "k_idx": k8, "k_scale": ks, "w": d["w"],
                       "q": q, "kv": kv,
                       "out": torch.empty(B, 1, wl.Hq, wl.Dv, dtype=torch.bfloat16, device=dev),
                       "lse": torch.empty(B, 1, wl.Hq, device=dev)})
    desc = ic.make_desc(L=L, k=k, H=wl.H, D=wl.D, idx_dtype=ic.IC_E4M3, heads=wl.Hq, dk=wl.Dk,
                        dv=wl.Dv, attn_dtype=ic.IC_BF16, scale=wl.scale, batch=B, decode=True)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=dev)
    t_cache = torch.empty(B, k, dtype=torch.int32, device=dev)
    _rounds(lambda: ic.ic_decode_step(wl.pattern, desc, layers, t_cache, ws))


CASES = {"indexer_longrows": indexer_longrows, "indexer_longrows_e4m3": indexer_longrows_e4m3,
         "attn_tail4k": attn_tail4k,
         "decode_indexer": decode_indexer, "decode_indexer_fused": decode_indexer_fused,
         "decode_attn": decode_attn,
         "decode_step": decode_step}


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    if len(argv) != 1 or argv[0] not in CASES:
        print("usage: python -m sparse_attention_indexer_sum_b200.profile_cases {%s}" %
              ",".join(CASES), file=sys.stderr)
        return 2
    CASES[argv[0]]()
    return 0


if __name__ == "__main__":
    sys.exit(main())
