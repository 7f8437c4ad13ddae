"""The CUDA path against the oracle at the workloads' own sizes.

* ``prefill_8k`` (one F layer, L = 8192, k = 2048, bf16) in full: every score of
  the indexer, the top-k bit for bit on the GPU's own scores, every row of the
  stack's index set (near-ties with the k-th score only) and every attention output.
* ``prefill_200k`` (L = 200000, layers F,S as in the benchmarked stack, bf16 and
  e4m3 indexers) on sampled query rows: the first rows (t < k), both sides of the
  4096-row block edges the stack streams through, the last two rows and random
  rows; plus 8-row score blocks far down the causal triangle.
* ``stack_32k`` (8 layers F,S,S,S,F,S,S,S at L = 32768) on sampled rows: both F
  layers' index sets and all eight layers' outputs.
* ``decode_200k`` (64 sequences x 1 token over 200000 keys, e4m3 key cache, F,S)
  on sampled sequences: the index set and both layers' outputs.

Tolerances as in test_gpu_parity.py.  Every input is drawn by the seeded
generators on the device; the oracle receives copies of the exact device values.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_indexer_sum_b200 import binding as ic
from sparse_attention_indexer_sum_b200 import synth
from tests.paritylib import (assert_attn_close, assert_fp8_scores_close_to_unquantised,
                             assert_scores_close, check_index_row)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    return t.detach().double().cpu().numpy()


def _inputs(wl, layers, fp8, device=DEV):
    """Device tensors of the given layers (indexer inputs on F layers)."""
    kinds = [c for c in wl.pattern if c in "FS"]
    out = []
    for l in layers:
        d = {}
        if kinds[l] == "F":
            d.update(synth.indexer_inputs(wl, l, device=device))
            if fp8:
                d["q_raw"], d["k_raw"] = d["q_idx"], d["k_idx"]
                d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_raw"])
                d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(d["k_raw"])
        d.update(synth.attn_inputs(wl, l, device=device))
        shape = (wl.batch, 1, wl.Hq, wl.Dv) if wl.decode else (wl.L, wl.Hq, wl.Dv)
        d["out"] = torch.empty(shape, dtype=torch.bfloat16, device=device)
        d["lse"] = torch.empty(shape[:-1], dtype=torch.float32, device=device)
        out.append(d)
    torch.cuda.synchronize()
    return out


def _desc(wl, fp8):
    return ic.make_desc(L=wl.L, k=wl.k, H=wl.H, D=wl.D,
                        idx_dtype=ic.IC_E4M3 if fp8 else ic.IC_BF16, heads=wl.Hq, dk=wl.Dk,
                        dv=wl.Dv, attn_dtype=ic.IC_BF16, scale=wl.scale, batch=wl.batch,
                        decode=wl.decode)


def _host_keys(d, fp8):
    """fp64 copy of a layer's indexer keys as the kernels see them."""
    if fp8:
        return oracle.dequant_rows_e4m3(d["k_idx"].cpu().numpy(), d["k_scale"].cpu().numpy())
    return _f64(d["k_idx"])


def _host_queries(d, rows_t, fp8):
    if fp8:
        return oracle.dequant_rows_e4m3(d["q_idx"][rows_t].cpu().numpy(),
                                        d["q_scale"][rows_t].cpu().numpy())
    return _f64(d["q_idx"][rows_t])


def _oracle_rows(d, rows, k_host, fp8):
    """Oracle scores of query rows `rows` (positions = rows) of a prefill F layer."""
    rows_t = torch.from_numpy(rows).to(d["q_idx"].device)
    return oracle.indexer_scores_at(_host_queries(d, rows_t, fp8), k_host, _f64(d["w"][rows_t]),
                                    rows)


def _attn_rows(d, rows, T_rows, kv_host, scale):
    rows_t = torch.from_numpy(rows).to(d["q"].device)
    ro, rl = oracle.sparse_attn(_f64(d["q"][rows_t]), kv_host, T_rows, scale, dv=512)
    assert_attn_close(d["out"][rows_t].float().cpu().numpy(), ro)
    np.testing.assert_allclose(d["lse"][rows_t].cpu().numpy(), rl, atol=2e-3, rtol=1e-3)


# ------------------------------------------------------------------------- prefill_8k, full
def test_prefill_8k_full_tensors():
    wl = synth.WORKLOADS["prefill_8k"]
    (d,) = _inputs(wl, [0], fp8=False)
    desc = _desc(wl, False)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    t_cache = torch.full((wl.L, wl.k), -7, dtype=torch.int32, device=DEV)
    ic.ic_layer_stack(wl.pattern, desc, [d], t_cache, ws)      # 4096-row blocks, as benchmarked
    scores = ic.ic_indexer_scores(d["q_idx"], d["k_idx"], d["w"])
    ic.ic_device_status()
    q, k, w = _f64(d["q_idx"]), _f64(d["k_idx"]), _f64(d["w"])
    ref = oracle.indexer_scores(q, k, w)
    del q
    got = scores.cpu().numpy()
    assert_scores_close(got, ref)
    # top-k bit for bit on the GPU's own fp32 scores
    T_own = ic.ic_topk(scores, wl.k, pos0=0).cpu().numpy()
    ic.ic_device_status()
    np.testing.assert_array_equal(T_own, oracle.topk(got, wl.k,
                                                     valid=oracle.causal_valid(wl.L, 0, wl.L)))
    del got, scores
    # the stack's index set: every row against the oracle's scores
    T = t_cache.cpu().numpy()
    np.testing.assert_array_equal(T, T_own)
    diffs = sum(check_index_row(T[t], ref[t], wl.k, t + 1) for t in range(wl.L))
    assert diffs <= wl.L * 8, diffs                 # near-ties only, and few of them
    del ref
    # every attention output and lse over the stack's T
    ro, rl = oracle.sparse_attn(_f64(d["q"]), _f64(d["kv"]), T, wl.scale, dv=wl.Dv)
    assert_attn_close(d["out"].float().cpu().numpy(), ro)
    np.testing.assert_allclose(d["lse"].cpu().numpy(), rl, atol=2e-3, rtol=1e-3)


# ---------------------------------------------------------------- prefill_200k, sampled rows
@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
def test_prefill_200k_sampled_rows(fp8):
    wl = synth.variant("prefill_200k", pattern="F,S")
    lay = _inputs(wl, [0, 1], fp8)
    desc = _desc(wl, fp8)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    t_cache = torch.full((wl.L, wl.k), -7, dtype=torch.int32, device=DEV)
    ic.ic_layer_stack(wl.pattern, desc, lay, t_cache, ws)
    ic.ic_device_status()
    del ws
    d0 = lay[0]
    rows = synth.sample_rows(wl.L, wl.k, 48, 4096).numpy()
    assert rows[-1] == wl.L - 1 and rows[-2] == wl.L - 2 and rows[0] == 0
    k_host = _host_keys(d0, fp8)
    ref = _oracle_rows(d0, rows, k_host, fp8)
    T = t_cache[torch.from_numpy(rows).to(DEV)].cpu().numpy()
    for j, t in enumerate(rows):
        check_index_row(T[j], ref[j], wl.k, t + 1, rtol=1e-2)
    # both layers attend over the F layer's set
    for d in lay:
        _attn_rows(d, rows, T, _f64(d["kv"]), wl.scale)
    # score blocks of 8 rows (4-token query blocks) far down the triangle
    for p0 in (4092, 100000, wl.L - 8):
        sl = slice(p0, p0 + 8)
        qs = d0["q_scale"][sl] if fp8 else None
        ks = d0["k_scale"][: p0 + 8] if fp8 else None
        got = ic.ic_indexer_scores(d0["q_idx"][sl], d0["k_idx"][: p0 + 8], d0["w"][sl], pos0=p0,
                                   q_scale=qs, k_scale=ks).cpu().numpy()
        ic.ic_device_status()
        blk = np.arange(p0, p0 + 8)
        assert_scores_close(got, _oracle_rows(d0, blk, k_host[: p0 + 8], fp8))
        if fp8:   # against the unquantised bf16 inputs
            q_raw = _f64(d0["q_raw"][sl])
            ref_raw = oracle.indexer_scores(q_raw, _f64(d0["k_raw"][: p0 + 8]),
                                            _f64(d0["w"][sl]), pos0=p0)
            assert_fp8_scores_close_to_unquantised(got, ref_raw)


# ------------------------------------------------------------------- stack_32k, sampled rows
def test_stack_32k_sampled_rows():
    wl = synth.WORKLOADS["stack_32k"]
    lay = _inputs(wl, list(range(wl.layers)), fp8=False)
    desc = _desc(wl, False)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    t_cache = torch.full((wl.L, wl.k), -7, dtype=torch.int32, device=DEV)
    ic.ic_layer_stack(wl.pattern, desc, lay, t_cache, ws)
    ic.ic_device_status()
    rows = synth.sample_rows(wl.L, wl.k, 40, 4096, seed=3).numpy()
    # layer 4 (F) overwrote T_cache: T is its set; layers 4..7 attended over it
    T4 = t_cache[torch.from_numpy(rows).to(DEV)].cpu().numpy()
    ref4 = _oracle_rows(lay[4], rows, _host_keys(lay[4], False), False)
    for j, t in enumerate(rows):
        check_index_row(T4[j], ref4[j], wl.k, t + 1)
    # layers 0..3 attended over layer 0's set, which layer 4 overwrote: the same
    # (deterministic) kernels on layer 0 alone give it back
    t0 = torch.full_like(t_cache, -7)
    solo = dict(lay[0], out=torch.empty_like(lay[0]["out"]), lse=torch.empty_like(lay[0]["lse"]))
    ic.ic_layer_stack("F", desc, [solo], t0, ws)
    ic.ic_device_status()
    assert torch.equal(solo["out"], lay[0]["out"])
    T0 = t0[torch.from_numpy(rows).to(DEV)].cpu().numpy()
    ref0 = _oracle_rows(lay[0], rows, _host_keys(lay[0], False), False)
    for j, t in enumerate(rows):
        check_index_row(T0[j], ref0[j], wl.k, t + 1)
    for l in range(wl.layers):
        _attn_rows(lay[l], rows, T0 if l < 4 else T4, _f64(lay[l]["kv"]), wl.scale)


# -------------------------------------------------------------- decode_200k, sampled sequences
def test_decode_200k_sampled_sequences():
    wl = synth.variant("decode_200k", pattern="F,S")
    lay = _inputs(wl, [0, 1], fp8=True)
    for d in lay:
        d.pop("q_raw", None)
        d.pop("k_raw", None)
    torch.cuda.empty_cache()
    desc = _desc(wl, True)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    t_cache = torch.full((wl.batch, wl.k), -7, dtype=torch.int32, device=DEV)
    ic.ic_decode_step(wl.pattern, desc, lay, t_cache, ws)
    ic.ic_device_status()
    T = t_cache.cpu().numpy()
    d0 = lay[0]
    pos = wl.L - 1
    for b in (0, 17, 42, 63):
        k_host = oracle.dequant_rows_e4m3(d0["k_idx"][b].cpu().numpy(),
                                          d0["k_scale"][b].cpu().numpy())
        q_host = oracle.dequant_rows_e4m3(d0["q_idx"][b].cpu().numpy(),
                                          d0["q_scale"][b].cpu().numpy())
        ref = oracle.indexer_scores(q_host, k_host, _f64(d0["w"][b]), pos0=pos)[0]
        check_index_row(T[b], ref, wl.k, wl.L)
        # both layers' outputs over T[b]; the oracle gets the selected latent rows
        sel = torch.from_numpy(T[b][T[b] >= 0].astype(np.int64)).to(DEV)
        idx_local = np.arange(sel.numel(), dtype=np.int32)[None, None, :]
        for d in lay:
            kv_rows = _f64(d["kv"][b][sel])
            ro, rl = oracle.sparse_attn(_f64(d["q"][b]), kv_rows, idx_local[0], wl.scale, dv=512)
            assert_attn_close(d["out"][b].float().cpu().numpy(), ro)
            np.testing.assert_allclose(d["lse"][b].cpu().numpy(), rl, atol=2e-3, rtol=1e-3)
