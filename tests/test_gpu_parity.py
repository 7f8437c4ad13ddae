"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Tolerances: indexer scores rel 1e-2 / abs 1e-3 (bf16 inputs) and rel 5e-2 (fp8);
top-k bit-exact on the same fp32 scores; index sets may differ from the oracle's
only on near-ties with the k-th score; attention max-abs 2e-2 and mean-abs 2e-3
(bf16 output).  Sizes span several tiles with ragged tails; every input is seeded.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_indexer_sum_b200 import binding as ic
from sparse_attention_indexer_sum_b200 import synth
from tests.paritylib import (IDX_ATOL, IDX_RTOL_BF16, assert_attn_close,
                             assert_fp8_scores_close_to_unquantised, assert_scores_close,
                             check_index_row)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def _sync():
    ic.ic_device_status()


# ------------------------------------------------------------------------------- top-k
@pytest.mark.parametrize("rows,n,k,pos0", [(64, 5000, 2048, -1), (33, 3000, 64, 0),
                                           (40, 2100, 2048, 2040), (7, 200000, 2048, -1)])
def test_topk_bit_exact_random(rows, n, k, pos0):
    g = torch.Generator().manual_seed(rows * 7 + n)
    s = torch.randn(rows, n, generator=g)
    got = ic.ic_topk(s.to(DEV), k, pos0=pos0)
    _sync()
    valid = np.full(rows, n, np.int32) if pos0 < 0 else oracle.causal_valid(rows, pos0, n)
    ref = oracle.topk(s.numpy(), k, valid=valid)
    np.testing.assert_array_equal(got.cpu().numpy(), ref)


def test_topk_ties_signed_zeros_and_degenerate_rows():
    k = 2048
    n = 12000
    rows = []
    rows.append(np.zeros(n, np.float32))                                   # all zero
    rows.append(np.full(n, 1.5, np.float32))                               # all equal
    r = np.zeros(n, np.float32)
    r[::2] = -0.0
    rows.append(r)                                                         # -0 / +0 mix
    g = np.random.default_rng(0)
    rows.append(g.choice([0.0, 0.25, 0.5, 1.0], size=n).astype(np.float32))  # heavy ties
    r = g.standard_normal(n).astype(np.float32)
    r[:9000] = 0.75                                                        # > CAP equal keys
    rows.append(r)
    r = np.maximum(g.standard_normal(n), 0).astype(np.float32)             # ReLU-like: many zeros
    rows.append(r)
    r = (1.0 + g.integers(0, 3, n) * 2.0 ** -20).astype(np.float32)        # ties in low bits
    rows.append(r)
    rows.append(-np.abs(g.standard_normal(n)).astype(np.float32))          # all negative
    s = np.stack(rows)
    got = ic.ic_topk(torch.from_numpy(s).to(DEV), k).cpu().numpy()
    _sync()
    np.testing.assert_array_equal(got, oracle.topk(s, k))


@pytest.mark.parametrize("nrows", [8, 17, 64])
def test_topk_row_clusters_with_ties(nrows):
    """Few long rows are split over a cluster of CTAs (8, 4 and 2 per row here):
    degenerate and tie-heavy rows (exact fallback in the merging CTA) and random rows,
    bit-exact."""
    k, n = 2048, 40000
    g = np.random.default_rng(nrows)
    rows = [np.zeros(n, np.float32), np.full(n, -2.5, np.float32)]
    r = np.zeros(n, np.float32)
    r[1::2] = -0.0
    rows.append(r)
    rows.append(g.choice([0.0, 0.5, 1.0], size=n).astype(np.float32))
    r = g.standard_normal(n).astype(np.float32)
    r[5000:12000] = 1.25                              # ties around the k-th key
    rows.append(r)
    r = g.standard_normal(n).astype(np.float32)
    r[-3000:] = 9.0                                   # the top keys all in the last part
    rows.append(r)
    while len(rows) < nrows:
        rows.append(g.standard_normal(n).astype(np.float32))
    s = np.stack(rows[:nrows])
    got = ic.ic_topk(torch.from_numpy(s).to(DEV), k).cpu().numpy()
    _sync()
    np.testing.assert_array_equal(got, oracle.topk(s, k))


def test_topk_decode_shape_clusters_and_causal():
    """64 rows of 200000 scores at causal position 199999 (the decode step's shape)."""
    g = torch.Generator().manual_seed(11)
    s = torch.randn(64, 200000, generator=g)
    got = ic.ic_topk(s.to(DEV), 2048, pos0=199999).cpu().numpy()
    _sync()
    ref = oracle.topk(s.numpy(), 2048, valid=oracle.causal_valid(64, 199999, 200000))
    np.testing.assert_array_equal(got, ref)


def test_topk_varlen_rows_bit_exact():
    """Per-row candidate counts from a device array: 0, 1, k-1, k, k+1, the whole
    row, counts past the row (clamped) and random ones, on random and tied rows."""
    k, n = 2048, 9000
    g = torch.Generator().manual_seed(21)
    s = torch.randn(40, n, generator=g)
    s[3] = 0.0
    s[4, ::3] = 1.0
    lens = [0, 1, k - 1, k, k + 1, n, n + 50, 4321] + \
        torch.randint(0, n + 1, (32,), generator=g).tolist()
    vl = torch.tensor(lens, dtype=torch.int32)
    got = ic.ic_topk_varlen(s.to(DEV), k, vl.to(DEV)).cpu().numpy()
    _sync()
    ref = oracle.topk(s.numpy(), k, valid=np.minimum(vl.numpy(), n))
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("n", [1, 2047, 2048, 2049, 4096])
def test_topk_sizes_around_k(n):
    k = 2048
    g = torch.Generator().manual_seed(n)
    s = torch.randn(3, n, generator=g)
    got = ic.ic_topk(s.to(DEV), k).cpu().numpy()
    _sync()
    np.testing.assert_array_equal(got, oracle.topk(s.numpy(), k))


def test_topk_strided_rows_and_causal():
    g = torch.Generator().manual_seed(5)
    big = torch.randn(50, 3001, generator=g)
    view = big[:, :2999]                       # ld = 3001 (not a multiple of 4): scalar loads
    dev = big.to(DEV)
    got = ic.ic_topk(dev[:, :2999], 100, n=2999, pos0=2950).cpu().numpy()
    _sync()
    ref = oracle.topk(view.numpy(), 100, valid=oracle.causal_valid(50, 2950, 2999))
    np.testing.assert_array_equal(got, ref)


# ------------------------------------------------------------------------------- indexer
def _idx_inputs(B, R, Lk, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, R, 64, 128, generator=g) / math.sqrt(128)).to(dtype)
    k = (torch.randn(B, Lk, 128, generator=g) / math.sqrt(128)).to(dtype)
    w = torch.rand(B, R, 64, generator=g) / 8
    return q, k, w


@pytest.mark.parametrize("B,R,Lk,pos0", [(1, 1000, 1000, 0), (1, 6, 300, 200), (3, 1, 777, 776),
                                         (2, 130, 259, 0), (1, 4, 129, 125)])
def test_indexer_bf16_parity(B, R, Lk, pos0):
    q, k, w = _idx_inputs(B, R, Lk, seed=B * 1000 + R)
    got = ic.ic_indexer_scores(q.to(DEV), k.to(DEV), w.to(DEV), pos0=pos0)
    _sync()
    ref = oracle.indexer_scores(q.float().numpy(), k.float().numpy(), w.numpy(), pos0=pos0)
    assert_scores_close(got.cpu().numpy(), ref)


def test_indexer_bf16_heavy_keys_and_ld():
    wl = synth.variant("prefill_8k", L=1500)
    d = synth.indexer_inputs(wl, 0)
    scores = torch.full((1500, 1600), 7.0, device=DEV)     # ld > Lk: columns >= Lk untouched
    ic.ic_indexer_scores(d["q_idx"].to(DEV), d["k_idx"].to(DEV), d["w"].to(DEV), scores=scores)
    _sync()
    ref = oracle.indexer_scores(d["q_idx"].float().numpy(), d["k_idx"].float().numpy(),
                                d["w"].numpy())
    got = scores.cpu().numpy()
    assert_scores_close(got[:, :1500], ref)
    assert (got[:, 1500:] == 7.0).all()


def test_quant_e4m3_bit_exact():
    g = torch.Generator().manual_seed(11)
    x = torch.randn(300, 128, generator=g) * torch.rand(300, 1, generator=g) * 5
    x[7] = 0
    xb = x.to(torch.bfloat16)
    codes, scales = ic.ic_quant_e4m3_rows(xb.to(DEV))
    _sync()
    rc, rs = oracle.quant_rows_e4m3(xb.float().numpy())
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)


@pytest.mark.parametrize("B,R,Lk,pos0", [(1, 700, 700, 0), (4, 1, 1000, 999)])
def test_indexer_fp8_parity(B, R, Lk, pos0):
    q, k, w = _idx_inputs(B, R, Lk, seed=77 + R)
    qc, qs = ic.ic_quant_e4m3_rows(q.to(DEV))
    kc, ks = ic.ic_quant_e4m3_rows(k.to(DEV))
    got = ic.ic_indexer_scores(qc, kc, w.to(DEV), pos0=pos0, q_scale=qs, k_scale=ks)
    _sync()
    got = got.cpu().numpy()
    # (i) same e4m3 values: tight
    ref_q = oracle.indexer_scores_e4m3(qc.cpu().numpy(), qs.cpu().numpy(), kc.cpu().numpy(),
                                       ks.cpu().numpy(), w.numpy(), pos0=pos0)
    assert_scores_close(got, ref_q)
    # (ii) against the unquantised bf16 inputs: rel 5e-2 with a row-RMS floor
    ref = oracle.indexer_scores(q.float().numpy(), k.float().numpy(), w.numpy(), pos0=pos0)
    assert_fp8_scores_close_to_unquantised(got, ref)


def test_indexer_f32_parity():
    wl = synth.WORKLOADS["tiny_stack"]
    d = synth.indexer_inputs(wl, 2)
    got = ic.ic_indexer_scores(d["q_idx"].to(DEV), d["k_idx"].to(DEV), d["w"].to(DEV))
    _sync()
    ref = oracle.indexer_scores(d["q_idx"].numpy(), d["k_idx"].numpy(), d["w"].numpy())
    assert_scores_close(got.cpu().numpy(), ref, atol=1e-5, rtol=1e-5)


# ------------------------------------------------------------------------------- attention
def _rand_idx(B, R, k, Lkv, seed, pad_from=None):
    g = np.random.default_rng(seed)
    idx = np.stack([np.stack([np.sort(g.permutation(Lkv)[:k]) for _ in range(R)])
                    for _ in range(B)]).astype(np.int32)
    if pad_from is not None:
        for r in range(R):
            cut = pad_from[r] if hasattr(pad_from, "__len__") else pad_from
            idx[:, r, cut:] = -1
    return idx


@pytest.mark.parametrize("B,R,k,Lkv", [(1, 37, 2048, 3000), (5, 1, 2048, 2500), (1, 9, 100, 150),
                                       (2, 7, 37, 90)])
def test_attn_mla_parity(B, R, k, Lkv):
    g = torch.Generator().manual_seed(B * 100 + R)
    q = torch.randn(B, R, 16, 576, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lkv, 576, generator=g).to(torch.bfloat16)
    pads = [k - (r * 37) % max(1, k // 2) for r in range(R)]
    idx = _rand_idx(B, R, k, Lkv, seed=R, pad_from=pads)
    idx[:, 0, 5] = -1                                   # a hole in the middle
    scale = 1 / math.sqrt(576)
    ws = torch.empty(ic.ic_attn_workspace_size(B, R, 16, 512, k) // 4 + 1, device=DEV)
    lse = torch.empty(B, R, 16, device=DEV)
    out = ic.ic_sparse_attn(q.to(DEV), kv.to(DEV), torch.from_numpy(idx).to(DEV), scale, lse=lse,
                            workspace=ws)
    _sync()
    ro, rl = oracle.sparse_attn(q.float().numpy(), kv.float().numpy(), idx, scale, dv=512)
    assert_attn_close(_np(out), ro)
    np.testing.assert_allclose(lse.cpu().numpy(), rl, atol=2e-3, rtol=1e-3)


def test_pack_kv_e4m3_bit_exact():
    g = torch.Generator().manual_seed(31)
    kv = torch.randn(333, 576, generator=g) * torch.rand(333, 1, generator=g) * 4
    kv[7] = 0
    kv[9, 128:256] = 0            # one all-zero group: scale 1, codes 0
    kv[11, :128] *= 1e-4          # a tiny group next to large ones
    kvb = kv.to(torch.bfloat16)
    packed = ic.ic_pack_kv_e4m3(kvb.to(DEV))
    _sync()
    P = packed.cpu().numpy()
    codes, scales, rope = oracle.kv_pack_e4m3(kvb.float().numpy())
    np.testing.assert_array_equal(P[:, :512], codes)
    np.testing.assert_array_equal(P[:, 512:528].view(np.float32), scales)
    np.testing.assert_array_equal(P[:, 528:].view(np.uint16),
                                  kvb[:, 512:].view(torch.int16).numpy().view(np.uint16))


def _unpack_kv8(P):
    P = np.ascontiguousarray(P)
    codes = P[..., :512]
    scales = np.ascontiguousarray(P[..., 512:528]).view(np.float32)
    rope = torch.from_numpy(np.ascontiguousarray(P[..., 528:]).view(np.int16)).view(
        torch.bfloat16).float().numpy()
    return codes, scales, rope


@pytest.mark.parametrize("B,R,k,Lkv", [(1, 37, 2048, 3000), (6, 1, 2048, 4000), (2, 7, 37, 90),
                                       (64, 1, 2048, 2100)])
def test_attn_mla_kv8_parity(B, R, k, Lkv):
    """Absorbed MLA over the fp8 cache (split and unsplit forms, ragged lists, a hole)
    against the oracle on the dequantised cache rows."""
    g = torch.Generator().manual_seed(B * 17 + R)
    q = torch.randn(B, R, 16, 576, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lkv, 576, generator=g).to(torch.bfloat16)
    pads = [k - (r * 37) % max(1, k // 2) for r in range(R)]
    idx = _rand_idx(B, R, k, Lkv, seed=R + 5, pad_from=pads)
    idx[:, 0, 5 % k] = -1
    packed = ic.ic_pack_kv_e4m3(kv.to(DEV))
    scale = 1 / math.sqrt(576)
    ws = torch.empty(ic.ic_attn_workspace_size(B, R, 16, 512, k) // 4 + 1, device=DEV)
    lse = torch.empty(B, R, 16, device=DEV)
    out = ic.ic_sparse_attn(q.to(DEV), packed, torch.from_numpy(idx).to(DEV), scale, lse=lse,
                            workspace=ws)
    _sync()
    codes, scales, rope = _unpack_kv8(packed.cpu().numpy())
    ro, rl = oracle.sparse_attn_kv_e4m3(q.float().numpy(), codes, scales, rope, idx, scale)
    assert_attn_close(_np(out), ro)
    np.testing.assert_allclose(lse.cpu().numpy(), rl, atol=2e-3, rtol=1e-3)


def test_attn_mla_decode_split_equals_unsplit():
    B, k, Lkv = 6, 2048, 4000
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, 1, 16, 576, generator=g).to(torch.bfloat16).to(DEV)
    kv = torch.randn(B, Lkv, 576, generator=g).to(torch.bfloat16).to(DEV)
    idx = torch.from_numpy(_rand_idx(B, 1, k, Lkv, seed=9)).to(DEV)
    ws = torch.empty(ic.ic_attn_workspace_size(B, 1, 16, 512, k) // 4 + 1, device=DEV)
    assert ws.numel() > 1
    o_split = ic.ic_sparse_attn(q, kv, idx, 0.05, workspace=ws)
    o_one = ic.ic_sparse_attn(q, kv, idx, 0.05)
    # a workspace that is large enough but not 16-byte aligned: no split, exactly
    # the result without a workspace
    o_mis = ic.ic_sparse_attn(q, kv, idx, 0.05, workspace=ws[1:])
    _sync()
    ro, _ = oracle.sparse_attn(q.float().cpu().numpy(), kv.float().cpu().numpy(),
                               idx.cpu().numpy(), 0.05, dv=512)
    assert_attn_close(_np(o_split), ro)
    assert_attn_close(_np(o_one), ro)
    assert torch.equal(o_mis, o_one)


@pytest.mark.parametrize("B,R,k,Lkv", [(1, 1, 2048, 5000), (2, 1, 2048, 3000), (3, 1, 1000, 1200),
                                       (1, 2, 33, 40), (64, 1, 2048, 2100)])
def test_attn_mla_split_pieces(B, R, k, Lkv):
    """Few queries: the (query, tile) pairs are cut into one range per SM, so a query
    can be split into up to 64 pieces (one or two tiles each) merged by the combine
    kernel; ragged lists (-1 tails) and a hole included."""
    g = torch.Generator().manual_seed(B * 1000 + R * 10 + k)
    q = torch.randn(B, R, 16, 576, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lkv, 576, generator=g).to(torch.bfloat16)
    idx = _rand_idx(B, R, k, Lkv, seed=k + B, pad_from=max(1, k - 5))
    idx[0, 0, 3] = -1
    scale = 1 / math.sqrt(576)
    ws = torch.empty(ic.ic_attn_workspace_size(B, R, 16, 512, k) // 4 + 1, device=DEV)
    assert ws.numel() > 1
    lse = torch.empty(B, R, 16, device=DEV)
    out = ic.ic_sparse_attn(q.to(DEV), kv.to(DEV), torch.from_numpy(idx).to(DEV), scale, lse=lse,
                            workspace=ws)
    _sync()
    ro, rl = oracle.sparse_attn(q.float().numpy(), kv.float().numpy(), idx, scale, dv=512)
    assert_attn_close(_np(out), ro)
    np.testing.assert_allclose(lse.cpu().numpy(), rl, atol=2e-3, rtol=1e-3)


def test_attn_f32_mqa_parity():
    wl = synth.WORKLOADS["tiny_stack"]
    a = synth.attn_inputs(wl, 1)
    idx = _rand_idx(1, wl.L, wl.k, wl.L, seed=4)[0]
    idx[:10, 3:] = -1
    out = ic.ic_sparse_attn(a["q"].to(DEV), a["kv"].to(DEV), torch.from_numpy(idx).to(DEV),
                            wl.scale, v=a["v"].to(DEV))
    _sync()
    ro, _ = oracle.sparse_attn(a["q"].numpy(), a["kv"].numpy(), idx, wl.scale, v=a["v"].numpy())
    np.testing.assert_allclose(out.cpu().numpy(), ro, atol=1e-5, rtol=1e-4)


# ------------------------------------------------------------------------------- stacks
def _stack_layers(wl, device, rows=None):
    layers, host = [], []
    for l in range(wl.layers):
        d = synth.indexer_inputs(wl, l)
        d.update(synth.attn_inputs(wl, l))
        host.append(d)
        dd = {k: v.to(device) for k, v in d.items()}
        layers.append(dd)
    return layers, host


def _desc(wl, idx_dtype):
    return ic.make_desc(L=wl.L, k=wl.k, H=wl.H, D=wl.D, idx_dtype=idx_dtype, heads=wl.Hq,
                        dk=wl.Dk, dv=wl.Dv,
                        attn_dtype=ic.IC_F32 if wl.attn == "mqa" else ic.IC_BF16,
                        scale=wl.scale, batch=wl.batch, decode=wl.decode)


def _run_stack(wl, pattern, layers, idx_dtype, decode=False, ws_bytes=None):
    desc = _desc(wl, idx_dtype)
    dev_layers = []
    for d in layers:
        R = 1 if decode else wl.L
        shape = (wl.batch, R, wl.Hq, wl.Dv) if decode else (wl.L, wl.Hq, wl.Dv)
        e = {"q_idx": d["q_idx"], "k_idx": d["k_idx"], "w": d["w"], "q": d["q"], "kv": d["kv"],
             "v": d.get("v"), "q_scale": d.get("q_scale"), "k_scale": d.get("k_scale"),
             "out": torch.empty(shape, dtype=d["q"].dtype, device=DEV),
             "lse": torch.empty(shape[:-1], dtype=torch.float32, device=DEV)}
        dev_layers.append(e)
    nrows = wl.batch if decode else wl.L
    t_cache = torch.full((nrows, wl.k), -7, dtype=torch.int32, device=DEV)
    ws_bytes = ws_bytes or ic.ic_stack_workspace_size(desc)
    ws = torch.empty(ws_bytes // 4 + 1, device=DEV)
    fn = ic.ic_decode_step if decode else ic.ic_layer_stack
    fn(pattern, desc, dev_layers, t_cache, ws)
    _sync()
    return dev_layers, t_cache


def test_stack_tiny_f32_full_parity():
    """Tiny 4-layer F,S,S,S fp32 stack, full tensors against the oracle stack."""
    wl = synth.WORKLOADS["tiny_stack"]
    layers, host = _stack_layers(wl, DEV)
    dl, t_cache = _run_stack(wl, wl.pattern, layers, ic.IC_F32)
    ref = oracle.layer_stack(wl.pattern, [{k: v.numpy() for k, v in h.items()} for h in host],
                             wl.k, wl.scale, keep_scores=True)
    # the index set: near-ties with the k-th score only
    diffs = 0
    T = t_cache.cpu().numpy()
    for t in range(wl.L):
        diffs += check_index_row(T[t], ref[0]["scores"][t], wl.k, t + 1, atol=1e-5, rtol=1e-5)
    assert diffs <= wl.L // 20
    # attention of every layer over the GPU's own T (S layers reuse it unchanged)
    for l in range(wl.layers):
        h = host[l]
        ro, rl = oracle.sparse_attn(h["q"].numpy(), h["kv"].numpy(), T, wl.scale, v=h["v"].numpy())
        np.testing.assert_allclose(dl[l]["out"].cpu().numpy(), ro, atol=1e-5, rtol=1e-4)
        np.testing.assert_allclose(dl[l]["lse"].cpu().numpy(), rl, atol=1e-5, rtol=1e-5)


def test_stack_bf16_row_blocks_and_sharing():
    """bf16 4-layer F,S,F,S stack at L=2600 (k=2048) with a workspace of a few row
    blocks: sampled rows of T against the oracle's scores, S layers bit-identical."""
    wl = synth.variant("stack_32k", L=2600, pattern="F,S,F,S")
    layers, host = _stack_layers(wl, DEV)
    ws_bytes = 1000 * wl.L * 4                     # 1000-row blocks: ragged last block
    dl, t_cache = _run_stack(wl, wl.pattern, layers, ic.IC_BF16, ws_bytes=ws_bytes)
    T = t_cache.cpu().numpy()
    # T holds the last F layer's (layer 2's) set; compare sampled rows with the oracle
    rows = synth.sample_rows(wl.L, wl.k, 40, 1000).numpy()
    ref = oracle.indexer_scores(host[2]["q_idx"].float().numpy(), host[2]["k_idx"].float().numpy(),
                                host[2]["w"].numpy(), rows_sel=rows)
    for j, t in enumerate(rows):
        check_index_row(T[t], ref[j], wl.k, t + 1)
    # layers 2 and 3 attend over the same T; compare their outputs on the sampled rows
    for l in (2, 3):
        h = host[l]
        ro, _ = oracle.sparse_attn(h["q"][rows].float().numpy(), h["kv"].float().numpy(), T[rows],
                                   wl.scale, dv=512)
        assert_attn_close(_np(dl[l]["out"][torch.from_numpy(rows).to(DEV)]), ro)


def test_stack_e4m3_row_blocks_and_sharing():
    """The e4m3 indexer inside the prefill stack (F,S,F,S at L=2600, k=2048) with
    1000-row blocks: each block's per-row query scales are offset with its rows.
    Sampled rows of T against the oracle on the same e4m3 codes and scales; the
    attention of both layers that use T on those rows."""
    wl = synth.variant("stack_32k", L=2600, pattern="F,S,F,S")
    layers, host = _stack_layers(wl, DEV)
    for d in layers:
        d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_idx"])
        d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(d["k_idx"])
    ws_bytes = 1000 * wl.L * 4                     # 1000-row blocks: ragged last block
    dl, t_cache = _run_stack(wl, wl.pattern, layers, ic.IC_E4M3, ws_bytes=ws_bytes)
    T = t_cache.cpu().numpy()
    rows = synth.sample_rows(wl.L, wl.k, 40, 1000).numpy()  # includes the block edges
    d2 = layers[2]
    ref = oracle.indexer_scores_e4m3(d2["q_idx"].cpu().numpy(), d2["q_scale"].cpu().numpy(),
                                     d2["k_idx"].cpu().numpy(), d2["k_scale"].cpu().numpy(),
                                     d2["w"].cpu().numpy(), rows_sel=rows)
    for j, t in enumerate(rows):
        check_index_row(T[t], ref[j], wl.k, t + 1)
    for l in (2, 3):
        h = host[l]
        ro, _ = oracle.sparse_attn(h["q"][rows].float().numpy(), h["kv"].float().numpy(), T[rows],
                                   wl.scale, dv=512)
        assert_attn_close(_np(dl[l]["out"][torch.from_numpy(rows).to(DEV)]), ro)


def test_stack_rows_zigzag_pieces_equal_the_whole_stack():
    """ic_layer_stack_rows over the zig-zag row pieces of 2 ranks (run one after the
    other here) gives the whole stack's index sets bit for bit and its outputs within
    the attention tolerance."""
    from sparse_attention_indexer_sum_b200.sharding import zigzag_row_ranges
    wl = synth.variant("prefill_8k", L=2600, pattern="F,S")
    layers, _ = _stack_layers(wl, DEV)
    full, t_full = _run_stack(wl, wl.pattern, layers, ic.IC_BF16)
    desc = _desc(wl, ic.IC_BF16)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    seen = 0
    for rank in range(2):
        for r0, n in zigzag_row_ranges(wl.L, 2, rank):
            lay = [{"q_idx": d["q_idx"][r0:r0 + n], "w": d["w"][r0:r0 + n], "k_idx": d["k_idx"],
                    "q": d["q"][r0:r0 + n], "kv": d["kv"],
                    "out": torch.empty(n, wl.Hq, wl.Dv, dtype=torch.bfloat16, device=DEV),
                    "lse": torch.empty(n, wl.Hq, device=DEV)} for d in layers]
            t = torch.full((n, wl.k), -7, dtype=torch.int32, device=DEV)
            ic.ic_layer_stack_rows(wl.pattern, desc, lay, r0, n, t, ws)
            _sync()
            assert torch.equal(t, t_full[r0:r0 + n]), (rank, r0, n)
            for l in range(len(lay)):
                assert_attn_close(_np(lay[l]["out"]), _np(full[l]["out"][r0:r0 + n]))
            seen += n
    assert seen == wl.L


def test_stack_varlen_batch_matches_the_oracle_per_sequence():
    """Sequences of 300, 0, 517 and 64 tokens packed along the rows (fp32 config), in
    shared launches (one attention launch per layer for all of them): each one's index
    set and outputs match the oracle's stack on that sequence alone."""
    lens = [300, 0, 517, 64]
    pattern = "F,S,S"
    seqs = [synth.variant("tiny_stack", L=max(n, 1), pattern=pattern) for n in lens]
    per = []
    for i, (wl, n) in enumerate(zip(seqs, lens)):
        lay = []
        for l in range(wl.layers):
            d = synth.indexer_inputs(wl, l, seed=i)
            d.update(synth.attn_inputs(wl, l, seed=i))
            lay.append({k: v[:n] for k, v in d.items()})
        per.append(lay)
    wl0 = seqs[0]
    packed = []
    for l in range(wl0.layers):
        e = {k: torch.cat([p[l][k] for p in per]).to(DEV) for k in per[0][l]}
        tot = sum(lens)
        e["out"] = torch.empty(tot, wl0.Hq, wl0.Dv, device=DEV)
        e["lse"] = torch.empty(tot, wl0.Hq, device=DEV)
        packed.append(e)
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    desc = ic.make_desc(L=max(lens), k=wl0.k, H=wl0.H, D=wl0.D, idx_dtype=ic.IC_F32,
                        heads=wl0.Hq, dk=wl0.Dk, dv=wl0.Dv, attn_dtype=ic.IC_F32, scale=wl0.scale)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    t = torch.full((sum(lens), wl0.k), -7, dtype=torch.int32, device=DEV)
    ic.ic_trace_begin(256)
    ic.ic_layer_stack_varlen(pattern, desc, packed, cu, t, ws)
    _, tr = ic.ic_trace_end(256)
    _sync()
    names = [x[0] for x in tr]
    assert names.count("attn_f32") == wl0.layers, names
    assert names.count("indexer_f32") == names.count("topk") <= 2, names  # score-row blocks
    T = t.cpu().numpy()
    for i, n in enumerate(lens):
        if n == 0:
            continue
        lay = [{k: v.numpy() for k, v in d.items()} for d in per[i]]
        ref = oracle.layer_stack(pattern, lay, wl0.k, wl0.scale, keep_scores=True)
        o0, o1 = cu[i], cu[i + 1]
        Ti = T[o0:o1]
        diffs = sum(check_index_row(Ti[r], ref[0]["scores"][r], wl0.k, r + 1, atol=1e-5,
                                    rtol=1e-5) for r in range(n))
        assert diffs <= max(1, n // 20)
        for l in range(wl0.layers):
            ro, rl = oracle.sparse_attn(lay[l]["q"], lay[l]["kv"], Ti, wl0.scale, v=lay[l]["v"])
            np.testing.assert_allclose(packed[l]["out"][o0:o1].cpu().numpy(), ro, atol=1e-5,
                                       rtol=1e-4)
            np.testing.assert_allclose(packed[l]["lse"][o0:o1].cpu().numpy(), rl, atol=1e-5,
                                       rtol=1e-5)


def _varlen_mla_case(lens, pattern, fp8, seed):
    """Per-sequence bf16 MLA stack inputs (shapes of prefill_8k) for `lens`, packed
    along the rows; fp8: e4m3 indexer inputs and an fp8 latent cache."""
    wl0 = synth.variant("prefill_8k", L=max(max(lens), 1), pattern=pattern)
    per = []
    for i, n in enumerate(lens):
        wl = synth.variant("prefill_8k", L=max(n, 1), pattern=pattern)
        lay = []
        for l in range(wl.layers):
            d = synth.indexer_inputs(wl, l, seed=seed + i)
            d.update(synth.attn_inputs(wl, l, seed=seed + i))
            lay.append({k: v[:n] for k, v in d.items()})
        per.append(lay)
    packed = []
    for l in range(wl0.layers):
        e = {k: torch.cat([p[l][k] for p in per]).to(DEV) for k in per[0][l]}
        if fp8:
            e["q_idx"], e["q_scale"] = ic.ic_quant_e4m3_rows(e["q_idx"])
            e["k_idx"], e["k_scale"] = ic.ic_quant_e4m3_rows(e["k_idx"])
            e["kv"] = ic.ic_pack_kv_e4m3(e["kv"])
        tot = sum(lens)
        e["out"] = torch.empty(tot, wl0.Hq, wl0.Dv, dtype=torch.bfloat16, device=DEV)
        e["lse"] = torch.empty(tot, wl0.Hq, device=DEV)
        packed.append(e)
    dt = ic.IC_E4M3 if fp8 else ic.IC_BF16
    desc = ic.make_desc(L=wl0.L, k=wl0.k, H=wl0.H, D=wl0.D, idx_dtype=dt, heads=wl0.Hq, dk=wl0.Dk,
                        dv=wl0.Dv, attn_dtype=dt, scale=wl0.scale,
                        ld_kv=ic.KV8_ROW_BYTES if fp8 else None)
    return wl0, per, packed, desc


def _check_varlen_sequence(wl0, packed, T, o0, n, rows, fp8, pattern):
    """Sampled rows of one packed sequence: its F layers' index sets against the
    oracle's scores over the sequence's own keys, every layer's attention against the
    oracle on those rows (on the dequantised cache rows for fp8)."""
    kinds = pattern.split(",")
    seq = slice(o0, o0 + n)
    Ti = T[o0:o0 + n]
    for l, kind in enumerate(kinds):
        e = packed[l]
        if kind == "F":
            if fp8:
                ref = oracle.indexer_scores_e4m3(e["q_idx"][seq].cpu().numpy(),
                                                 e["q_scale"][seq].cpu().numpy(),
                                                 e["k_idx"][seq].cpu().numpy(),
                                                 e["k_scale"][seq].cpu().numpy(),
                                                 e["w"][seq].cpu().numpy(), rows_sel=rows)
                atol, rtol = 1e-3, 1e-3   # same e4m3 codes: only summation order differs
            else:
                ref = oracle.indexer_scores(e["q_idx"][seq].float().cpu().numpy(),
                                            e["k_idx"][seq].float().cpu().numpy(),
                                            e["w"][seq].cpu().numpy(), rows_sel=rows)
                atol, rtol = IDX_ATOL, IDX_RTOL_BF16
            for j, r in enumerate(rows):
                check_index_row(Ti[r], ref[j], wl0.k, r + 1, atol=atol, rtol=rtol)
        q = e["q"][seq][torch.from_numpy(rows).to(DEV)].float().cpu().numpy()
        if fp8:
            codes, scales, rope = _unpack_kv8(e["kv"][seq].cpu().numpy())
            ro, rl = oracle.sparse_attn_kv_e4m3(q, codes, scales, rope, Ti[rows], wl0.scale)
        else:
            ro, rl = oracle.sparse_attn(q, e["kv"][seq].float().cpu().numpy(), Ti[rows], wl0.scale,
                                        dv=512)
        got = e["out"][seq][torch.from_numpy(rows).to(DEV)]
        assert_attn_close(_np(got), ro, what="layer %d" % l)


@pytest.mark.parametrize("fp8", [False, True])
def test_stack_varlen_shared_launches(fp8):
    """bf16 / e4m3 stack over packed sequences of 300, 0, 1, 2, 517, 64, 2100, 5 and 1300
    tokens, pattern F,S: one indexer, one valid-length fill, one top-k and one
    attention launch per layer cover every sequence (the trace counts them), and each
    sequence's index sets and outputs match the oracle on that sequence alone."""
    lens = [300, 0, 1, 2, 517, 64, 2100, 5, 1300]
    pattern = "F,S"
    wl0, per, packed, desc = _varlen_mla_case(lens, pattern, fp8, seed=11)
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    # room for every packed row's scores (and valid length): one block
    ws = torch.empty(sum(lens) * (wl0.L + 1) + 64, device=DEV)
    t = torch.full((sum(lens), wl0.k), -7, dtype=torch.int32, device=DEV)
    ic.ic_trace_begin(256)
    ic.ic_layer_stack_varlen(pattern, desc, packed, cu, t, ws)
    n_launch, tr = ic.ic_trace_end(256)
    _sync()
    names = [x[0] for x in tr]
    assert names.count("topk") == 1 and names.count("fill_valid") == 1, names
    assert n_launch <= 6, names  # F: indexer, fill, top-k, attention; S: attention (+merges)
    T = t.cpu().numpy()
    for i, n in enumerate(lens):
        if n == 0:
            continue
        rows = np.unique(np.clip(np.array([0, 1, n // 2, n - 2, n - 1, 2047, 2048, 2049]), 0, n - 1))
        _check_varlen_sequence(wl0, packed, T, cu[i], n, rows, fp8, pattern)


def test_stack_varlen_many_sequences_and_small_blocks():
    """70 packed sequences of 0..180 tokens (more than one launch group) with a
    workspace of 700 score rows, so that row blocks cut through sequences: every
    sequence's index sets (all earlier tokens, k = 2048) and both layers' outputs
    match the oracle on that sequence alone."""
    g = np.random.default_rng(5)
    lens = g.integers(0, 181, size=70).tolist()
    lens[3] = 0
    lens[10] = 1
    pattern = "F,S"
    wl0, per, packed, desc = _varlen_mla_case(lens, pattern, False, seed=40)
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    ws = torch.empty((700 * wl0.L * 4 + 700 * 4) // 4 + 64, device=DEV)
    t = torch.full((sum(lens), wl0.k), -7, dtype=torch.int32, device=DEV)
    ic.ic_layer_stack_varlen(pattern, desc, packed, cu, t, ws)
    _sync()
    T = t.cpu().numpy()
    for i, n in enumerate(lens):
        if n == 0:
            continue
        rows = np.unique(np.array([0, n // 3, n - 1]))
        _check_varlen_sequence(wl0, packed, T, cu[i], n, rows, False, pattern)


def test_decode_step_parity():
    """Decode: 6 sequences x 1 token over a 3000-token context, fp8 indexer cache,
    pattern F,S: T per sequence and both layers' outputs against the oracle."""
    wl = synth.variant("decode_200k", L=3000, batch=6, pattern="F,S")
    layers, host = _stack_layers(wl, DEV)
    for d in layers:
        d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_idx"])
        d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(d["k_idx"])
    dl, t_cache = _run_stack(wl, wl.pattern, layers, ic.IC_E4M3, decode=True)
    T = t_cache.cpu().numpy()
    d0 = layers[0]
    ref = oracle.indexer_scores_e4m3(d0["q_idx"].cpu().numpy(), d0["q_scale"].cpu().numpy(),
                                     d0["k_idx"].cpu().numpy(), d0["k_scale"].cpu().numpy(),
                                     d0["w"].cpu().numpy(), pos0=wl.L - 1)
    for b in range(wl.batch):
        check_index_row(T[b], ref[b, 0], wl.k, wl.L)
    for l in range(2):
        h = host[l]
        ro, _ = oracle.sparse_attn(h["q"].float().numpy(), h["kv"].float().numpy(), T[:, None, :],
                                   wl.scale, dv=512)
        assert_attn_close(_np(dl[l]["out"]), ro)


def test_decode_step_fp8_kv_cache():
    """Decode over an fp8 latent cache (e4m3 indexer cache too), pattern F,S,S: T
    against the oracle's scores, every layer's output against the oracle on the
    dequantised cache rows."""
    wl = synth.variant("decode_200k", L=4500, batch=5, pattern="F,S,S")
    layers, host = _stack_layers(wl, DEV)
    for d in layers:
        d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_idx"])
        d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(d["k_idx"])
        d["kv"] = ic.ic_pack_kv_e4m3(d["kv"])
    desc = ic.make_desc(L=wl.L, k=wl.k, H=wl.H, D=wl.D, idx_dtype=ic.IC_E4M3, heads=wl.Hq,
                        dk=wl.Dk, dv=wl.Dv, attn_dtype=ic.IC_E4M3, scale=wl.scale,
                        ld_kv=ic.KV8_ROW_BYTES, batch=wl.batch, decode=True)
    dl = []
    for d in layers:
        e = dict(d)
        e["out"] = torch.empty(wl.batch, 1, wl.Hq, wl.Dv, dtype=torch.bfloat16, device=DEV)
        e["lse"] = torch.empty(wl.batch, 1, wl.Hq, device=DEV)
        dl.append(e)
    t_cache = torch.full((wl.batch, wl.k), -7, dtype=torch.int32, device=DEV)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    ic.ic_decode_step(wl.pattern, desc, dl, t_cache, ws)
    _sync()
    T = t_cache.cpu().numpy()
    d0 = layers[0]
    ref = oracle.indexer_scores_e4m3(d0["q_idx"].cpu().numpy(), d0["q_scale"].cpu().numpy(),
                                     d0["k_idx"].cpu().numpy(), d0["k_scale"].cpu().numpy(),
                                     d0["w"].cpu().numpy(), pos0=wl.L - 1)
    for b in range(wl.batch):
        check_index_row(T[b], ref[b, 0], wl.k, wl.L)
    for l in range(3):
        codes, scales, rope = _unpack_kv8(dl[l]["kv"].cpu().numpy())
        ro, rl = oracle.sparse_attn_kv_e4m3(host[l]["q"].float().numpy(), codes, scales, rope,
                                            T[:, None, :], wl.scale)
        assert_attn_close(_np(dl[l]["out"]), ro)
        np.testing.assert_allclose(dl[l]["lse"].cpu().numpy(), rl, atol=2e-3, rtol=1e-3)


def test_decode_step_two_full_layers_overwrite_t_cache():
    """Decode with pattern F,F,S: the second F layer overwrites T_cache, so the final
    T is layer 1's index set (checked against the oracle's scores of layer 1), and
    layer 0 attended over layer 0's own set."""
    wl = synth.variant("decode_200k", L=2500, batch=4, pattern="F,F,S")
    layers, host = _stack_layers(wl, DEV)
    for d in layers:
        d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_idx"])
        d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(d["k_idx"])
    dl, t_cache = _run_stack(wl, wl.pattern, layers, ic.IC_E4M3, decode=True)
    T = t_cache.cpu().numpy()
    refs = []
    for l in (0, 1):
        d = layers[l]
        refs.append(oracle.indexer_scores_e4m3(d["q_idx"].cpu().numpy(), d["q_scale"].cpu().numpy(),
                                               d["k_idx"].cpu().numpy(), d["k_scale"].cpu().numpy(),
                                               d["w"].cpu().numpy(), pos0=wl.L - 1))
    for b in range(wl.batch):
        check_index_row(T[b], refs[1][b, 0], wl.k, wl.L)
    # layer 0's own set, from the oracle's layer-0 scores: its attention used that set
    T0 = oracle.topk(refs[0][:, 0, :].astype(np.float32), wl.k)
    for l, Tl in ((0, T0), (1, T), (2, T)):
        h = host[l]
        ro, _ = oracle.sparse_attn(h["q"].float().numpy(), h["kv"].float().numpy(), Tl[:, None, :],
                                   wl.scale, dv=512)
        assert_attn_close(_np(dl[l]["out"]), ro)


def test_decode_step_graph_replay_matches_eager():
    """The decode step captured in a CUDA graph (programmatic launch edges
    included) and replayed gives bit-identical T and outputs to eager calls, also
    after its inputs change in place."""
    wl = synth.variant("decode_200k", L=5000, batch=5, pattern="F,S,S")
    layers, _ = _stack_layers(wl, DEV)
    for d in layers:
        d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_idx"])
        d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(d["k_idx"])
    dl, t_eager = _run_stack(wl, wl.pattern, layers, ic.IC_E4M3, decode=True)
    out_eager = [d["out"].clone() for d in dl]
    desc = _desc(wl, ic.IC_E4M3)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    t_cache = torch.full_like(t_eager, -7)
    for d in dl:
        d["out"].zero_()
    g = ic.decode_step_graph(wl.pattern, desc, dl, t_cache, ws, warmup=0)
    g.replay()
    _sync()
    assert torch.equal(t_cache, t_eager)
    for d, o in zip(dl, out_eager):
        assert torch.equal(d["out"], o)
    # new queries written in place: the replay follows them like an eager call
    for d in dl:
        d["q"].copy_(torch.flip(d["q"], dims=[0]))
        d["q_idx"].copy_(torch.flip(d["q_idx"], dims=[0]))
        d["q_scale"].copy_(torch.flip(d["q_scale"], dims=[0]))
        d["w"].copy_(torch.flip(d["w"], dims=[0]))
    g.replay()
    _sync()
    t_graph = t_cache.clone()
    out_graph = [d["out"].clone() for d in dl]
    ic.ic_decode_step(wl.pattern, desc, dl, t_cache, ws)
    _sync()
    assert torch.equal(t_cache, t_graph)
    for d, o in zip(dl, out_graph):
        assert torch.equal(d["out"], o)
    assert not torch.equal(t_graph, t_eager)
    del g


# ------------------------------------------------------------------ fused indexer -> top-k
def _fused_vs_unfused(q, k, w, pos0, k_top, q_scale=None, k_scale=None):
    B, Lk = k.shape[0], k.shape[1]
    ws = torch.empty(ic.ic_indexer_topk_workspace_size(B, Lk, pos0) // 4 + 4, device=DEV)
    got = ic.ic_indexer_topk(q, k, w, k_top, ws, pos0=pos0, q_scale=q_scale, k_scale=k_scale)
    scores = ic.ic_indexer_scores(q, k, w, pos0=pos0, q_scale=q_scale, k_scale=k_scale)
    ref = ic.ic_topk(scores.view(B, Lk), k_top, pos0=pos0)
    _sync()
    assert torch.equal(got, ref)
    return got, scores


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
@pytest.mark.parametrize("B,Lk,pos0,k_top", [(6, 5000, 4999, 2048), (64, 30000, 29999, 2048),
                                             (3, 20000, 11000, 2048), (2, 1500, 1499, 2048),
                                             (5, 9000, 8999, 100), (1, 60000, 59999, 1),
                                             (4, 2100, 2047, 2048)])
def test_indexer_topk_fused_equals_scores_then_topk(fp8, B, Lk, pos0, k_top):
    """The fused indexer -> top-k selects exactly what ic_topk selects on the scores
    ic_indexer_scores writes for the same inputs (one query per sequence): many CTA
    pieces per row (B = 1..6), several rows per CTA (B = 64), masked keys past pos0,
    rows with fewer candidates than k, k = 1 and k = 100."""
    q, k, w = _idx_inputs(B, 1, Lk, seed=B * 7 + Lk)
    q, k, w = q.to(DEV), k.to(DEV), w.to(DEV)
    qs = ks = None
    if fp8:
        q, qs = ic.ic_quant_e4m3_rows(q)
        k, ks = ic.ic_quant_e4m3_rows(k)
    got, scores = _fused_vs_unfused(q, k, w, pos0, k_top, qs, ks)
    # and the oracle's top-k on those scores, as for ic_topk
    ref = oracle.topk(scores.view(B, Lk).cpu().numpy(), k_top,
                      valid=np.full(B, min(Lk, pos0 + 1), np.int32))
    np.testing.assert_array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
def test_indexer_topk_fused_repeatable(fp8):
    """Ten calls in a row on a shape with several compactions per epilogue set and
    rows split over CTAs: every call selects exactly what ic_topk selects."""
    B, Lk = 64, 30000
    q, k, w = _idx_inputs(B, 1, Lk, seed=99)
    q, k, w = q.to(DEV), k.to(DEV), w.to(DEV)
    qs = ks = None
    if fp8:
        q, qs = ic.ic_quant_e4m3_rows(q)
        k, ks = ic.ic_quant_e4m3_rows(k)
    scores = ic.ic_indexer_scores(q, k, w, pos0=Lk - 1, q_scale=qs, k_scale=ks)
    ref = ic.ic_topk(scores.view(B, Lk), 2048, pos0=Lk - 1)
    ws = torch.empty(ic.ic_indexer_topk_workspace_size(B, Lk, Lk - 1) // 4 + 4, device=DEV)
    for _ in range(10):
        ws.fill_(float("nan"))   # leftovers must not matter
        got = ic.ic_indexer_topk(q, k, w, 2048, ws, pos0=Lk - 1, q_scale=qs, k_scale=ks)
        _sync()
        assert torch.equal(got, ref)


def test_indexer_topk_fused_ties():
    """Tied scores: all zero (queries 0), every head dead (negated queries over keys
    with positive dots) and four distinct values; the lowest indices win."""
    B, Lk = 4, 40000
    g = torch.Generator().manual_seed(5)
    k = torch.rand(B, Lk, 128, generator=g).to(torch.bfloat16).to(DEV)      # k >= 0
    w = torch.rand(B, 1, 64, generator=g).to(DEV)
    q0 = torch.zeros(B, 1, 64, 128, dtype=torch.bfloat16, device=DEV)
    qneg = (-torch.rand(B, 1, 64, 128, generator=g)).to(torch.bfloat16).to(DEV)
    for q in (q0, qneg):
        got, _ = _fused_vs_unfused(q, k, w, Lk - 1, 2048)
        assert torch.equal(got, torch.arange(2048, device=DEV, dtype=torch.int32).expand(B, -1))
    # four distinct scores: keys are one of four vectors along one direction
    u = torch.zeros(128)
    u[0] = 1.0
    kk = (torch.randint(0, 4, (B, Lk, 1), generator=g).float() * u).to(torch.bfloat16).to(DEV)
    qq = torch.zeros(B, 1, 64, 128)
    qq[..., 0] = 1.0
    _fused_vs_unfused(qq.to(torch.bfloat16).to(DEV), kk, w, Lk - 1, 2048)


def test_decode_step_fused_equals_unfused_top_k():
    """ic_decode_step writes the scores and runs ic_topk by default; with
    IC_STACK_FUSED_TOPK it fuses the indexer and the top-k.  Same T and outputs, bit
    for bit."""
    wl = synth.variant("decode_200k", L=7000, batch=9, pattern="F,S,F")
    layers, _ = _stack_layers(wl, DEV)
    for d in layers:
        d["q_idx"], d["q_scale"] = ic.ic_quant_e4m3_rows(d["q_idx"])
        d["k_idx"], d["k_scale"] = ic.ic_quant_e4m3_rows(d["k_idx"])
    dl, t_fused = _run_stack(wl, wl.pattern, layers, ic.IC_E4M3, decode=True)
    outs = [d["out"].clone() for d in dl]
    desc = _desc(wl, ic.IC_E4M3)
    desc.flags = ic.IC_STACK_FUSED_TOPK
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    t_unf = torch.full_like(t_fused, -7)
    ic.ic_decode_step(wl.pattern, desc, dl, t_unf, ws)
    _sync()
    assert torch.equal(t_fused, t_unf)
    for d, o in zip(dl, outs):
        assert torch.equal(d["out"], o)


def test_trace_records_every_launch_in_order():
    q, k, w = _idx_inputs(1, 8, 300, seed=3)
    q, k, w = q.to(DEV), k.to(DEV), w.to(DEV)
    ic.ic_indexer_scores(q, k, w, pos0=100)      # warm up (attributes, tensor maps)
    _sync()
    ic.ic_trace_begin(16)
    s = ic.ic_indexer_scores(q, k, w, pos0=100)
    ic.ic_topk(s[0], 64, pos0=100)
    n, tr = ic.ic_trace_end(16)
    assert n == 3
    assert [t[0] for t in tr] == ["indexer_tc_bf16", "fill_masked", "topk"]
    assert all(ms > 0 for _, ms, _ in tr)
    assert tr[0][2] == 2.0 * 64 * 128 * sum(min(300, 100 + r + 1) for r in range(8))
