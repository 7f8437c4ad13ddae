"""Pins of the CPU oracle against what the pages and the mathematics fix.

No test here re-types an oracle formula: each one checks the oracle against a
hand-worked fixture (tests/golden/), a closed form, a special case that reduces
to a library routine, brute force by a different algorithm on tiny inputs, or
an invariant the pages state.  Pages cited: "IndexCache: Wie DeepSeek
O(NL^2)-Kosten in Sparse Attention um 75% reduziert" (itoverdose.com) for the
routing loop, the F/S rules, k and the score -> ReLU -> top-k shape; the
parapluman.nl article ("Aandacht cachen met IndexCache") for "S reuses the
nearest preceding F".
"""
import heapq
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_indexer_sum_b200 import synth

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLD, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln


# ------------------------------------------------------------------------------ e4m3
def test_e4m3_decode_matches_spec_table():
    n = 0
    for ln in _lines("e4m3_codes.txt"):
        code, val = ln.split()
        got = oracle.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val), (code, got, val)
            assert math.copysign(1.0, got) == math.copysign(1.0, float(val))
        n += 1
    assert n >= 15


def test_e4m3_all_codes_monotone_and_roundtrip():
    vals = [oracle.e4m3_decode(c) for c in range(0x7F)]  # 0x00..0x7E finite, non-negative
    assert all(a < b for a, b in zip(vals, vals[1:]))
    assert vals[-1] == 448.0
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(v):
            assert c in (0x7F, 0xFF)
            continue
        assert oracle.e4m3_encode(v) == c


def test_e4m3_rne_midpoints_and_saturation():
    # midpoints between neighbours go to the even mantissa
    assert oracle.e4m3_encode(1.0625) == 0x38      # between 1 (m=0) and 1.125 (m=1)
    assert oracle.e4m3_encode(1.1875) == 0x3A      # between 1.125 (m=1) and 1.25 (m=2)
    assert oracle.e4m3_encode(1.0625 + 1e-9) == 0x39
    assert oracle.e4m3_encode(2 ** -10) == 0x00    # half the smallest subnormal -> 0 (even)
    assert oracle.e4m3_encode(3 * 2 ** -10) == 0x02  # between 1 and 2 subnormal steps -> 2
    assert oracle.e4m3_encode(-1.0625) == 0xB8
    assert oracle.e4m3_encode(464.0) == 0x7E        # saturate (finite max 448)
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE


def test_e4m3_matches_torch_cast_in_range():
    # special case reducing to a library routine: in range, torch's float8_e4m3fn cast
    # is round-to-nearest-even onto the same grid
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(20000, generator=g, dtype=torch.float64) * 60).clamp(-440, 440)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x.tolist()], dtype=np.uint8)
    np.testing.assert_array_equal(got, ref)


def test_quant_rows_e4m3_scale_and_amax_code():
    g = torch.Generator().manual_seed(2)
    x = torch.randn(37, 128, generator=g).numpy().astype(np.float32)
    x[5] = 0.0
    codes, scales = oracle.quant_rows_e4m3(x)
    amax = np.abs(x).max(axis=1)
    np.testing.assert_array_equal(scales[amax > 0], (amax[amax > 0] / np.float32(448)).astype(np.float32))
    assert scales[5] == 1.0 and (codes[5] == 0).all()
    for r in range(37):
        if amax[r] == 0:
            continue
        j = int(np.abs(x[r]).argmax())
        assert codes[r, j] & 0x7F == 0x7E            # the amax element lands on 448
    deq = oracle.dequant_rows_e4m3(codes, scales)
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range
    big = np.abs(x) > scales[:, None] * 2 ** -6
    assert (np.abs(deq - x)[big] <= np.abs(x)[big] * 2 ** -4 + 1e-12).all()


# ------------------------------------------------------------------------------ indexer
def _read_indexer_fixture():
    L = H = D = None
    k, q, w, I, T = {}, {}, {}, {}, {}
    for ln in _lines("indexer_tiny.txt"):
        p = ln.split()
        if p[0] in ("L", "H", "D"):
            v = int(p[1])
            if p[0] == "L":
                L = v
            elif p[0] == "H":
                H = v
            else:
                D = v
        elif p[0] == "k":
            k[int(p[1])] = [float(x) for x in p[2:]]
        elif p[0] == "q":
            q[(int(p[1]), int(p[2]))] = [float(x) for x in p[3:]]
        elif p[0] == "w":
            w[int(p[1])] = [float(x) for x in p[2:]]
        elif p[0] == "I":
            I[int(p[1])] = [float(x) for x in p[2:]]
        elif p[0] == "T":
            T[int(p[1])] = [int(x) for x in p[2:]]
    qa = np.array([[q[(t, h)] for h in range(H)] for t in range(L)])
    ka = np.array([k[s] for s in range(L)])
    wa = np.array([w[t] for t in range(L)])
    Ia = np.array([I[t] for t in range(L)])
    Ta = np.array([T[t] for t in range(L)], dtype=np.int32)
    return qa, ka, wa, Ia, Ta


def test_indexer_golden_hand_worked():
    q, k, w, I, T = _read_indexer_fixture()
    got = oracle.indexer_scores(q, k, w)
    np.testing.assert_array_equal(got, I)
    Tg = oracle.topk(got.astype(np.float32), 2, valid=oracle.causal_valid(3, 0, 3))
    np.testing.assert_array_equal(Tg, T)


def test_indexer_single_head_unit_weight_is_relu_gemm():
    # H = 1, w = 1: I = ReLU(Q K^T) below the diagonal (numpy matmul as the library routine)
    g = np.random.default_rng(3)
    L, D = 40, 16
    q = g.standard_normal((L, 1, D))
    k = g.standard_normal((L, D))
    w = np.ones((L, 1))
    got = oracle.indexer_scores(q, k, w)
    ref = np.maximum(q[:, 0, :] @ k.T, 0.0)
    tri = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(got[tri], ref[tri], rtol=1e-12, atol=1e-12)
    assert np.isneginf(got[~tri]).all()


def test_indexer_nonnegative_inputs_reduce_to_gemv():
    # q >= 0 and k >= 0 make every gate the identity: I[t,s] = (sum_h w[t,h] q[t,h]) . k[s]
    g = np.random.default_rng(4)
    L, H, D = 33, 5, 8
    q = np.abs(g.standard_normal((L, H, D)))
    k = np.abs(g.standard_normal((L, D)))
    w = g.uniform(0, 1, (L, H))
    got = oracle.indexer_scores(q, k, w)
    qw = np.einsum("th,thd->td", w, q)
    ref = qw @ k.T
    tri = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(got[tri], ref[tri], rtol=1e-12)


def test_indexer_rank_one_closed_form_catches_transposes():
    # q[t,h] = a[t,h] u, k[s] = b[s] u, |u| = 1  =>  I[t,s] = sum_h w[t,h] max(0, a[t,h] b[s])
    g = np.random.default_rng(5)
    L, H, D = 17, 3, 6
    u = g.standard_normal(D)
    u /= np.linalg.norm(u)
    a = g.standard_normal((L, H))
    b = g.standard_normal(L) * np.arange(1, L + 1)       # scale grows with s: asymmetric
    w = g.uniform(0, 1, (L, H)) * np.arange(1, L + 1)[:, None]
    got = oracle.indexer_scores(a[:, :, None] * u, b[:, None] * u, w)
    for t in range(L):
        for s in range(L):
            if s > t:
                assert got[t, s] == -np.inf
            else:
                ref = sum(w[t, h] * max(0.0, a[t, h] * b[s]) for h in range(H))
                assert abs(got[t, s] - ref) <= 1e-12 * (1 + abs(ref))


def test_indexer_zero_weights_dead_heads_and_nonnegativity():
    g = np.random.default_rng(6)
    L, H, D = 25, 4, 8
    q = g.standard_normal((L, H, D))
    k = g.standard_normal((L, D))
    w = g.uniform(0, 1, (L, H))
    tri = np.tril(np.ones((L, L), dtype=bool))
    assert (oracle.indexer_scores(q, k, np.zeros_like(w))[tri] == 0).all()
    I = oracle.indexer_scores(q, k, w)
    assert (I[tri] >= 0).all()                       # ReLU gate with w >= 0
    # all dots positive -> negating q kills every head
    qp = np.abs(q)
    kp = np.abs(k) + 0.1
    assert (oracle.indexer_scores(qp, kp, w)[tri] > 0).all()
    assert (oracle.indexer_scores(-qp, kp, w)[tri] == 0).all()


def test_indexer_rows_sel_batch_and_pos0():
    g = np.random.default_rng(7)
    B, R, H, D, Lk = 2, 6, 3, 4, 10
    q = g.standard_normal((B, R, H, D))
    k = g.standard_normal((B, Lk, D))
    w = g.uniform(0, 1, (B, R, H))
    full = oracle.indexer_scores(q, k, w, pos0=4)
    sel = oracle.indexer_scores(q, k, w, pos0=4, rows_sel=[5, 0, 3])
    np.testing.assert_array_equal(sel, full[:, [5, 0, 3]])
    for r in range(R):
        assert np.isfinite(full[:, r, : 4 + r + 1]).all() and np.isneginf(full[:, r, 4 + r + 1:]).all()
    # batch b uses its own keys: shuffling batch 1's keys leaves batch 0 alone
    k2 = k.copy()
    k2[1] = k2[1, ::-1]
    np.testing.assert_array_equal(oracle.indexer_scores(q, k2, w, pos0=4)[0], full[0])


def test_indexer_scores_at_positions_map_to_causal_rows():
    # Rows scored one by one at arbitrary positions p_j must equal rows p_j of the
    # whole causal matrix (the pinned rows_sel path) and the rank-one closed form.
    g = np.random.default_rng(17)
    L, H, D = 23, 3, 5
    u = g.standard_normal(D)
    u /= np.linalg.norm(u)
    a = g.standard_normal((L, H))
    b = g.standard_normal(L) * np.arange(1, L + 1)
    w = g.uniform(0, 1, (L, H)) * np.arange(1, L + 1)[:, None]
    q, k = a[:, :, None] * u, b[:, None] * u
    pos = np.array([22, 0, 7, 8, 21, 3])              # unsorted, first and last rows
    got = oracle.indexer_scores_at(q[pos], k, w[pos], pos, nthreads=3)
    np.testing.assert_array_equal(got, oracle.indexer_scores(q, k, w, rows_sel=pos))
    for j, p in enumerate(pos):
        assert np.isneginf(got[j, p + 1:]).all()
        for s in range(p + 1):
            ref = sum(w[p, h] * max(0.0, a[p, h] * b[s]) for h in range(H))
            assert abs(got[j, s] - ref) <= 1e-12 * (1 + abs(ref))
    # an off-by-one in the position mapping would unmask key p + 1 or mask key p
    assert np.isfinite(got[:, 0]).all()


def test_indexer_e4m3_is_definition_on_dequantised_values():
    # integer-valued codes with unit scales: the e4m3 indexer equals exact integer arithmetic
    q_codes = np.zeros((4, 2, 4), dtype=np.uint8)
    k_codes = np.zeros((4, 4), dtype=np.uint8)
    enc = {v: oracle.e4m3_encode(v) for v in (-2.0, -1.0, 0.0, 1.0, 2.0, 3.0)}
    g = np.random.default_rng(8)
    qv = g.choice([-2.0, -1.0, 0.0, 1.0, 2.0, 3.0], size=(4, 2, 4))
    kv = g.choice([-2.0, -1.0, 0.0, 1.0, 2.0, 3.0], size=(4, 4))
    for i, v in np.ndenumerate(qv):
        q_codes[i] = enc[v]
    for i, v in np.ndenumerate(kv):
        k_codes[i] = enc[v]
    w = np.array([[1.0, 2.0]] * 4)
    got = oracle.indexer_scores_e4m3(q_codes, np.ones((4, 2), np.float32), k_codes,
                                     np.ones(4, np.float32), w)
    for t in range(4):
        for s in range(t + 1):
            ref = sum(w[t, h] * max(0.0, float(np.dot(qv[t, h], kv[s]))) for h in range(2))
            assert got[t, s] == ref
    # scales multiply through: k_scale 2 on every key doubles every score
    got2 = oracle.indexer_scores_e4m3(q_codes, np.ones((4, 2), np.float32), k_codes,
                                      np.full(4, 2.0, np.float32), w)
    tri = np.tril(np.ones((4, 4), dtype=bool))
    np.testing.assert_array_equal(got2[tri], 2 * got[tri])


# ------------------------------------------------------------------------------ top-k
def _brute_topk(row, k, valid):
    """Repeated selection with a heap -- a different algorithm from the oracle's sort."""
    cand = [(-float(row[s]) + 0.0, s) for s in range(valid)]   # + 0.0 folds -0 into +0
    best = heapq.nsmallest(min(k, valid), cand)
    out = sorted(s for _, s in best)
    return out + [-1] * (k - len(out))


def test_topk_golden_rows():
    n = 0
    for ln in _lines("topk_small.txt"):
        head, sc, ex = [p.strip() for p in ln.split("|")]
        k, valid = (int(x) for x in head.split())
        scores = np.array([float(x) for x in sc.split()], dtype=np.float32)
        exp = [int(x) for x in ex.split()]
        got = oracle.topk(scores, k, valid=valid)
        assert got.tolist() == exp, (ln, got)
        n += 1
    assert n >= 10


def test_topk_brute_force_tiny_with_ties():
    g = np.random.default_rng(9)
    for trial in range(300):
        n = int(g.integers(1, 40))
        k = int(g.integers(1, 20))
        valid = int(g.integers(0, n + 1))
        row = g.choice([-1.0, -0.0, 0.0, 0.5, 1.0, 2.0], size=n).astype(np.float32)
        got = oracle.topk(row, k, valid=valid)
        assert got.tolist() == _brute_topk(row, k, valid), (row, k, valid)


def test_topk_invariants_random_rows():
    g = np.random.default_rng(10)
    rows, n, k = 64, 3000, 257
    s = g.standard_normal((rows, n)).astype(np.float32)
    valid = g.integers(0, n + 1, rows).astype(np.int32)
    T = oracle.topk(s, k, valid=valid)
    for r in range(rows):
        m = min(k, int(valid[r]))
        sel = T[r, :m]
        assert (T[r, m:] == -1).all()
        assert (np.diff(sel) > 0).all()                      # ascending, distinct
        assert ((sel >= 0) & (sel < valid[r])).all()
        if m < valid[r]:
            rest = np.setdiff1d(np.arange(valid[r]), sel)
            assert s[r, sel].min() >= s[r, rest].max()
        assert sel.tolist() == _brute_topk(s[r], k, int(valid[r]))[:m]


def test_topk_special_rows():
    k = 8
    assert oracle.topk(np.full(20, 3.0, np.float32), k).tolist() == list(range(8))
    dec = np.arange(20, 0, -1).astype(np.float32)
    assert oracle.topk(dec, k).tolist() == list(range(8))
    assert oracle.topk(dec[::-1].copy(), k).tolist() == list(range(12, 20))
    assert oracle.topk(np.zeros(8, np.float32), k).tolist() == list(range(8))     # n == k
    row = np.ones(9, np.float32)
    row[4] = -1
    assert oracle.topk(row, k).tolist() == [0, 1, 2, 3, 5, 6, 7, 8]                # n == k + 1
    assert oracle.topk(np.ones(3, np.float32), k).tolist() == [0, 1, 2] + [-1] * 5  # n < k


# ------------------------------------------------------------------------------ attention
def _read_attn_fixture():
    d = {"kv": []}
    for ln in _lines("attn_tiny.txt"):
        p = ln.split()
        if p[0] == "kv":
            d["kv"].append([float(x) for x in p[1:]])
        else:
            d[p[0]] = [float(x) for x in p[1:]]
    return d


def test_attn_golden_hand_worked():
    d = _read_attn_fixture()
    q = np.array(d["q"])[None, None, :]
    kv = np.array(d["kv"])
    idx = np.array(d["idx"], dtype=np.int32)[None, :]
    out, lse = oracle.sparse_attn(q, kv, idx, 1.0, dv=2)
    np.testing.assert_allclose(out[0, 0], d["out"], rtol=1e-15, atol=1e-16)
    np.testing.assert_allclose(lse[0, 0], d["lse"][0], rtol=1e-15)
    # the closed form written out: (e, 1) / (1 + 2e)
    e = math.e
    np.testing.assert_allclose(out[0, 0], [e / (1 + 2 * e), 1 / (1 + 2 * e)], rtol=1e-15)


def test_kv_e4m3_pack_groups_and_rope():
    # each 128-dim latent group has its own scale (amax / 448), so a group of small
    # values keeps its precision next to a group of large ones; rope is untouched
    g = np.random.default_rng(21)
    kv = g.standard_normal((5, 576)).astype(np.float32)
    kv[:, 128:256] *= 1e-3
    kv[2, 256:384] = 0.0
    codes, scales, rope = oracle.kv_pack_e4m3(kv)
    assert codes.shape == (5, 512) and scales.shape == (5, 4) and rope.shape == (5, 64)
    for gi in range(4):
        amax = np.abs(kv[:, 128 * gi:128 * (gi + 1)]).max(axis=1)
        want = np.where(amax > 0, (amax / np.float32(448)).astype(np.float32), 1.0)
        np.testing.assert_array_equal(scales[:, gi], want.astype(np.float32))
    np.testing.assert_array_equal(rope, kv[:, 512:])
    deq = oracle.kv_dequant_e4m3(codes, scales, rope)
    # 3 mantissa bits: relative error at most 2^-4 of the group's amax-scaled grid
    for gi in range(4):
        sl = slice(128 * gi, 128 * (gi + 1))
        err = np.abs(deq[:, sl] - kv[:, sl])
        assert (err <= np.abs(kv[:, sl]) * 2.0 ** -4 + scales[:, gi:gi + 1] * 2.0 ** -9).all()
    np.testing.assert_array_equal(deq[:, 512:], kv[:, 512:])
    assert (deq[2, 256:384] == 0).all()


def test_kv_e4m3_attention_hand_worked():
    # the hand-worked example of attn_tiny.txt, carried by an fp8 cache: latent dims
    # 0..2 hold the example's rows (exact e4m3 values with unit scales), the rest 0
    d = _read_attn_fixture()
    rows = np.zeros((4, 576), dtype=np.float64)
    rows[:, :3] = np.array(d["kv"])
    codes = np.zeros((4, 512), dtype=np.uint8)
    for r in range(4):
        for c in range(3):
            codes[r, c] = oracle.e4m3_encode(rows[r, c])
    scales = np.ones((4, 4), dtype=np.float32)
    rope = np.zeros((4, 64), dtype=np.float32)
    q = np.zeros((1, 1, 576))
    q[0, 0, :3] = d["q"]
    idx = np.array(d["idx"], dtype=np.int32)[None, :]
    out, lse = oracle.sparse_attn_kv_e4m3(q, codes, scales, rope, idx, 1.0)
    e = math.e
    # values are the first 512 latent dims: dim 2 carries row 2's 0.5 as well
    np.testing.assert_allclose(out[0, 0, :3], [e / (1 + 2 * e), 1 / (1 + 2 * e),
                                               0.5 * e / (1 + 2 * e)], rtol=1e-15)
    assert (out[0, 0, 3:] == 0).all()
    np.testing.assert_allclose(lse[0, 0], d["lse"][0], rtol=1e-15)
    # a group scale of 2 doubles that group's values: logits of q on group 0 double
    out2, lse2 = oracle.sparse_attn_kv_e4m3(q, codes, scales * 2, rope, idx, 0.5)
    np.testing.assert_allclose(out2[0, 0, :2], 2 * out[0, 0, :2], rtol=1e-14)
    # rope dims take part in the logits but not in the values
    rope2 = rope.copy()
    rope2[1, 0] = 1.0
    q2 = q.copy()
    q2[0, 0, 512] = math.log(3.0)
    out3, _ = oracle.sparse_attn_kv_e4m3(q2, codes, scales, rope2, idx, 1.0)
    w = np.array([1.0, 3 * e, e])   # rows 0, 1, 2: z = 0, 1 + log 3, 1
    want = (w[1] * np.array([1, 0]) + w[0] * np.array([0, 1])) / w.sum()
    np.testing.assert_allclose(out3[0, 0, :2], want, rtol=1e-14)


def test_attn_single_index_returns_that_value_row():
    g = np.random.default_rng(11)
    R, H, Dk, Dv, L, k = 5, 3, 12, 8, 20, 6
    q = g.standard_normal((R, H, Dk))
    kv = g.standard_normal((L, Dk))
    idx = np.full((R, k), -1, np.int32)
    js = g.integers(0, L, R)
    for r in range(R):
        idx[r, r % k] = js[r]
    out, lse = oracle.sparse_attn(q, kv, idx, 0.3, dv=Dv)
    for r in range(R):
        for h in range(H):
            np.testing.assert_array_equal(out[r, h], kv[js[r], :Dv])
            assert abs(lse[r, h] - 0.3 * float(q[r, h] @ kv[js[r]])) < 1e-12


def test_attn_equal_logits_give_mean_of_values():
    g = np.random.default_rng(12)
    R, H, Dk, Dv, L, k = 4, 2, 10, 7, 30, 9
    q = np.zeros((R, H, Dk))
    v = g.standard_normal((L, Dv))
    kv = g.standard_normal((L, Dk))
    idx = np.stack([g.permutation(L)[:k] for _ in range(R)]).astype(np.int32)
    out, lse = oracle.sparse_attn(q, kv, idx, 1.0, v=v)
    for r in range(R):
        np.testing.assert_allclose(out[r, 0], v[idx[r]].mean(axis=0), rtol=1e-12, atol=1e-14)
        assert abs(lse[r, 0] - math.log(k)) < 1e-12


def test_attn_full_index_set_is_dense_causal_attention():
    # T = every s <= t (k >= L) reduces to textbook causal softmax attention (torch, fp64)
    g = np.random.default_rng(13)
    L, H, Dk, Dv = 24, 3, 16, 16
    q = g.standard_normal((L, H, Dk))
    kv = g.standard_normal((L, Dk))
    v = g.standard_normal((L, Dv))
    idx = np.full((L, L), -1, np.int32)
    for t in range(L):
        idx[t, : t + 1] = np.arange(t + 1)
    out, lse = oracle.sparse_attn(q, kv, idx, 0.25, v=v)
    qt, kt, vt = (torch.from_numpy(x) for x in (q, kv, v))
    logits = torch.einsum("thd,sd->hts", qt, kt) * 0.25
    mask = torch.triu(torch.ones(L, L, dtype=torch.bool), 1)
    logits = logits.masked_fill(mask, float("-inf"))
    ref = torch.einsum("hts,sd->thd", torch.softmax(logits, -1), vt).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1).T.numpy(), rtol=1e-12)


def test_attn_index_order_and_padding_do_not_matter():
    g = np.random.default_rng(14)
    R, H, Dk, Dv, L, k = 6, 2, 9, 5, 40, 12
    q = g.standard_normal((R, H, Dk))
    kv = g.standard_normal((L, Dk))
    idx = np.stack([g.permutation(L)[:k] for _ in range(R)]).astype(np.int32)
    o1, l1 = oracle.sparse_attn(q, kv, idx, 0.5, dv=Dv)
    perm = np.concatenate([idx[:, ::-1], np.full((R, 5), -1, np.int32)], axis=1)
    o2, l2 = oracle.sparse_attn(q, kv, perm, 0.5, dv=Dv)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-12)


def test_attn_batched_uses_own_sequence():
    g = np.random.default_rng(15)
    B, H, Dk, Dv, L, k = 3, 2, 8, 6, 50, 7
    q = g.standard_normal((B, 1, H, Dk))
    kv = g.standard_normal((B, L, Dk))
    idx = g.integers(0, L, (B, 1, k)).astype(np.int32)
    out, lse = oracle.sparse_attn(q, kv, idx, 0.4, dv=Dv)
    for b in range(B):
        o, l = oracle.sparse_attn(q[b], kv[b], idx[b], 0.4, dv=Dv)
        np.testing.assert_array_equal(out[b], o)
        np.testing.assert_array_equal(lse[b], l)


# ------------------------------------------------------------------------------ F/S stack
def test_pattern_grammar():
    assert oracle.parse_pattern("F,S,S,S") == ["F", "S", "S", "S"]
    assert oracle.parse_pattern("F S S S F S S S") == list("FSSSFSSS")
    assert oracle.parse_pattern("FSFS") == list("FSFS")
    for bad in ("", " , ", "S,F", "F,X", "f,s", "F;S"):
        with pytest.raises(ValueError):
            oracle.parse_pattern(bad)


def _tiny_layers(wl, nlayers):
    layers = []
    for l in range(nlayers):
        d = synth.indexer_inputs(wl, l)
        d.update(synth.attn_inputs(wl, l))
        layers.append({k: v.numpy() for k, v in d.items()})
    return layers


def test_stack_shared_layers_reuse_last_full_layer():
    wl = synth.variant("tiny_stack", L=96, k=16)
    layers = _tiny_layers(wl, 6)
    res = oracle.layer_stack("F,S,S,F,S,S", layers, wl.k, wl.scale)
    np.testing.assert_array_equal(res[1]["T"], res[0]["T"])
    np.testing.assert_array_equal(res[2]["T"], res[0]["T"])
    np.testing.assert_array_equal(res[4]["T"], res[3]["T"])
    np.testing.assert_array_equal(res[5]["T"], res[3]["T"])
    # an F layer recomputes from its own inputs
    allf = oracle.layer_stack("F,F,F,F,F,F", layers, wl.k, wl.scale)
    np.testing.assert_array_equal(res[3]["T"], allf[3]["T"])
    np.testing.assert_array_equal(res[0]["out"], allf[0]["out"])       # layer 1 identical
    for l in range(6):
        T = allf[l]["T"]
        for t in range(wl.L):
            m = min(wl.k, t + 1)
            assert (T[t, m:] == -1).all() and (T[t, :m] <= t).all()
            assert len(set(T[t, :m].tolist())) == m


def test_stack_layer_count_must_match():
    wl = synth.variant("tiny_stack", L=16, k=4)
    with pytest.raises(ValueError):
        oracle.layer_stack("F,S", _tiny_layers(wl, 3), wl.k, wl.scale)


def test_synth_ar1_layer_correlation():
    wl = synth.variant("tiny_stack", L=512)
    k0 = synth.indexer_inputs(wl, 0)["k_idx"].double().flatten()
    k1 = synth.indexer_inputs(wl, 1)["k_idx"].double().flatten()
    c = float(torch.corrcoef(torch.stack([k0, k1]))[0, 1])
    assert abs(c - 0.9) < 0.02
    assert abs(float(k1.std()) * math.sqrt(wl.D) - 1.0) < 0.03  # 0.9^2 + 0.436^2 ~ 1
