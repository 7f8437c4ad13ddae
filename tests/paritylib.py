"""Comparison helpers shared by the GPU parity tests (no arithmetic of the method here)."""
import numpy as np

# Tolerances of the indexer scores (bf16 and fp8 inputs) and of the attention output.
IDX_ATOL, IDX_RTOL_BF16, IDX_RTOL_FP8 = 1e-3, 1e-2, 5e-2
ATTN_MAX_ABS, ATTN_MEAN_ABS = 2e-2, 2e-3


def assert_scores_close(got, ref, atol=IDX_ATOL, rtol=IDX_RTOL_BF16, what="scores"):
    """|got - ref| <= atol + rtol |ref| on finite entries; -inf exactly where ref is -inf."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    ninf = np.isneginf(ref)
    assert (np.isneginf(got) == ninf).all(), "%s: masked entries differ" % what
    fin = ~ninf
    err = np.abs(got[fin] - ref[fin])
    lim = atol + rtol * np.abs(ref[fin])
    bad = err > lim
    assert not bad.any(), "%s: %d of %d entries out of tolerance, worst %.3g (ref %.3g)" % (
        what, bad.sum(), bad.size, err.max(), ref[fin][np.argmax(err - lim)])


def assert_fp8_scores_close_to_unquantised(got, ref, rtol=IDX_RTOL_FP8):
    """Scores from e4m3 inputs against the oracle on the unquantised inputs:
    |got - ref| <= rtol * max(|ref|, rms of the row's finite refs) on finite entries
    (the row-RMS floor keeps near-zero gated scores from dominating a relative test);
    -inf exactly where ref is -inf.  Differences are taken on finite entries only."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    fin = np.isfinite(ref)
    assert (np.isneginf(got) == ~fin).all(), "masked entries differ"
    sq = np.zeros_like(ref)
    sq[fin] = ref[fin] ** 2
    rms = np.sqrt(sq.sum(axis=-1, keepdims=True) / np.maximum(fin.sum(axis=-1, keepdims=True), 1))
    err = np.zeros_like(ref)
    err[fin] = np.abs(got[fin] - ref[fin])
    lim = rtol * np.maximum(np.abs(np.where(fin, ref, 0.0)), rms)
    assert (err <= lim).all(), float((err - lim).max())


def check_index_row(T_row, ref_scores_row, k, valid, atol=IDX_ATOL, rtol=IDX_RTOL_BF16):
    """T_row: the GPU's index set (ascending, -1 padded).  ref_scores_row: the oracle's scores.

    The set must be valid (distinct, ascending, causal, |T| = min(k, valid)); any index
    on which it differs from the oracle's own top-k must have an oracle score within
    the tolerance of the oracle's k-th largest score."""
    T_row = np.asarray(T_row)
    m = min(k, valid)
    sel = T_row[:m]
    assert (T_row[m:] == -1).all(), "padding"
    assert (sel >= 0).all() and (sel < valid).all(), "range"
    assert (np.diff(sel) > 0).all(), "ascending and distinct"
    if m == valid:
        assert (sel == np.arange(valid)).all()
        return 0
    s = np.asarray(ref_scores_row[:valid], dtype=np.float64)
    order = np.lexsort((np.arange(valid), -s.astype(np.float32)))
    ref_set = set(order[:m].tolist())
    kth = float(s[order[m - 1]])
    diff = ref_set.symmetric_difference(sel.tolist())
    for j in diff:
        assert abs(s[j] - kth) <= atol + rtol * abs(kth), (
            "index %d (score %.6g) differs but the k-th score is %.6g" % (j, s[j], kth))
    return len(diff) // 2


def assert_attn_close(got, ref, max_abs=ATTN_MAX_ABS, mean_abs=ATTN_MEAN_ABS, what="attn"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    assert err.max() <= max_abs, "%s: max abs err %.3g" % (what, err.max())
    assert err.mean() <= mean_abs, "%s: mean abs err %.3g" % (what, err.mean())
