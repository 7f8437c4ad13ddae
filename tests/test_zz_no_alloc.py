"""ic_sparse_attn_noalloc: the attention entry point for callers that cannot allocate
device memory (a plugin handed only its input and output buffers, a process whose
memory pool already owns the device).  Its split scratch is a fixed array inside the
library, so these tests check that it answers like ic_sparse_attn given a workspace,
and that a second call in a row is not disturbed by what the first left in the array.

The file name sorts last so that pytest collects it after every other test; it also
passes on its own in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from sparse_attention_indexer_sum_b200 import binding as ic
from tests.paritylib import assert_attn_close

MAX_QUERIES = 64  # IC_NOALLOC_MAX_QUERIES in include/ic.h


def _inputs(B, R, k, Lkv, seed, pad=False):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, R, 16, 576, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, Lkv, 576, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(seed)
    idx = np.stack([np.stack([np.sort(rng.permutation(Lkv)[:k]) for _ in range(R)])
                    for _ in range(B)]).astype(np.int32)
    if pad:  # ragged index lists: row r keeps k - 7 r entries, the rest are -1
        for r in range(R):
            idx[:, r, max(1, k - 7 * r):] = -1
    return q, kv, torch.from_numpy(idx)


SCRATCH_BYTES = 64 * 8 * 16 * 514 * 4  # IC_NOALLOC_SCRATCH_BYTES in include/ic.h


@pytest.mark.gpu
def test_noalloc_scratch_covers_every_accepted_query_count_on_this_device():
    # the split's scratch need (as the workspace query reports it for this device's
    # SM count) fits the fixed array for every batch * rows the entry point accepts
    for n in range(1, MAX_QUERIES + 1):
        for B, R in ((n, 1), (1, n)):
            need = ic.ic_attn_workspace_size(B, R, 16, 512, 2048)
            assert need <= SCRATCH_BYTES, (B, R, need)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    dev = "cuda"
    scale = 1 / math.sqrt(576)
    # first call: the largest accepted batch (64 decode queries, k = 2048, up to 4
    # pieces each on 148 SMs); second call: 5 queries at k = 2048, the shape with
    # the most pieces per query (about 30 each), so it reads slots the first call
    # left holding other partials; third call: a ragged, smaller shape
    for B, R, k, Lkv, seed, pad in ((MAX_QUERIES, 1, 2048, 5000, 11, False),
                                    (5, 1, 2048, 4000, 13, False),
                                    (3, 5, 1000, 1500, 12, True)):
        q, kv, idx = _inputs(B, R, k, Lkv, seed, pad)
        q, kv, idx = q.to(dev), kv.to(dev), idx.to(dev)
        ws = torch.empty(ic.ic_attn_workspace_size(B, R, 16, 512, k) // 4 + 1, device=dev)
        assert ws.numel() > 1, "the shape must take the split path"
        lse_ref = torch.empty(B, R, 16, device=dev)
        ref = ic.ic_sparse_attn(q, kv, idx, scale, lse=lse_ref, workspace=ws)
        lse = torch.full((B, R, 16), float("nan"), device=dev)
        out = torch.full((B, R, 16, 512), float("nan"), dtype=torch.bfloat16, device=dev)
        ic.ic_sparse_attn_noalloc(q, kv, idx, scale, out=out, lse=lse)
        ic.ic_device_status()
        assert_attn_close(out.float().cpu().numpy(), ref.float().cpu().numpy(),
                          what="noalloc B=%d R=%d k=%d" % (B, R, k))
        np.testing.assert_allclose(lse.cpu().numpy(), lse_ref.cpu().numpy(), atol=2e-3,
                                   rtol=1e-3)


def test_noalloc_rejects_oversize_and_mqa_before_touching_the_device():
    lib = ic.lib()
    fake = ctypes.c_void_p(256)  # never dereferenced: the checks fail first
    st = lib.ic_sparse_attn_noalloc(fake, fake, 576, None, fake, ic.IC_BF16, MAX_QUERIES + 1, 1,
                                    16, 576, 512, 4096, 2048, 1.0, fake, None, None)
    assert st == ic.IC_ERR_UNSUPPORTED
    assert "maximum of %d" % MAX_QUERIES in ic.ic_last_error()
    st = lib.ic_sparse_attn_noalloc(fake, fake, 64, fake, fake, ic.IC_F32, 1, 4, 4, 64, 64, 100,
                                    16, 1.0, fake, None, None)
    assert st == ic.IC_ERR_UNSUPPORTED
    st = lib.ic_sparse_attn_noalloc(fake, fake, 576, None, fake, ic.IC_BF16, 1, 4, 16, 576, 512,
                                    100, 4096, 1.0, fake, None, None)
    assert st == ic.IC_ERR_UNSUPPORTED  # k above 2048, as for ic_sparse_attn
    # the Python wrapper allocates nothing either: `out` is required and checked
    q = torch.zeros(1, 2, 16, 576, dtype=torch.bfloat16)
    idx = torch.zeros(1, 2, 8, dtype=torch.int32)
    with pytest.raises(TypeError):
        ic.ic_sparse_attn_noalloc(q, q[0, 0], idx, 1.0)  # noqa: missing out
    with pytest.raises(ValueError):
        ic.ic_sparse_attn_noalloc(q, q[0, 0], idx, 1.0,
                                  out=torch.zeros(1, 2, 16, 511, dtype=torch.bfloat16))
