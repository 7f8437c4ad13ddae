"""The debug-bounds build (libic_b200_debug.so, -DIC_DEBUG_BOUNDS) on the GPU.

It must agree with the release build where every index is in range, and report
IC_ERR_BOUNDS where an index list holds entries outside its cache (which every
build skips). Each run of the debug library is a child process with
IC_DEBUG_BOUNDS=1, since a process loads one build of the library."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from sparse_attention_indexer_sum_b200 import binding as ic
from sparse_attention_indexer_sum_b200 import build, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# The child: the F,S stack of a 2600-token prefill (bf16) and one attention call
# with out-of-range index entries; writes T, the attention output and both statuses.
CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
from sparse_attention_indexer_sum_b200 import binding as ic
from tests.test_gpu_debug_bounds import stack_case, attn_case
out = {}
T, o = stack_case()
try:
    ic.ic_device_status(); out["stack_status"] = 0
except ic.ICError as e:
    out["stack_status"] = e.status
np.save(sys.argv[2] + "_T.npy", T.cpu().numpy())
np.save(sys.argv[2] + "_o.npy", o.float().cpu().numpy())
a = attn_case()
try:
    ic.ic_device_status(); out["attn_status"] = 0
except ic.ICError as e:
    out["attn_status"] = e.status
np.save(sys.argv[2] + "_a.npy", a.float().cpu().numpy())
print(json.dumps(out))
"""


def stack_case():
    wl = synth.variant("prefill_8k", L=2600, pattern="F,S")
    layers = []
    for l in range(wl.layers):
        d = synth.indexer_inputs(wl, l, device=DEV)
        d.update(synth.attn_inputs(wl, l, device=DEV))
        d["out"] = torch.empty(wl.L, wl.Hq, wl.Dv, dtype=torch.bfloat16, device=DEV)
        d["lse"] = torch.empty(wl.L, wl.Hq, device=DEV)
        layers.append(d)
    desc = ic.make_desc(L=wl.L, k=wl.k, H=wl.H, D=wl.D, idx_dtype=ic.IC_BF16, heads=wl.Hq,
                        dk=wl.Dk, dv=wl.Dv, attn_dtype=ic.IC_BF16, scale=wl.scale)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device=DEV)
    t = torch.full((wl.L, wl.k), -7, dtype=torch.int32, device=DEV)
    ic.ic_layer_stack(wl.pattern, desc, layers, t, ws)
    torch.cuda.synchronize()
    return t, layers[1]["out"]


def attn_case():
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 5, 16, 576, generator=g).to(torch.bfloat16).to(DEV)
    kv = torch.randn(1, 300, 576, generator=g).to(torch.bfloat16).to(DEV)
    idx = torch.randint(0, 300, (1, 5, 64), generator=g, dtype=torch.int32)
    idx[0, 1, 7] = 300 + 3        # past the cache
    idx[0, 3, 0] = -5             # below the -1 padding
    return ic.ic_sparse_attn(q, kv, idx.to(DEV), 576 ** -0.5)


def test_debug_bounds_build_agrees_and_reports(tmp_path):
    build.build(debug_bounds=True)
    env = dict(os.environ, IC_DEBUG_BOUNDS="1", PYTHONPATH=ROOT)
    base = str(tmp_path / "dbg")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, base], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    st = json.loads(r.stdout.strip().splitlines()[-1])
    # every index in range: no report, and the same index sets and outputs as the release build
    assert st["stack_status"] == 0
    T, o = stack_case()
    ic.ic_device_status()
    assert np.array_equal(np.load(base + "_T.npy"), T.cpu().numpy())
    assert np.array_equal(np.load(base + "_o.npy"), o.float().cpu().numpy())
    # out-of-range entries: skipped by both builds (same output), reported by the debug one
    assert st["attn_status"] == ic.IC_ERR_BOUNDS
    a = attn_case()
    ic.ic_device_status()
    assert np.array_equal(np.load(base + "_a.npy"), a.float().cpu().numpy())
