"""The greedy F/S pattern search (training-free layer selection): its stopping rules
and evaluation count, optimality where greedy is provably optimal (a loss that adds
one cost per Shared layer), and an end-to-end search whose loss runs the layer stack
(oracle on the CPU; the CUDA stack on the GPU)."""
import itertools

import numpy as np
import pytest

from sparse_attention_indexer_sum_b200 import synth
from sparse_attention_indexer_sum_b200.pattern_search import greedy_pattern_search


def _additive(costs):
    def loss(p):
        kinds = p.split(",")
        return 1.0 + sum(c for c, k in zip(costs, kinds) if k == "S")
    return loss


def test_additive_loss_reaches_the_optimum_in_cost_order():
    costs = [0.0, 0.7, 0.1, 0.9, 0.3, 0.05, 0.6, 0.2]
    r = greedy_pattern_search(8, _additive(costs), n_full=2)
    # optimum: the 6 cheapest layers among 1..7 Shared (layer 0 always Full)
    best = min((set(s) for s in itertools.combinations(range(1, 8), 6)),
               key=lambda s: sum(costs[i] for i in s))
    assert {l for l, k in enumerate(r.pattern.split(",")) if k == "S"} == best
    assert [st.layer for st in r.steps] == [5, 2, 7, 4, 6, 1]   # cheapest first
    assert r.pattern.split(",")[0] == "F"
    assert r.base_loss == 1.0
    assert r.evaluations == 1 + 7 + 6 + 5 + 4 + 3 + 2           # O(N^2) forward passes


def test_stopping_rules_and_defaults():
    costs = [0.0, 0.5, 0.1, 0.2, 0.4, 0.3, 0.6, 0.7]
    r = greedy_pattern_search(8, _additive(costs), max_loss_increase=0.35, n_full=1)
    assert [st.layer for st in r.steps] == [2, 3]            # 0.1, then 0.1 + 0.2 = 0.3
    assert r.pattern == "F,F,S,S,F,F,F,F"
    r = greedy_pattern_search(8, _additive(costs))            # default: keep a quarter
    assert r.pattern.count("F") == 2
    r = greedy_pattern_search(4, _additive([0, 1, 2, 3]), n_full=4)
    assert r.pattern == "F,F,F,F" and r.steps == [] and r.evaluations == 1
    r = greedy_pattern_search(1, _additive([0]))
    assert r.pattern == "F"
    with pytest.raises(ValueError):
        greedy_pattern_search(4)
    with pytest.raises(ValueError):
        greedy_pattern_search(4, _additive([0] * 4), n_full=0)


def test_batched_evaluation_gets_one_call_per_step_and_ties_go_low():
    calls = []

    def many(pats):
        calls.append(len(pats))
        return [1.0] * len(pats)   # every conversion costs nothing: ties everywhere

    r = greedy_pattern_search(6, evaluate_many=many, n_full=3)
    assert calls == [1, 5, 4, 3]
    assert [st.layer for st in r.steps] == [1, 2, 3]


def _stack_layers(wl):
    return [dict(synth.indexer_inputs(wl, l), **synth.attn_inputs(wl, l))
            for l in range(wl.layers)]


def _deviation_loss(run_stack, wl):
    """Calibration-style loss: mean |out_l(pattern) - out_l(all F)| over the layers."""
    ref = run_stack(",".join("F" * wl.layers))

    def loss(p):
        outs = run_stack(p)
        return float(np.mean([np.abs(a - b).mean() for a, b in zip(outs, ref)]))
    return loss


def test_search_over_the_oracle_stack():
    import oracle
    wl = synth.variant("tiny_stack", L=192, k=24, pattern="F,S,S,S,F,S,S,S")
    lay = [{k: v.numpy() for k, v in d.items()} for d in _stack_layers(wl)]

    def run(p):
        return [r["out"] for r in oracle.layer_stack(p, lay, wl.k, wl.scale)]

    loss = _deviation_loss(run, wl)
    r = greedy_pattern_search(wl.layers, loss, n_full=2)
    kinds = r.pattern.split(",")
    assert kinds[0] == "F" and kinds.count("F") == 2 and len(kinds) == 8
    assert r.base_loss == 0.0
    assert all(st.loss >= 0.0 for st in r.steps)
    # each accepted step is the best of its candidates: re-evaluate the last one
    assert loss(r.pattern) == pytest.approx(r.steps[-1].loss)


@pytest.mark.gpu
def test_search_over_the_cuda_stack_matches_the_oracle_search():
    import torch
    import oracle
    from sparse_attention_indexer_sum_b200 import binding as ic
    wl = synth.variant("tiny_stack", L=192, k=24, pattern="F,S,S,S,F,S,S,S")
    host = _stack_layers(wl)
    lay = [{k: v.numpy() for k, v in d.items()} for d in host]
    dev = [{k: v.cuda() for k, v in d.items()} for d in host]
    for d in dev:
        d["out"] = torch.empty(wl.L, wl.Hq, wl.Dv, device="cuda")
        d["lse"] = torch.empty(wl.L, wl.Hq, device="cuda")
    desc = ic.make_desc(L=wl.L, k=wl.k, H=wl.H, D=wl.D, idx_dtype=ic.IC_F32, heads=wl.Hq,
                        dk=wl.Dk, dv=wl.Dv, attn_dtype=ic.IC_F32, scale=wl.scale)
    ws = torch.empty(ic.ic_stack_workspace_size(desc) // 4 + 1, device="cuda")
    t_cache = torch.empty(wl.L, wl.k, dtype=torch.int32, device="cuda")

    def run_gpu(p):
        ic.ic_layer_stack(p, desc, dev, t_cache, ws)
        ic.ic_device_status()
        return [d["out"].cpu().numpy() for d in dev]

    def run_cpu(p):
        return [r["out"] for r in oracle.layer_stack(p, lay, wl.k, wl.scale)]

    r_gpu = greedy_pattern_search(wl.layers, _deviation_loss(run_gpu, wl), n_full=2)
    cpu_loss = _deviation_loss(run_cpu, wl)
    # replay on the oracle: every step the GPU search took is (within rounding) the
    # best conversion the oracle sees from the same starting pattern, and the GPU
    # losses agree with the oracle's
    kinds = ["F"] * wl.layers
    for st in r_gpu.steps:
        cands = [l for l in range(1, wl.layers) if kinds[l] == "F"]
        losses = {}
        for l in cands:
            trial = list(kinds)
            trial[l] = "S"
            losses[l] = cpu_loss(",".join(trial))
        assert losses[st.layer] <= min(losses.values()) * (1 + 1e-3) + 1e-6
        assert st.loss == pytest.approx(losses[st.layer], rel=1e-3, abs=1e-5)
        kinds[st.layer] = "S"
    assert ",".join(kinds) == r_gpu.pattern
