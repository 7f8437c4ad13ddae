"""Training-free choice of the F/S layer pattern by greedy search.

Follows "IndexCache: Wie DeepSeek O(NL^2)-Kosten in Sparse Attention um 75%
reduziert", section "Training-freie Optimierung: Greedy-Suche mit minimalem
Verlust":
- start with every layer Full;
- on a small calibration set, try each Full layer in turn as Shared;
- at every step keep the one conversion that raises the model's loss least.

That takes O(N^2) forward passes. The candidates of one step are independent and
may be evaluated together (the pages evaluate blocks of layers in parallel with
pipeline parallelism). Layer 0 stays Full: the first layer of a stack always
has its own indexer ("Der unsichtbare Datenstrom").

The loss is the caller's. Typically it runs the model over the calibration set
with the candidate pattern, i.e. `ic_layer_stack` with that pattern string for
the attention layers, and returns a scalar. This module only drives the search.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional, Sequence


def pattern_string(kinds: Sequence[str]) -> str:
    """["F", "S", ...] -> "F,S,..." (the grammar ic_layer_stack accepts)."""
    return ",".join(kinds)


@dataclasses.dataclass
class SearchStep:
    layer: int          # the layer turned Shared at this step
    loss: float         # the loss with it Shared (and every earlier choice)
    pattern: str        # the pattern after this step


@dataclasses.dataclass
class SearchResult:
    pattern: str                 # the final pattern
    base_loss: float             # the all-Full loss
    steps: list                  # SearchStep per accepted conversion, in order
    evaluations: int             # loss evaluations made


def greedy_pattern_search(n_layers: int,
                          loss: Optional[Callable[[str], float]] = None,
                          *,
                          evaluate_many: Optional[Callable[[list], list]] = None,
                          n_full: Optional[int] = None,
                          max_loss_increase: Optional[float] = None) -> SearchResult:
    """Greedy F -> S conversion.

    loss(pattern) returns the calibration loss of one pattern string, or
    evaluate_many(patterns) returns the losses of a list of patterns (so the
    caller can evaluate one step's candidates in parallel); give one of them.

    The search stops when n_full Full layers remain (default: a quarter of the
    layers, at least one), or before a step whose best conversion would lift the
    loss more than max_loss_increase above the all-Full loss.
    """
    if n_layers < 1:
        raise ValueError("n_layers must be >= 1")
    if (loss is None) == (evaluate_many is None):
        raise ValueError("give exactly one of loss and evaluate_many")
    if n_full is None:
        n_full = max(1, n_layers // 4)
    if not 1 <= n_full <= n_layers:
        raise ValueError("n_full must be in [1, n_layers]")
    if evaluate_many is None:
        evaluate_many = lambda pats: [float(loss(p)) for p in pats]  # noqa: E731

    kinds = ["F"] * n_layers
    base = float(evaluate_many([pattern_string(kinds)])[0])
    evals = 1
    steps = []
    while sum(k == "F" for k in kinds) > n_full:
        cands = [l for l in range(1, n_layers) if kinds[l] == "F"]
        if not cands:
            break
        pats = []
        for l in cands:
            trial = list(kinds)
            trial[l] = "S"
            pats.append(pattern_string(trial))
        losses = [float(x) for x in evaluate_many(pats)]
        evals += len(pats)
        if len(losses) != len(pats):
            raise ValueError("evaluate_many returned %d losses for %d patterns" %
                             (len(losses), len(pats)))
        # smallest loss; ties go to the lower layer index
        j = min(range(len(cands)), key=lambda i: (losses[i], cands[i]))
        if max_loss_increase is not None and losses[j] - base > max_loss_increase:
            break
        kinds[cands[j]] = "S"
        steps.append(SearchStep(layer=cands[j], loss=losses[j], pattern=pattern_string(kinds)))
    return SearchResult(pattern=pattern_string(kinds), base_loss=base, steps=steps,
                        evaluations=evals)
