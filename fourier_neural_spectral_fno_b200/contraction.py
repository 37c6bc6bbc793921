"""Greedy ordering of the spectral block's tensor contractions.

The mixed-precision training page ("Guaranteed approximation bounds and
efficient mixed-precision training for neural operators", summary) orders the
FNO block's memory-bound half-precision tensor contractions with a simple
greedy algorithm, and runs TFNO, whose spectral weights are factorised.  The
page gives neither the factorisation nor the greedy rule; the readings are

* the factorised weight is a rank-r CP (canonical polyadic) tensor
  ``R[i, o, k] = sum_r lam[r] A[i, r] B[o, r] C[k, r]``, so the mixing
  ``yhat[b, o, k] = sum_i xhat[b, i, k] R[i, o, k]`` becomes the network
  ``bik, r, ir, or, kr -> bok``;
* greedy: while more than one operand is left, contract the pair that frees
  the most memory -- smallest (result elements - elements of the two
  operands) -- ties broken by the pair's multiply-add count, then by
  position.  An index leaves a pairwise result when neither another remaining
  operand nor the output carries it.  (Ranking pairs by the result's size
  alone is myopic: it multiplies the small CP factors together first and so
  rebuilds the dense weight.)

Host logic only.  A plan is a list of pairwise steps; the GPU mixing kernel for
factorised weights contracts in the order this plan gives at low rank.
"""

from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

Step = Tuple[int, int, str]     # positions in the current operand list, result indices


def _prod(indices: str, sizes: Dict[str, int]) -> int:
    n = 1
    for c in indices:
        n *= sizes[c]
    return n


def pair_result(a: str, b: str, others: Sequence[str], output: str) -> str:
    """Indices that a pairwise contraction of ``a`` and ``b`` keeps (in first-seen order)."""
    keep = set(output)
    for o in others:
        keep.update(o)
    out = []
    for c in a + b:
        if c in keep and c not in out:
            out.append(c)
    return "".join(out)


def pair_cost(a: str, b: str, result: str, sizes: Dict[str, int]) -> Tuple[int, int]:
    """(result elements, multiply-adds) of contracting ``a`` with ``b`` into ``result``."""
    union = "".join(dict.fromkeys(a + b))
    return _prod(result, sizes), _prod(union, sizes)


def greedy_path(inputs: Sequence[str], output: str, sizes: Dict[str, int]) -> List[Step]:
    """Greedy pairwise order for ``inputs -> output`` (einsum index strings).

    Each step ``(i, j, res)`` contracts operands ``i < j`` of the current list,
    removes both and appends the result (indices ``res``).  After the last step
    the single remaining operand carries the output's indices, possibly
    permuted, which the caller transposes.
    """
    for s in list(inputs) + [output]:
        for c in s:
            if c not in sizes:
                raise ValueError(f"index {c!r} has no size")
    ops = list(inputs)
    path: List[Step] = []
    while len(ops) > 1:
        best = None
        for i in range(len(ops)):
            for j in range(i + 1, len(ops)):
                others = [ops[k] for k in range(len(ops)) if k not in (i, j)]
                res = pair_result(ops[i], ops[j], others, output)
                size, macs = pair_cost(ops[i], ops[j], res, sizes)
                freed = size - _prod(ops[i], sizes) - _prod(ops[j], sizes)
                key = (freed, macs, i, j)
                if best is None or key < best[0]:
                    best = (key, i, j, res)
        _, i, j, res = best
        path.append((i, j, res))
        ops = [ops[k] for k in range(len(ops)) if k not in (i, j)] + [res]
    if len(ops) == 1 and sorted(ops[0]) != sorted(output):
        raise ValueError(f"indices {ops[0]!r} left, output is {output!r}")
    return path


def path_cost(inputs: Sequence[str], output: str, sizes: Dict[str, int],
              path: Sequence[Step]) -> Tuple[int, int]:
    """(largest intermediate, total multiply-adds) of a path."""
    ops = list(inputs)
    peak, macs = 0, 0
    for i, j, res in path:
        others = [ops[k] for k in range(len(ops)) if k not in (i, j)]
        if res != pair_result(ops[i], ops[j], others, output):
            raise ValueError("path step does not match its operands")
        size, m = pair_cost(ops[i], ops[j], res, sizes)
        peak, macs = max(peak, size), macs + m
        ops = others + [res]
    return peak, macs


def cp_mixing_operands(batch: int, cin: int, cout: int, n_modes: int, rank: int):
    """Einsum form of the mixing with rank-``rank`` CP weights: (inputs, output, sizes)."""
    inputs = ["bik", "r", "ir", "or", "kr"]
    sizes = {"b": batch, "i": cin, "o": cout, "k": n_modes, "r": rank}
    return inputs, "bok", sizes
