"""Factorised spectral weights (CP reading of TFNO) and the greedy contraction
order (CPU): the oracle's CP weight against hand values and the single-mode
closed form, and the planner against brute force and against direct einsum."""

import itertools

import numpy as np
import pytest

import oracle as O
from fourier_neural_spectral_fno_b200 import contraction as C


def test_cp_weight_hand_values():
    # rank 2, Ci = Co = 2, |K| = 2, integer factors: R[i,o,k] = sum_r lam_r a_ir b_or c_kr
    lam = [1.0, 2.0]
    a = [[1.0, 0.0], [0.0, 1.0]]
    b = [[1.0, 1.0], [2.0, 0.0]]
    c = [[1.0, 1.0], [0.0, 3.0]]
    r = O.cp_weights(lam, a, b, c)
    # i=0 uses only r=0 (lam 1): b[:,0] (1, 2) x c[:,0] (1, 0)
    np.testing.assert_array_equal(r[0].real, [[1.0, 0.0], [2.0, 0.0]])
    # i=1 uses only r=1 (lam 2): b[:,1] (1, 0) x c[:,1] (1, 3) times 2
    np.testing.assert_array_equal(r[1].real, [[2.0, 6.0], [0.0, 0.0]])
    assert not r.imag.any()


def test_cp_single_mode_closed_form():
    """Rank-1 complex weight, input cos(theta(k*, n)) on channel i: output channel o
    is |R| cos(theta + arg R) with R = lam a_i b_o c_k* (the single-mode response)."""
    grid, modes = (8, 6), (2, 3)
    rng = np.random.default_rng(31)
    nk = O.num_modes(grid, modes)
    lam = np.array([0.7 - 0.2j])
    a = rng.standard_normal((2, 1)) + 1j * rng.standard_normal((2, 1))
    b = rng.standard_normal((3, 1)) + 1j * rng.standard_normal((3, 1))
    c = rng.standard_normal((nk, 1)) + 1j * rng.standard_normal((nk, 1))
    k0, k1 = -1, 2                                  # a negative-block row, last-axis column 2
    n0, n1 = np.indices(grid)
    theta = 2 * np.pi * (k0 * n0 / grid[0] + k1 * n1 / grid[1])
    x = np.zeros((1, 2) + grid)
    x[0, 1] = np.cos(theta)
    slot = (2 * modes[0] - 1) * modes[1] + k1       # k0 = -1 is the last row of its block
    y, _ = O.spectral_conv_fwd_cp(x, lam, a, b, c, modes)
    for o in range(3):
        rr = lam[0] * a[1, 0] * b[o, 0] * c[slot, 0]
        np.testing.assert_allclose(y[0, o], np.abs(rr) * np.cos(theta + np.angle(rr)), atol=1e-12)


def _run_path(path, inputs, output, arrays):
    ops, arrs = list(inputs), list(arrays)
    for i, j, res in path:
        new = np.einsum(f"{ops[i]},{ops[j]}->{res}", arrs[i], arrs[j])
        keep = [k for k in range(len(ops)) if k not in (i, j)]
        ops, arrs = [ops[k] for k in keep] + [res], [arrs[k] for k in keep] + [new]
    return np.einsum(f"{ops[0]}->{output}", arrs[0])


@pytest.mark.parametrize("shape", [(2, 3, 4, 5, 2), (3, 4, 4, 6, 12), (1, 2, 5, 3, 40)])
def test_greedy_path_computes_the_mixing(shape):
    bsz, ci, co, nk, rank = shape
    rng = np.random.default_rng(32)
    xh = rng.standard_normal((bsz, ci, nk)) + 1j * rng.standard_normal((bsz, ci, nk))
    lam = rng.standard_normal(rank) + 0j
    a = rng.standard_normal((ci, rank)) + 1j * rng.standard_normal((ci, rank))
    b = rng.standard_normal((co, rank)) + 1j * rng.standard_normal((co, rank))
    c = rng.standard_normal((nk, rank)) + 1j * rng.standard_normal((nk, rank))
    inputs, output, sizes = C.cp_mixing_operands(*shape)
    path = C.greedy_path(inputs, output, sizes)
    got = _run_path(path, inputs, output, [xh, lam, a, b, c])
    ref = np.einsum("bik,iok->bok", xh, O.cp_weights(lam, a, b, c))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def _all_paths(inputs, output):
    """Every pairwise order (brute force, for a handful of operands)."""
    if len(inputs) == 1:
        yield []
        return
    for i, j in itertools.combinations(range(len(inputs)), 2):
        others = [inputs[k] for k in range(len(inputs)) if k not in (i, j)]
        res = C.pair_result(inputs[i], inputs[j], others, output)
        for rest in _all_paths(others + [res], output):
            yield [(i, j, res)] + rest


@pytest.mark.parametrize("shape", [(16, 32, 32, 512, 8), (32, 64, 64, 1152, 16),
                                   (8, 64, 64, 2048, 64), (4, 20, 20, 288, 20)])
def test_greedy_is_memory_optimal_for_low_rank_cp(shape):
    """On the workloads' shapes at low rank the greedy order reaches the smallest
    possible peak intermediate and never forms the dense [Ci][Co][|K|] weight."""
    inputs, output, sizes = C.cp_mixing_operands(*shape)
    path = C.greedy_path(inputs, output, sizes)
    peak, macs = C.path_cost(inputs, output, sizes, path)
    best_peak = min(C.path_cost(inputs, output, sizes, p)[0] for p in _all_paths(inputs, output))
    assert peak == best_peak
    assert all(sorted(res) != sorted("iok") for _, _, res in path)
    bsz, ci, co, nk, rank = shape
    if 2 * rank <= min(ci, co):                      # then also cheaper than the dense mixing
        assert macs < bsz * ci * co * nk


def test_greedy_rebuilds_the_weight_at_high_rank():
    """When the rank exceeds what the factors save, forming R first frees the most."""
    inputs, output, sizes = C.cp_mixing_operands(16, 32, 32, 512, 512)
    path = C.greedy_path(inputs, output, sizes)
    assert any(sorted(res) == sorted("iok") for _, _, res in path)


def test_path_cost_hand_example():
    # ab,bc->ac with a=2, b=3, c=4: one step, result 8 elements, 24 multiply-adds
    sizes = {"a": 2, "b": 3, "c": 4}
    path = C.greedy_path(["ab", "bc"], "ac", sizes)
    assert path == [(0, 1, "ac")]
    assert C.path_cost(["ab", "bc"], "ac", sizes, path) == (8, 24)
    with pytest.raises(ValueError):
        C.greedy_path(["ab", "bz"], "ac", sizes)
