"""CPU checks of the parity checker itself (tests/parity.py): a single wrong
128-row tile of a long head must fail even where the whole-tensor norm
absorbs it, and the noise level of correct bf16 results must pass."""

import numpy as np
import pytest

from tests.parity import TOL, compare_arrays, rel_fro, tile_errors


def _head(T=8192, D=128, seed=0):
    rng = np.random.default_rng(seed)
    ref = rng.standard_normal((1, T, D))
    # a result carrying the error level of a correct bf16 run (~2e-3)
    got = ref + 2e-3 * np.abs(ref).mean() * rng.standard_normal(ref.shape)
    return rng, ref, got


def test_correct_result_passes_both_checks():
    _, ref, got = _head()
    errs = compare_arrays({"o": got}, {"o": ref}, TOL["bf16"], keys=("o",))
    assert errs["o"] < 3e-3 and errs["o_tile"] < 4e-3


def test_one_wrong_tile_fails_although_the_whole_tensor_norm_passes():
    rng, ref, got = _head()
    bad = got.copy()
    bad[0, 4096:4224] += 0.06 * rng.standard_normal((128, 128))  # one tile 6 % off
    assert rel_fro(bad, ref) < TOL["bf16"]["o"]  # the norm alone lets it through
    with pytest.raises(AssertionError, match="o_tile"):
        compare_arrays({"o": bad}, {"o": ref}, TOL["bf16"], keys=("o",))


def test_one_row_replaced_by_its_neighbour_fails():
    _, ref, got = _head()
    bad = got.copy()
    bad[0, 777] = bad[0, 778]  # an off-by-one row inside one tile
    with pytest.raises(AssertionError, match="o_tile"):
        compare_arrays({"o": bad}, {"o": ref}, TOL["bf16"], keys=("o",))


def test_tile_floor_guards_tiles_with_a_near_zero_reference():
    rng, ref, got = _head(T=1024, D=64)
    ref[0, 896:] *= 1e-6  # a tile whose reference is almost zero ...
    got[0, 896:] = ref[0, 896:] + 1e-6 * 2e-3 * rng.standard_normal((128, 64))
    # ... with a tiny absolute error is not divided by ~0
    assert tile_errors(got, ref).max() < 4e-3


def test_lse_shape_is_handled():
    rng = np.random.default_rng(3)
    ref = 5.0 + rng.standard_normal((2, 300))
    got = ref * (1 + 1e-6 * rng.standard_normal(ref.shape))
    errs = compare_arrays({"lse": got}, {"lse": ref}, TOL["bf16"], keys=("lse",))
    assert errs["lse_tile"] < 1e-5
