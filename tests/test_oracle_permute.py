"""Pins for the oracle's token permutations (CPU only): each order and cell
partition against numpy's axis transposes of the token grid, a hand-listed
case, bijectivity and the inverse."""
import numpy as np
import pytest

from oracle import permutation, permute_tokens

ORDERS = ("thw", "twh", "htw", "hwt", "wth", "wht")
AXES = {"t": 0, "h": 1, "w": 2}


@pytest.mark.parametrize("order", ORDERS)
def test_axis_orders_equal_grid_transposes(order):
    T, Hh, Ww = 3, 4, 5
    grid = np.arange(T * Hh * Ww).reshape(T, Hh, Ww)
    expect = np.transpose(grid, [AXES[a] for a in order]).ravel()
    assert np.array_equal(permutation(T, Hh, Ww, order), expect)
    assert np.array_equal(permutation(T, Hh, Ww, ORDERS.index(order)), expect)


def test_hand_listed_hwt():
    # grid T=2, Hh=2, Ww=3, raster n = (t*2 + h)*3 + w; order h, w, t
    assert permutation(2, 2, 3, "hwt").tolist() == [0, 6, 1, 7, 2, 8, 3, 9, 4, 10, 5, 11]


def test_cell_partitions_equal_blocked_transposes():
    T, Hh, Ww = 6, 4, 6
    grid = np.arange(T * Hh * Ww).reshape(T, Hh, Ww)
    # 1D temporal cells of 3 frames: raster order already
    assert np.array_equal(permutation(T, Hh, Ww, "thw", (3, Hh, Ww)), grid.ravel())
    # 2D spatial cells 2 x 3 over all frames: (cell y, cell x, t, y in, x in)
    g2 = grid.reshape(T, Hh // 2, 2, Ww // 3, 3).transpose(1, 3, 0, 2, 4).ravel()
    assert np.array_equal(permutation(T, Hh, Ww, "thw", (T, 2, 3)), g2)
    # 3D cells 3 x 2 x 3: (cell t, cell y, cell x, t in, y in, x in)
    g3 = grid.reshape(T // 3, 3, Hh // 2, 2, Ww // 3, 3).transpose(0, 2, 4, 1, 3, 5).ravel()
    assert np.array_equal(permutation(T, Hh, Ww, "thw", (3, 2, 3)), g3)
    # cells with a non-raster axis order: cell tuple and in-cell tuple both in that order
    g4 = grid.reshape(T // 3, 3, Hh // 2, 2, Ww // 3, 3).transpose(4, 2, 0, 5, 3, 1).ravel()
    assert np.array_equal(permutation(T, Hh, Ww, "wht", (3, 2, 3)), g4)


def test_bijection_inverse_and_per_head_orders():
    rng = np.random.default_rng(0)
    T, Hh, Ww = 2, 3, 4
    x = rng.normal(size=(2, 3, T * Hh * Ww, 8))
    orders = [1, 3, 5]
    y = permute_tokens(x, T, Hh, Ww, orders, cells=(1, 1, 2))
    for h, o in enumerate(orders):
        perm = permutation(T, Hh, Ww, o, (1, 1, 2))
        assert sorted(perm.tolist()) == list(range(T * Hh * Ww))
        assert np.array_equal(y[:, h], x[:, h, perm])
    assert np.array_equal(permute_tokens(y, T, Hh, Ww, orders, cells=(1, 1, 2), inverse=True), x)
    with pytest.raises(ValueError):
        permutation(T, Hh, Ww, "thw", (1, 2, 1))
