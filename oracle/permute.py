"""Token permutations of the (t, h, w) grid (oracle; test infrastructure only).

PAROAttention write-up (pattern-aware reordering: the 6 orders of the three
axes, one per attention head) and VMoBA write-up (layer-wise recurrent 1D /
2D / 3D block partition into temporal, spatial and spatio-temporal cells).

Reading: tokens are sorted by the key (cell coordinates, coordinates inside
the cell), each tuple listed in the head's axis order, slowest axis first;
cells are ct x ch x cw and divide the grid.  1 x 1 x 1 cells give the pure
axis orders; order "thw" with cells (ct, Hh, Ww), (T, ch, cw) or (ct, ch, cw)
gives the 1D, 2D and 3D partitions.  Written as a lexicographic sort of the
tokens' keys (numpy lexsort), not as index arithmetic.
"""
from __future__ import annotations

import numpy as np

AXIS_ORDERS = ("thw", "twh", "htw", "hwt", "wth", "wht")   # index = the library's order code


def permutation(T, Hh, Ww, order="thw", cells=(1, 1, 1)):
    """perm[n'] = raster index of the token at permuted position n'."""
    if isinstance(order, int):
        order = AXIS_ORDERS[order]
    size = {"t": T, "h": Hh, "w": Ww}
    cell = dict(zip("thw", cells))
    for a in "thw":
        if size[a] % cell[a]:
            raise ValueError("cells must divide the grid")
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(Ww), indexing="ij")
    coord = {"t": t.ravel(), "h": h.ravel(), "w": w.ravel()}
    keys = [coord[a] // cell[a] for a in order] + [coord[a] % cell[a] for a in order]
    return np.lexsort(keys[::-1])          # lexsort: the last key is the primary one


def permute_tokens(x, T, Hh, Ww, orders, cells=(1, 1, 1), inverse=False):
    """x [B, H, N, d] -> the same rows reordered per head (orders: one code or
    name per head, or a single one for all heads)."""
    x = np.asarray(x)
    B, H = x.shape[:2]
    if isinstance(orders, (int, str)):
        orders = [orders] * H
    out = np.empty_like(x)
    for h in range(H):
        perm = permutation(T, Hh, Ww, orders[h], cells)
        if inverse:
            out[:, h, perm] = x[:, h]
        else:
            out[:, h] = x[:, h, perm]
    return out
