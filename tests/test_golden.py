"""Oracle pins from the hand-worked fixtures in tests/golden/ (CPU only).

The pages print no numeric worked example, so each fixture is a small case
worked out by hand from the rule a page states (the citation and the reading
head each file).  No value in them comes from code.
"""
import math

import numpy as np
import pytest

from oracle import lite_step, permutation, pyramid_attention, radial_mask
from oracle.lite import skip_flags
from oracle.masks import global_head, global_mask, level_counts, level_map, level_row, tau_mask, tau_row

from _golden import floats as _floats, ints as _ints, matrix, records as _records


@pytest.mark.parametrize("rec", _records("axis_orders.txt"), ids=lambda r: f"{r['grid']}/{r['cells']}/{r['order']}")
def test_axis_orders(rec):
    T, Hh, Ww = _ints(rec["grid"])
    perm = permutation(T, Hh, Ww, rec["order"], tuple(_ints(rec["cells"])))
    assert perm.tolist() == rec["list"]


@pytest.mark.parametrize("rec", _records("tau_rows.txt"), ids=lambda r: f"{r['p']}@{r['tau']}")
def test_tau_rows(rec):
    p = np.array(_floats(rec["p"]))
    keep, _, _, _ = tau_row(np.log(p), float(rec["tau"]))
    assert np.nonzero(keep)[0].tolist() == _ints(rec["keep"])


@pytest.mark.parametrize("rec", _records("level_rows.txt"), ids=lambda r: f"{r['p']}@{r['fr']}")
def test_level_rows(rec):
    p = np.array(_floats(rec["p"]))
    code, _ = level_row(np.log(p), level_counts(p.size, _floats(rec["fr"])))
    assert code.tolist() == _ints(rec["code"])


@pytest.mark.parametrize("rec", _records("global_heads.txt"), ids=lambda r: f"{r['p']}@{r['tau']}")
def test_global_heads(rec):
    p = np.array(matrix(rec["p"]))
    keep = global_head(np.log(p), float(rec["tau"]))[0]
    expect = np.array(matrix(rec["keep"], _ints))
    assert np.array_equal(np.asarray(keep, dtype=np.int64), expect)


@pytest.mark.parametrize("rec", _records("radial_rows.txt"), ids=lambda r: f"{r['grid']}/{r['block']}/{r['row']}")
def test_radial_rows(rec):
    T, Hh, Ww = _ints(rec["grid"])
    m = radial_mask(T, Hh, Ww, int(rec["block"]))
    assert np.nonzero(m[int(rec["row"])])[0].tolist() == _ints(rec["keep"])


@pytest.mark.parametrize("rec", _records("lite_skip.txt"), ids=lambda r: f"q{r['q']}/eps{r['eps']}")
def test_lite_skip(rec):
    q = np.array(_floats(rec["q"])).reshape(1, 1, 6, 1)
    k = np.array(_floats(rec["k"])).reshape(1, 1, 6, 1)
    v = np.arange(6, dtype=np.float64).reshape(1, 1, 6, 1)
    _, _, skip, margin = lite_step(q, k, v, 2, eps=float(rec["eps"]), scale=1.0)
    assert skip[0, 0, 0].tolist() == _ints(rec["bits"])
    got = margin[0, 0, 0]
    assert math.isnan(got[0])
    assert np.allclose(got[1:], _floats(rec["margins"]), rtol=0, atol=1e-12)


def check_margin_flags(rec):
    """One record of margin_flags.txt: decisions and their margin flags."""
    kind = rec["kind"]
    if kind == "tau":
        keep, flag, _, _ = tau_row(np.log(np.array(_floats(rec["p"]))), float(rec["tau"]))
        assert np.nonzero(keep)[0].tolist() == _ints(rec["keep"])
        assert np.nonzero(flag)[0].tolist() == _ints(rec["flag"])
    elif kind == "level":
        code, flag = level_row(np.array(_floats(rec["s"])), _ints(rec["counts"]))
        assert code.tolist() == _ints(rec["code"])
        assert np.nonzero(flag)[0].tolist() == _ints(rec["flag"])
    elif kind == "global":
        keep, flag = global_head(np.log(np.array(matrix(rec["p"]))), float(rec["tau"]))
        assert np.array_equal(np.asarray(keep, dtype=np.int64), np.array(matrix(rec["keep"], _ints)))
        assert np.array_equal(np.asarray(flag, dtype=np.int64), np.array(matrix(rec["flag"], _ints)))
    else:
        assert kind == "skip"
        flag = skip_flags(np.array(_floats(rec["margin"])))
        assert np.nonzero(flag)[0].tolist() == _ints(rec["flag"])


@pytest.mark.parametrize("rec", _records("margin_flags.txt"),
                         ids=lambda r: "-".join(f"{k}{v}" for k, v in r.items() if k in ("kind", "p", "s", "tau")))
def test_margin_flags(rec):
    check_margin_flags(rec)


def _qk_for_scores(heads, block=3):
    """fp64 Q, K [1, len(heads), nb * block, d] whose block scores are ln P for each head's
    [nb, nb] matrix P (d = nb, scale 1 / sqrt(d)): every row of q-block i is sqrt(d) e_i and
    every row of k-block j holds ln P[i, j] in dimension i, so the block means are those rows and
    S[i, j] = (1 / sqrt(d)) * sqrt(d) * ln P[i, j]."""
    nb = heads[0].shape[0]
    d, N = nb, nb * block
    q = np.zeros((1, len(heads), N, d))
    k = np.zeros((1, len(heads), N, d))
    for h, P in enumerate(heads):
        for i in range(nb):
            q[0, h, i * block:(i + 1) * block, i] = math.sqrt(d)
            for j in range(nb):
                k[0, h, j * block:(j + 1) * block, i] = math.log(P[i, j])
    return q, k


def _fixture_row_heads(p):
    """Head 0: row 0 is the fixture's row, the other rows uniform; head 1: every row uniform."""
    nb = p.size
    uniform = np.full((nb, nb), 1.0 / nb)
    h0 = uniform.copy()
    h0[0] = p
    return [h0, uniform]


@pytest.mark.parametrize("rec", _records("tau_rows.txt"), ids=lambda r: f"{r['p']}@{r['tau']}")
def test_tau_rows_through_the_mask_wrapper(rec):
    """The whole oracle path (block means, scores, per-row selection over every head and row)
    reproduces the fixture's row; uniform rows keep the first ceil(tau * Nb) blocks."""
    p = np.array(_floats(rec["p"]))
    nb, tau = p.size, float(rec["tau"])
    q, k = _qk_for_scores(_fixture_row_heads(p))
    m = tau_mask(q, k, 3, tau)
    first = list(range(math.ceil(tau * nb - 1e-9)))
    assert np.nonzero(m[0, 0, 0])[0].tolist() == _ints(rec["keep"])
    for h, i in [(0, i) for i in range(1, nb)] + [(1, i) for i in range(nb)]:
        assert np.nonzero(m[0, h, i])[0].tolist() == first, (h, i)


@pytest.mark.parametrize("rec", _records("level_rows.txt"), ids=lambda r: f"{r['p']}@{r['fr']}")
def test_level_rows_through_the_map_wrapper(rec):
    """As above for the level map; uniform rows take the codes in index order."""
    p = np.array(_floats(rec["p"]))
    nb = p.size
    q, k = _qk_for_scores(_fixture_row_heads(p))
    lv = level_map(q, k, 3, _floats(rec["fr"]))
    counts = level_counts(nb, _floats(rec["fr"]))
    uniform = [1 if r < counts[0] else 2 if r < counts[1] else 3 if r < counts[2] else 4 for r in range(nb)]
    assert lv[0, 0, 0].tolist() == _ints(rec["code"])
    for h, i in [(0, i) for i in range(1, nb)] + [(1, i) for i in range(nb)]:
        assert lv[0, h, i].tolist() == uniform, (h, i)


@pytest.mark.parametrize("rec", [r for r in _records("global_heads.txt") if len(matrix(r["p"])) == len(matrix(r["p"])[0])],
                         ids=lambda r: f"{r['p']}@{r['tau']}")
def test_global_heads_through_the_mask_wrapper(rec):
    """As above for the global selection (the square fixtures); head 1's uniform scores keep the
    first ceil(tau * Nb * Nb) pairs in index order."""
    P = np.array(matrix(rec["p"]))
    nb, tau = P.shape[0], float(rec["tau"])
    q, k = _qk_for_scores([P, np.full((nb, nb), 1.0 / nb)])
    m = global_mask(q, k, 3, tau)
    assert np.array_equal(m[0, 0].astype(np.int64), np.array(matrix(rec["keep"], _ints)))
    n_keep = math.ceil(tau * nb * nb - 1e-9)
    assert m[0, 1].ravel().tolist() == [1] * n_keep + [0] * (nb * nb - n_keep)


@pytest.mark.parametrize("rec", _records("pyramid_rows.txt"), ids=lambda r: f"codes{r['codes']}")
def test_pyramid_rows(rec):
    """d = 1, scale 1, block 8, 16 tokens, every query 1; k-block 0: keys 0, values 1."""
    k = np.array([0.0] * 8 + _floats(rec["k1"])).reshape(1, 1, 16, 1)
    v = np.array([1.0] * 8 + _floats(rec["v1"])).reshape(1, 1, 16, 1)
    q = np.ones((1, 1, 16, 1))
    codes = np.array([_ints(rec["codes"])] * 2, dtype=np.uint8)
    O, L = pyramid_attention(q, k, v, 8, codes, scale=1.0)
    assert np.allclose(O[0, 0, :8, 0], float(rec["o"]), rtol=0, atol=1e-12)
    assert np.allclose(L[0, 0, :8], float(rec["lse"]), rtol=0, atol=1e-12)
