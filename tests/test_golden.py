"""Oracle pins from the hand-worked fixtures in tests/golden/ (CPU only).

The pages print no numeric worked example, so each fixture is a small case
worked out by hand from the rule a page states (the citation and the reading
head each file).  No value in them comes from code.
"""
import math

import numpy as np
import pytest

from oracle import lite_step, permutation, radial_mask
from oracle.lite import skip_flags
from oracle.masks import global_head, level_counts, level_row, tau_row

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
