"""Reader for the hand-worked fixtures in tests/golden/.

Each data line is a run of 'key=value' fields, optionally followed by
' : ' and a space-separated list (kept under the key 'list'); lines that
start with '#' carry the citation and the reading the values were worked from.
"""
import pathlib

GOLDEN = pathlib.Path(__file__).parent / "golden"


def records(name):
    out = []
    for line in (GOLDEN / name).read_text(encoding="utf-8").splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, _, tail = line.partition(" : ")
        rec = dict(f.split("=", 1) for f in head.split())
        if tail:
            rec["list"] = [int(x) for x in tail.split()]
        out.append(rec)
    assert out, name
    return out


def ints(s):
    return [int(x) for x in s.split(",")] if s else []


def floats(s):
    return [float(x) for x in s.split(",")]


def matrix(s, conv=floats):
    """'a,b/c,d' -> [[a, b], [c, d]]."""
    return [conv(row) for row in s.split("/")]
