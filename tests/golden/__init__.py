"""Parsers for the worked examples printed on the nanoMoE slides."""
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def _rows(name):
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def load_m1():
    """List of (logits[3], kept (lo, hi), gates (lo, hi))."""
    out = []
    for line in _rows("m1_router.txt"):
        a, b, c = [p.split() for p in line.split("|")]
        out.append(([float(v) for v in a], tuple(int(v) for v in b), tuple(float(v) for v in c)))
    return out


def load_m2():
    d = {}
    for line in _rows("m2_capacity.txt"):
        key, _, rest = line.partition(" ")
        if key in ("E", "k", "C"):
            d[key] = int(rest)
        elif key == "used":
            d[key] = [int(v) for v in rest.split()]
        elif key == "combine":
            rows = []
            for part in rest.split("|"):
                terms = []
                for term in part.split(";"):
                    if term.strip():
                        g, e, t = term.split()
                        terms.append((float(g), int(e), int(t)))
                rows.append(terms)
            d[key] = rows
        else:
            conv = float if key == "gates" else int
            d[key] = [[conv(v) for v in part.split()] for part in rest.split("|")]
    return d
