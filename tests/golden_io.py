"""Reader for the worked-example fixtures under tests/golden/.

Each fixture is plain text: '#' comment lines carry the citation, the other
lines are `key = values` (whitespace-separated numbers).  Repeated keys (such
as `row`) accumulate into a list of rows.
"""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _num(tok):
    try:
        return int(tok)
    except ValueError:
        return float(tok)


def load(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            vals = [_num(t) for t in val.split()]
            v = vals[0] if len(vals) == 1 else vals
            if key == "row":
                out.setdefault("rows", []).append(vals)
            else:
                out[key] = v
    return out
