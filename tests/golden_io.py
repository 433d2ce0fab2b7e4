"""Reader of the small text fixtures under tests/golden/.

Format: '#' comments; ``key v1 v2 ...`` for scalars and vectors; ``key`` alone on a
line followed by rows of numbers and ``end`` for matrices; ``case name`` starts a
named sub-record.
"""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _num(s):
    try:
        return int(s)
    except ValueError:
        return float(s)


def read(name):
    rec = {}
    cur = rec
    mat_key, mat_rows = None, None
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            if mat_key is not None:
                if line == "end":
                    cur[mat_key] = mat_rows
                    mat_key, mat_rows = None, None
                else:
                    mat_rows.append([_num(v) for v in line.split()])
                continue
            parts = line.split()
            key, vals = parts[0], parts[1:]
            if key == "case":
                cur = {}
                rec.setdefault("cases", {})[vals[0]] = cur
            elif not vals:
                if key in ("special_pairs",):
                    cur[key] = []
                else:
                    mat_key, mat_rows = key, []
            elif key == "special_pairs":
                cur[key] = [tuple(int(p) for p in v.split(",")) for v in vals]
            elif key == "dtype":
                cur[key] = vals[0]
            elif len(vals) == 1:
                cur[key] = _num(vals[0])
            else:
                cur[key] = [_num(v) for v in vals]
    return rec
