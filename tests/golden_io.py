"""Readers for the hand-worked fixtures under tests/golden/."""
import os

from conftest import GOLDEN


def _num(s):
    s = s.strip()
    return float.fromhex(s) if "0x" in s and "p" in s else float(s)


def read_floats(name):
    vals = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(float(line))
    return vals


def read_cases(name):
    """Parse 'case'/'in'/'scale'/'absmax'/'codes'/'bytes' records."""
    cases, cur = [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(" ")
            if key == "case":
                cur = {"name": rest}
                cases.append(cur)
                continue
            if cur is None:
                cur = {"name": "only"}
                cases.append(cur)
            pairs = [p.split(":") for p in rest.split()]
            if key == "in":
                cur["in"] = {int(i): _num(v) for i, v in pairs}
            elif key in ("codes", "bytes"):
                cur[key] = {int(i): int(v, 0) for i, v in pairs}
            elif key in ("scale", "absmax"):
                cur[key] = _num(rest)
    return cases
