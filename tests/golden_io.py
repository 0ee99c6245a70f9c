"""Reader for the text fixtures under tests/golden/ (parsing only)."""
import math
import os
from fractions import Fraction

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _num(tok: str) -> float:
    # closed-form tokens: integers, fractions, sqrt(...), (a+b)/c
    allowed = {"sqrt": math.sqrt, "Fraction": Fraction, "__builtins__": {}}
    return float(eval(tok, allowed, {}))  # noqa: S307 - fixture text written in this repo


def read_cases(name: str):
    cases, cur = [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            if line == "end":
                cases.append(cur)
                cur = None
                continue
            key, val = [t.strip() for t in line.split("=", 1)]
            if key == "case":
                cur = {"case": val}
            elif key == "bytes":
                cur[key] = [int(t, 16) for t in val.split()]
            elif key in ("codes", "s", "G"):
                cur[key] = [int(t) for t in val.split()]
            else:
                cur[key] = [_num(t) for t in val.split()]
    return cases
