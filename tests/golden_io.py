"""Reader for the hand-worked golden plans in tests/golden/."""
import os
from fractions import Fraction

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _ints(s):
    return [int(v) for v in s.split()]


def _rows(s):
    return [_ints(part) for part in s.split("|")]


def _fraction_expr(s):
    # "a*b/c-1"
    num, rest = s.split("/")
    den, minus = rest.split("-")
    a, b = num.split("*")
    return Fraction(int(a) * int(b), int(den)) - int(minus)


def load_plans(name="hand_worked_plans.txt"):
    cases = []
    cur = None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case "):
                cur = dict(name=line.split()[1])
                cases.append(cur)
                continue
            if line.startswith("R="):
                for kv in line.split():
                    k, v = kv.split("=")
                    cur[k] = int(v)
                continue
            k, v = line.split("=", 1)
            if k in ("idx", "slot_expert", "cu_seqlens", "dst_row"):
                cur[k] = _rows(v)
            elif k in ("expert_count", "rank_load", "src_of_row"):
                cur[k] = _ints(v)
            elif k == "maxvio":
                cur[k] = _fraction_expr(v)
            else:
                cur[k] = int(v)
    return cases
