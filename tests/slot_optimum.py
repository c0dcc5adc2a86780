"""The fewest slots any plan can need (test infrastructure, CPU only).

A plan keeps exactly C = S*K rows on every rank ([ainovat], the hard S x K
invariant).  An over-full rank keeps C of its home rows, split over its home
experts in any way, and hands the rest on; an under-full rank keeps all of
its home rows and takes def = C - load rows handed on by others.  A receiving
rank needs one slot per distinct expert it takes rows of ([ainovat], the
redundant-experts paragraph).  Rows of one expert are interchangeable, so
only the per-expert counts matter.

`min_max_slots` finds the smallest possible largest slot count over the
receiving ranks by integer programming (scipy.optimize.milp); the pages call
the library's choice of replicas "near-optimal" ([findrepo] "Strengths"),
and this is the optimum that claim is measured against.
`brute_min_max_slots` finds the same number by enumerating every split on
tiny cases, and pins the former.
"""
import itertools
from functools import lru_cache

import numpy as np


def _split(cnt, R, C):
    cnt = np.asarray(cnt, np.int64)
    E = cnt.size
    Er = E // R
    load = cnt.reshape(R, Er).sum(1)
    over = [h for h in range(R) if load[h] > C]
    under = [r for r in range(R) if load[r] < C]
    return cnt, Er, load, over, under


def min_max_slots(cnt, R, C, time_limit=60.0):
    """Smallest max over receiving ranks of the distinct experts received."""
    from scipy.optimize import Bounds, LinearConstraint, milp
    cnt, Er, load, over, under = _split(cnt, R, C)
    if not over:
        return 0
    experts = [e for h in over for e in range(h * Er, (h + 1) * Er) if cnt[e] > 0]
    ne, nr = len(experts), len(under)
    # variables: k_e (ne), x_{e,r} (ne*nr), y_{e,r} (ne*nr), z
    nk, nx, ny = ne, ne * nr, ne * nr
    n = nk + nx + ny + 1
    iz = n - 1

    def ix(i, j):
        return nk + i * nr + j

    def iy(i, j):
        return nk + nx + i * nr + j

    rows, lo, hi = [], [], []

    def add(coefs, l, h):
        a = np.zeros(n)
        for j, v in coefs:
            a[j] += v
        rows.append(a)
        lo.append(l)
        hi.append(h)

    pos = {e: i for i, e in enumerate(experts)}
    for h in over:  # an over-full rank keeps exactly C rows
        add([(pos[e], 1.0) for e in range(h * Er, (h + 1) * Er) if e in pos], C, C)
    for i, e in enumerate(experts):  # every row is kept or handed on
        add([(i, 1.0)] + [(ix(i, j), 1.0) for j in range(nr)], cnt[e], cnt[e])
    for j, r in enumerate(under):  # every receiver is filled to C
        d = C - load[r]
        add([(ix(i, j), 1.0) for i in range(ne)], d, d)
    for i, e in enumerate(experts):  # rows taken only with a slot
        for j, r in enumerate(under):
            m = min(cnt[e], C - load[r])
            add([(ix(i, j), 1.0), (iy(i, j), -float(m))], -np.inf, 0)
    for j in range(nr):  # slots per receiver <= z
        add([(iy(i, j), 1.0) for i in range(ne)] + [(iz, -1.0)], -np.inf, 0)
    lb = np.zeros(n)
    ub = np.full(n, np.inf)
    ub[:nk] = [cnt[e] for e in experts]
    ub[nk + nx:nk + nx + ny] = 1
    c = np.zeros(n)
    c[iz] = 1.0
    res = milp(c, constraints=LinearConstraint(np.array(rows), lo, hi),
               integrality=np.ones(n), bounds=Bounds(lb, ub),
               options=dict(time_limit=time_limit))
    if res.status != 0:
        raise RuntimeError("milp: %s" % res.message)
    return int(round(res.x[iz]))


def brute_min_max_slots(cnt, R, C):
    """The same optimum by enumeration (tiny cases only)."""
    cnt, Er, load, over, under = _split(cnt, R, C)
    if not over:
        return 0
    defs = tuple(int(C - load[r]) for r in under)

    def keeps(h):  # every way rank h can keep C of its home rows
        cs = [int(cnt[e]) for e in range(h * Er, (h + 1) * Er)]
        for ks in itertools.product(*[range(c + 1) for c in cs]):
            if sum(ks) == C:
                yield tuple(c - k for c, k in zip(cs, ks))

    @lru_cache(maxsize=None)
    def best(ovf, room, used):
        # ovf: remaining overflow per expert; room: remaining capacity per
        # receiver; used: slots used per receiver so far -> least max slots
        if not ovf:
            return max(used) if used else 0
        o, rest = ovf[0], ovf[1:]
        if o == 0:
            return best(rest, room, used)
        res = None
        nr = len(room)

        def parts(i, left, take):
            if i == nr:
                if left == 0:
                    yield take
                return
            for t in range(min(left, room[i]) + 1):
                yield from parts(i + 1, left - t, take + (t,))

        for take in parts(0, o, ()):
            room2 = tuple(a - t for a, t in zip(room, take))
            used2 = tuple(u + (t > 0) for u, t in zip(used, take))
            v = best(rest, room2, used2)
            res = v if res is None else min(res, v)
        return res if res is not None else 10 ** 9

    out = None
    for combo in itertools.product(*[list(keeps(h)) for h in over]):
        ovf = tuple(o for part in combo for o in part)
        v = best(ovf, defs, tuple(0 for _ in defs))
        out = v if out is None else min(out, v)
    return out


def plan_max_slots(pl, B):
    """Largest slot count over the ranks of an oracle plan made with enough
    slots (B at least the count any rank can need)."""
    se = np.asarray(pl["slot_expert"]).reshape(-1, B)
    return int((se >= 0).sum(1).max()) if B else 0
