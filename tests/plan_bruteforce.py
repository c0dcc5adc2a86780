"""An independent, literal planner used to pin the oracle's plan.

It never shares a step with the oracle: it builds the full list of
(expert, token, k) triples, sorts it, slices it per rank, and walks the rule
with Python lists.  The oracle instead counting-sorts picks and fills rows
through index arithmetic.  Both follow the same written rule:

  each rank keeps its home experts' rows (experts in index order, rows in
  (token, k) order) up to C = S*K (rule 0), or keeps, per expert, what fits
  when its experts are filled lightest first (rule 1); the rows not kept form
  one stream in (rank, expert, token, k) order; ranks with room take the next
  rows of the stream in rank order; each distinct expert a rank receives
  takes one slot in order of first appearance; more than B slots fails.
  Rule 2 keeps rows as rule 1, orders the stream's experts by decreasing
  overflow count (ties: lower index) and walks the receiving ranks by
  decreasing deficit (ties: lower index).
"""
from collections import Counter


def brute_plan(idx, R, S, E, K, B, rule=0):
    T = R * S
    C = S * K
    Er = E // R
    triples = [(int(idx[t][k]), t, k) for t in range(T) for k in range(K)]
    for e, _, _ in triples:
        if not 0 <= e < E:
            return dict(status=4)
    cnt = Counter(e for e, _, _ in triples)
    counts = [cnt.get(e, 0) for e in range(E)]
    max_count = max(counts)
    maxvio = max_count / ((T * K) / E) - 1.0
    rank_load = [sum(counts[r * Er:(r + 1) * Er]) for r in range(R)]

    rows = [[] for _ in range(R)]  # per rank: list of (group, triple)
    stream = []
    for r in range(R):
        home = sorted(tr for tr in triples if tr[0] // Er == r)
        if rule == 0:
            kept, over = home[:C], home[C:]
        else:  # rules 1 and 2: lightest experts kept first
            experts = sorted(range(r * Er, (r + 1) * Er), key=lambda e: (counts[e], e))
            room = C
            quota = {}
            for e in experts:
                quota[e] = min(counts[e], room)
                room -= quota[e]
            seen = Counter()
            kept, over = [], []
            for tr in home:  # home is sorted by (e, t, k)
                if seen[tr[0]] < quota[tr[0]]:
                    kept.append(tr)
                else:
                    over.append(tr)
                seen[tr[0]] += 1
        rows[r] = [(tr[0], tr) for tr in kept]
        stream.extend(over)

    if rule == 2:
        over_n = Counter(tr[0] for tr in stream)
        stream.sort(key=lambda tr: (-over_n[tr[0]], tr[0], tr[1], tr[2]))
        walk = sorted(range(R), key=lambda r: (-(C - len(rows[r])), r))
    else:
        walk = list(range(R))
    slot_expert = [[-1] * B for _ in range(R)]
    at = 0
    failing = []
    for r in walk:
        need = C - len(rows[r])
        seg = stream[at:at + need]
        at += need
        distinct = []
        for tr in seg:
            if tr[0] not in distinct:
                distinct.append(tr[0])
        if len(distinct) > B:
            failing.append((r, len(distinct)))
            continue
        for j, e in enumerate(distinct):
            slot_expert[r][j] = e
        rows[r].extend((E + distinct.index(tr[0]), tr) for tr in seg)
    assert at == len(stream)
    if failing:
        r, n = min(failing)
        return dict(status=3, fail_rank=r, fail_slots=n, expert_count=counts,
                    rank_load=rank_load, max_count=max_count, maxvio=maxvio)

    cu = []
    dst_row = [[None] * K for _ in range(T)]
    src_of_row = [None] * (R * C)
    for r in range(R):
        assert len(rows[r]) == C
        gc = Counter(g for g, _ in rows[r])
        acc, line = 0, []
        for g in range(E + B):
            acc += gc.get(g, 0)
            line.append(acc)
        cu.append(line)
        for i, (g, (e, t, k)) in enumerate(rows[r]):
            dst_row[t][k] = r * C + i
            src_of_row[r * C + i] = t * K + k
    return dict(status=0, expert_count=counts, rank_load=rank_load, max_count=max_count,
                maxvio=maxvio, slot_expert=slot_expert, cu_seqlens=cu, dst_row=dst_row,
                src_of_row=src_of_row)


def check_plan_invariants(pl, idx, R, S, E, K, B, rule=0):
    """The invariants every successful plan must satisfy (numpy arrays from
    the oracle or the GPU).  Raises AssertionError on the first violation."""
    import numpy as np
    T, C, Er = R * S, S * K, E // R
    P = T * K
    idx = np.asarray(idx).reshape(T, K)
    dst = np.asarray(pl["dst_row"]).reshape(-1).astype(np.int64)
    src = np.asarray(pl["src_of_row"]).reshape(-1).astype(np.int64)
    cu = np.asarray(pl["cu_seqlens"]).reshape(R, E + B)
    se = np.asarray(pl["slot_expert"]).reshape(R, B)
    cnt = np.bincount(idx.reshape(-1), minlength=E)
    # every (token, k) placed exactly once, and the maps are inverse
    assert np.array_equal(np.sort(dst), np.arange(P))
    assert np.array_equal(src[dst], np.arange(P))
    # each rank holds exactly C rows; cu_seqlens is non-decreasing and ends at C
    assert np.all(cu[:, -1] == C)
    assert np.all(np.diff(cu, axis=1) >= 0) and np.all(cu[:, 0] >= 0)
    # slots used <= B, packed at the front, distinct per rank
    for r in range(R):
        used = se[r][se[r] >= 0]
        assert np.all(se[r][len(used):] == -1)
        assert len(set(used.tolist())) == len(used)
    # group membership and in-group order
    load = cnt.reshape(R, Er).sum(1)
    for r in range(R):
        start = 0
        for g in range(E + B):
            end = int(cu[r, g])
            ps = src[r * C + start: r * C + end]
            if end > start:
                e = g if g < E else int(se[r, g - E])
                assert e >= 0
                assert np.all(idx.reshape(-1)[ps] == e)
                assert np.all(np.diff(ps) > 0)
                if g < E:
                    assert g // Er == r  # home groups only hold home experts
            start = end
        if load[r] <= C:  # an under-full rank keeps all its home rows
            assert int(cu[r, (r + 1) * Er - 1] - (cu[r, r * Er - 1] if r * Er > 0 else 0)) == load[r]
    # replicas exist only for overloaded experts: the expert's home rank is
    # over-full and some of its rows sit outside its home rank
    home_rank_of_row = np.repeat(np.arange(R), C)[dst]
    for r in range(R):
        for e in se[r][se[r] >= 0]:
            e = int(e)
            assert load[e // Er] > C
            rows_e = np.nonzero(idx.reshape(-1) == e)[0]
            assert np.any(home_rank_of_row[rows_e] != e // Er)
            assert r != e // Er
