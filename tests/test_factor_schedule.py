"""The factor graph's task numbering, on the CPU.

The factor kernel (csrc/factor.cu) runs the blocked Cholesky and the blocked inverse of every problem as
64x64 tile tasks that CTAs take from one global counter, in number order, and each task waits until
its inputs' tiles have reached the states it needs. That schedule is deadlock-free only if the
numbering is topological: every task a task waits on has a smaller number. This test restates the
numbering (the stage layout and class counts of stage_counts and the class decode of decode_task)
and checks:
  * run in number order, every task finds its inputs in the states it waits for, each tile update
    is applied exactly once and in order (a two-level task, which applies the updates of panels m-1
    and m to its tile together, advances it by two), and every tile ends final (L_ij: state j + 1,
    Y_ji: i - j + 1);
  * counting a two-level task as two, the graph applies the plain blocked algorithm's updates;
  * a model of the in-order ticket protocol (W CTAs, each holding a running task and the next
    number it has taken, a finished task released at once) always drains, for several W.
The same checks run on the Cholesky-only graph of the block-scaled factor F (classes F, Q and FQ
empty): L final, no Y tile beyond the diagonal tasks' touched.
"""
import math
import random

import pytest


def stage_counts(nt, s, inv=True):
    """Tasks per problem in stage s by class: [lookahead G(i,m+1,m), P(m+1), F(j,m), one-level Q,
    two-level FQ (odd m), bulk G (even m: the column m+2, one level; odd m: FG over j >= m+2, levels
    m-1 and m), S(i,m+1)] (stage 0: P(0), S(i,0)). inv=False: the Cholesky only (F, Q, FQ empty)."""
    n = [0] * 7
    if s == 0:
        n[1], n[6] = 1, nt - 1
        return n
    m = s - 1
    R = nt - 1 - m
    if R < 0:
        return n
    R1 = max(R - 1, 0)
    n[0], n[1], n[2] = R, 1 if R >= 1 else 0, m
    if m % 2 == 0:
        n[3] = (m + 1) * min(R, 2)
        n[5] = R1
    else:
        n[3] = (m + 1) * min(R, 1) + R1
        n[4] = m * R1
        n[5] = (R - 1) * R // 2 if R >= 1 else 0
    n[6] = R1
    if not inv:
        n[2] = n[3] = n[4] = 0
    return n


def decode(nt, s, c, local):
    m = s - 1
    if c == 0:
        return ("G", m, m + 1 + local, m + 1)
    if c == 1:
        return ("P", s, 0, 0)
    if c == 2:
        return ("F", m, 0, local)
    if c == 3:
        if m % 2 == 0:
            ii, j = divmod(local, m + 1)
            return ("Q", m, m + 1 + ii, j)
        if local < m + 1:
            return ("Q", m, m + 1, local)
        return ("Q", m, m + 2 + local - (m + 1), m)
    if c == 4:
        ii, j = divmod(local, m)
        return ("FQ", m, m + 2 + ii, j)
    if c == 5:
        if m % 2 == 0:
            return ("G", m, m + 2 + local, m + 2)
        # the kernel's closed form: column k = j - (m+2), the smaller root of the triangular count
        R2 = nt - m - 2
        B = 2 * R2 + 1
        k = int((B - math.sqrt(float(B * B - 8 * local))) // 2)
        cum = lambda kk: kk * R2 - kk * (kk - 1) // 2
        while k > 0 and cum(k) > local:
            k -= 1
        while cum(k + 1) <= local:
            k += 1
        j = m + 2 + k
        return ("FG", m, j + local - cum(k), j)
    return ("S", s, s + 1 + local, s)


def tasks(nt, inv=True):
    out = []
    for s in range(nt + 1):
        for c, cnt in enumerate(stage_counts(nt, s, inv)):
            out += [decode(nt, s, c, local) for local in range(cnt)]
    return out


def deps(task):
    """(tile kind, i, j, state needed) of the inputs, and (tile kind, i, j, new state) of the outputs.
    A two-level task waits for level m's operands only: they are final only after level m-1's are."""
    kind, m, i, j = task
    if kind == "P":
        return [("A", m, m, m)], [("A", m, m, m + 1), ("Y", m, m, 1)]
    if kind == "S":
        return [("A", i, m, m), ("A", m, m, m + 1)], [("A", i, m, m + 1)]
    if kind == "G":
        return [("A", i, m, m + 1), ("A", j, m, m + 1), ("A", i, j, m)], [("A", i, j, m + 1)]
    if kind == "FG":
        return [("A", i, m, m + 1), ("A", j, m, m + 1), ("A", i, j, m - 1)], [("A", i, j, m + 1)]
    if kind == "F":
        return [("Y", j, m, m - j), ("A", m, m, m + 1)], [("Y", j, m, m - j + 1)]
    if kind == "FQ":
        return [("Y", j, m, m - j + 1), ("A", i, m, m + 1), ("Y", j, i, m - 1 - j)], [("Y", j, i, m - j + 1)]
    return [("Y", j, m, m - j + 1), ("A", i, m, m + 1), ("Y", j, i, m - j)], [("Y", j, i, m - j + 1)]


def _levels(t):
    return 2 if t[0] in ("FG", "FQ") else 1


@pytest.mark.parametrize("inv", [True, False])
@pytest.mark.parametrize("nt", list(range(1, 40)))
def test_numbering_is_topological_and_complete(nt, inv):
    state = {}
    for t in tasks(nt, inv):
        ins, outs = deps(t)
        for key in ins:
            assert state.get(key[:3], 0) >= key[3], (t, key, state.get(key[:3], 0))
        for key in outs:   # each update once, in order (a two-level task applies two)
            assert state.get(key[:3], 0) == key[3] - _levels(t), (t, key)
            state[key[:3]] = key[3]
    for i in range(nt):
        for j in range(i + 1):
            assert state[("A", i, j)] == j + 1
            if inv:
                assert state[("Y", j, i)] == i - j + 1
            else:
                assert state.get(("Y", j, i), 0) == (1 if i == j else 0)


def _fg_by_walk(nt, m, local):
    """The bulk task's tiles by walking the columns (the plain definition of the numbering)."""
    rem, j = local, m + 2
    while rem >= nt - j:
        rem -= nt - j
        j += 1
    return j + rem, j


@pytest.mark.parametrize("nt", [3, 4, 17, 64, 224, 448, 1000])
def test_bulk_task_closed_form_decode(nt):
    """The closed-form decode of a two-level bulk task (a quadratic's root and a unit correction) gives
    the tiles that walking the columns gives, for every task of small graphs and a sample of large ones."""
    for m in range(1, nt, 2):
        R = nt - 1 - m
        n = (R - 1) * R // 2 if R >= 1 else 0
        step = max(1, n // 2000)
        for local in list(range(0, n, step)) + ([n - 1] if n else []):
            _, _, i, j = decode(nt, m + 1, 5, local)
            assert (i, j) == _fg_by_walk(nt, m, local), (nt, m, local)


@pytest.mark.parametrize("nt", [1, 2, 5, 16, 128])
def test_level_updates_match_the_one_level_graph(nt):
    """Counting a two-level task as two, the graph applies exactly the updates of the plain blocked
    algorithm: per problem sum_m (1 + 2R + m + (m + 1) R + (R - 1) R / 2), R = nt - 1 - m."""
    plain = sum(1 + 2 * R + m + (m + 1) * R + ((R - 1) * R // 2 if R >= 1 else 0)
                for m in range(nt) for R in [nt - 1 - m])
    assert sum(_levels(t) for t in tasks(nt)) == plain
    assert len(tasks(nt)) == sum(sum(stage_counts(nt, s)) for s in range(nt + 1))
    # the Cholesky alone: sum_m (1 + 2R + (R - 1) R / 2 + R) one-level tile updates (P, S, G)
    chol = sum(1 + 2 * R + ((R - 1) * R // 2 if R >= 1 else 0) for m in range(nt) for R in [nt - 1 - m])
    assert sum(_levels(t) for t in tasks(nt, False)) == chol


@pytest.mark.parametrize("inv", [True, False])
@pytest.mark.parametrize("n_cta", [1, 2, 7, 64])
def test_in_order_ticket_protocol_drains(n_cta, inv):
    """Several problems of two sizes interleaved (stage by stage, as the kernel numbers them); CTAs
    take numbers in order, each holds at most its running task and its next number, and a task
    starts only when its inputs are final. Random completion order; it must never stall."""
    groups = [(6, 3), (3, 2), (9, 1)]   # (nt, batch)
    numbered = []
    for s in range(max(nt for nt, _ in groups) + 1):
        for gi, (nt, batch) in enumerate(groups):
            if s > nt:
                continue
            for c, cnt in enumerate(stage_counts(nt, s, inv)):
                for local in range(cnt):
                    for b in range(batch):
                        numbered.append((gi, b, decode(nt, s, c, local)))
    rng = random.Random(n_cta)
    state, nxt = {}, 0
    held = [[] for _ in range(n_cta)]   # per CTA: [running or waiting task, next number]
    done = 0
    while done < len(numbered):
        for h in held:                   # take numbers in order
            while len(h) < 2 and nxt < len(numbered):
                h.append(nxt)
                nxt += 1
        ready = []
        for ci, h in enumerate(held):
            if h:
                gi, b, t = numbered[h[0]]
                ins, _ = deps(t)
                if all(state.get((gi, b) + k[:3], 0) >= k[3] for k in ins):
                    ready.append(ci)
        assert ready, "stalled"
        ci = rng.choice(ready)
        gi, b, t = numbered[held[ci].pop(0)]
        for k in deps(t)[1]:
            state[(gi, b) + k[:3]] = k[3]
        done += 1
