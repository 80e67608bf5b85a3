"""Model check of the Cholesky + inverse kernel's dataflow schedule (host logic, no GPU).

The cooperative kernel (csrc/chol.cu) orders its tile tasks through per-tile counters.
This test restates its task lists -- CTA 0's critical chain, CTA 1's helper tasks and the
round-robin pool of CTAs 2.. with the L^-1 tasks one step behind -- with the counter each
task waits for and the counter it advances, and executes them: each CTA takes its own
tasks in order, a task may run only when every counter it waits on has exactly the value
it names (exact, not just "at least", so that no update can be applied twice or out of
order), and the run must finish for every block count up to 64 (r <= 4096) and several
grid sizes.  At the end every tile of L has seen its k updates plus its Cholesky or panel
solve, and every tile of L^-1 below the diagonal its updates plus its finalisation.
"""
import pytest


def _tasks(nb, G):
    """Per-CTA task lists: (waits [(counter, value)], effects [(counter, inc)], name)."""
    C = lambda i, k: ("L", i, k)          # noqa: E731
    I = lambda i, k: ("I", i, k)          # noqa: E731
    q = [[] for _ in range(G)]
    # CTA 0: Cholesky of (0, 0), then per step j: panel (j+1, j), look-ahead + Cholesky
    q[0].append(([], [(C(0, 0), 1)], "chol 0"))
    for j in range(nb - 1):
        q[0].append(([(C(j + 1, j), j), (C(j + 1, j + 1), j)], [(C(j + 1, j), 1)],
                     f"panel {j+1},{j}"))
        q[0].append(([], [(C(j + 1, j + 1), 2)], f"lookahead+chol {j+1}"))
    # CTA 1: panel (j+2, j), then the step-j updates of (j+2, j+1) and (j+2, j+2)
    for j in range(nb - 2):
        q[1].append(([(C(j, j), j + 1), (C(j + 2, j), j)], [(C(j + 2, j), 1)],
                     f"helper panel {j+2},{j}"))
        q[1].append(([(C(j + 1, j), j + 1), (C(j + 2, j + 1), j), (C(j + 2, j + 2), j)],
                     [(C(j + 2, j + 1), 1), (C(j + 2, j + 2), 1)], f"helper upd {j}"))
    # CTAs 2..: round-robin over the global task order
    W = G - 2
    base = 0
    for sj in range(nb + 1):
        jf = sj if sj < nb else -1
        ji = sj - 1
        Tf = nb - 1 - jf if jf >= 0 else 0
        P = Tf - 2 if Tf > 1 else 0
        U = Tf * (Tf + 1) // 2 - 3 if Tf > 1 else 0
        Ti = nb - 1 - ji if ji >= 0 else 0
        F = ji if ji >= 0 else 0
        V = (ji + 1) * Ti if ji >= 0 else 0
        n = P + U + F + V
        for loc in range(n):
            w = (base + loc) % W
            if loc < P:
                j, i = jf, jf + 3 + loc
                task = ([(C(j, j), j + 1), (C(i, j), j)], [(C(i, j), 1)], f"panel {i},{j}")
            elif loc < P + U:
                j = jf
                idx = loc - P + 3
                a = 0
                while (a + 1) * (a + 2) // 2 <= idx:
                    a += 1
                ii, kk = a, idx - a * (a + 1) // 2
                i, k = j + 1 + ii, j + 1 + kk
                task = ([(C(i, j), j + 1), (C(k, j), j + 1), (C(i, k), j)], [(C(i, k), 1)],
                        f"upd {i},{k} step {j}")
            elif loc < P + U + F:
                j, m = ji, loc - P - U
                task = ([(I(j, m), j - m), (C(j, j), j + 1)], [(I(j, m), 1)], f"fin {j},{m}")
            else:
                j = ji
                v = loc - P - U - F
                m, i = v // Ti, j + 1 + v % Ti
                waits = [(C(i, j), j + 1)]
                waits += [(I(j, m), j - m + 1), (I(i, m), j - m)] if m < j else [(C(j, j), j + 1)]
                task = (waits, [(I(i, m), 1)], f"inv upd {i},{m} step {j}")
            q[2 + w].append(task)
        base += n
    return q


def _run(nb, G):
    q = _tasks(nb, G)
    cnt = {}
    pos = [0] * G
    done = 0
    total = sum(len(x) for x in q)
    progress = True
    while progress:
        progress = False
        for c in range(G):
            while pos[c] < len(q[c]):
                waits, effects, name = q[c][pos[c]]
                if not all(cnt.get(k, 0) == v for k, v in waits):
                    # a wait may only ever be short of its value, never past it
                    for k, v in waits:
                        assert cnt.get(k, 0) <= v or k[0] == "L" and k[1] == k[2], (name, k)
                    break
                for k, inc in effects:
                    cnt[k] = cnt.get(k, 0) + inc
                pos[c] += 1
                done += 1
                progress = True
    assert done == total, f"deadlock at nb={nb}, G={G}: {done}/{total} tasks"
    return cnt


@pytest.mark.parametrize("G", [3, 4, 7, 148])
@pytest.mark.parametrize("nb", [1, 2, 3, 4, 5, 8, 17, 32, 64])
def test_schedule_completes_with_exact_counts(nb, G):
    cnt = _run(nb, G)
    for i in range(nb):
        for k in range(i + 1):
            assert cnt.get(("L", i, k), 0) == k + 1, ("L", i, k)
        for m in range(i):
            assert cnt.get(("I", i, m), 0) == i - m + 1, ("I", i, m)
