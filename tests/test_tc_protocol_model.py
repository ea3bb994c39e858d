"""A discrete-event model of the tensor-core kernel's pipeline, checked for
deadlock under random timings (CPU only).

Each CTA runs the kernel's roles as sequential programs whose steps wait on
the same conditions the kernel's barriers and flags express:
  producer  per tile: its scale copy (the tile two back must have had its
            scale factors moved to tensor memory), then one stage per
            K-chunk into the ring (a slot is free once the MMA of its previous
            stage has committed);
  MMA       per tile: the accumulator two tiles back read by the epilogue,
            this tile's scale factors in tensor memory and, for a down tile,
            its B operand built; then each stage once it has landed; the
            accumulator (and a down tile's B buffer) is released when the
            tile's last MMA completes;
  epilogue  the scale factors of tiles 0 and 1, then per tile: read the
            accumulator; a gate/up tile publishes its h (one count per expert
            it touches, GPU-wide) and then moves the scale factors of tile
            it+2; a down tile moves them and writes its outputs; after its
            last tile, the CTA's arrival on the grid count;
  gatekeeper raises each expert's flag, in order, once every tile touching
            it (on every CTA) has published;
  builders  per down tile: its expert's flag and the B buffer back from the
            tile two before;
  combine   waits for every CTA's arrival.
Gate/up tiles are dealt round robin with the kernel's tile-size formula,
down tiles (expert, pair group of <= 16, 128-row block) likewise. A state with
work left and no step able to run is a deadlock.

The publish-before-next-scale order matters: the model with the epilogue
moving tile it+2's scale factors before publishing (what the kernel once
did) deadlocks when a CTA's last gate/up tile is followed by down tiles that
fill the ring, and the test checks that the model finds it.
"""
import heapq
import random

import pytest

PAIRS_PER_TILE = 16


def schedule(G, U, upe, tu_max, pairs, RB):
    """Per CTA: list of tiles ('gu', entries) and ('dn', entry)."""
    T = U * upe
    rounds = max(1, -(-T // (G * tu_max)))
    tu = -(-T // (G * rounds))
    ntile = -(-T // tu)
    tiles = [[] for _ in range(G)]
    for t in range(ntile):
        f0, f1 = t * tu, min(T, t * tu + tu)
        tiles[t % G].append(("gu", tuple(range(f0 // upe, (f1 - 1) // upe + 1))))
    need = [0] * U
    for t in range(ntile):
        f0, f1 = t * tu, min(T, t * tu + tu)
        for u in range(f0 // upe, (f1 - 1) // upe + 1):
            need[u] += 1
    d = 0
    for u in range(U):
        for _g in range(-(-pairs[u] // PAIRS_PER_TILE)):
            for _r in range(RB):
                tiles[d % G].append(("dn", u))
                d += 1
    return tiles, need


def simulate(G, U, upe, tu_max, pairs, RB, nst_gu, nst_dn, ns, rng, old_order=False):
    tiles, need = schedule(G, U, upe, tu_max, pairs, RB)
    count = [0] * U
    grid = [0]
    st = []
    for b in range(G):
        tl = tiles[b]
        dn = [i for i, t in enumerate(tl) if t[0] == "dn"]
        stages = []  # (tile index, global stage index)
        for i, t in enumerate(tl):
            for _ in range(nst_gu if t[0] == "gu" else nst_dn):
                stages.append(i)
        st.append(dict(tl=tl, dn=dn, stages=stages, landed=set(), committed=set(), sc=set(), sf=set(),
                       acc_full=set(), acc_read=set(), b_full=set(), b_empty=set(), flag=set()))

    progs = []  # (cta, role, steps); a step is (precondition, effect)

    for b in range(G):
        s = st[b]
        tl, stages = s["tl"], s["stages"]
        # producer
        steps = []
        gs = 0
        for it in range(len(tl)):
            steps.append((lambda s=s, it=it: it < 2 or (it - 2) in s["sf"], lambda s=s, it=it: s["sc"].add(it)))
            for _ in range(nst_gu if tl[it][0] == "gu" else nst_dn):
                steps.append((lambda s=s, g=gs: g < ns or (g - ns) in s["committed"],
                              lambda s=s, g=gs: s["landed"].add(g)))
                gs += 1
        progs.append((b, "producer", steps))
        # MMA
        steps = []
        gs = 0
        for it in range(len(tl)):
            k = s["dn"].index(it) if tl[it][0] == "dn" else None
            steps.append((lambda s=s, it=it, k=k: (it < 2 or (it - 2) in s["acc_read"]) and it in s["sf"] and
                          (k is None or k in s["b_full"]), lambda: None))
            n = nst_gu if tl[it][0] == "gu" else nst_dn
            for j in range(n):
                last = j == n - 1

                def eff(s=s, g=gs, it=it, k=k, last=last):
                    s["committed"].add(g)
                    if last:
                        s["acc_full"].add(it)
                        if k is not None:
                            s["b_empty"].add(k)
                steps.append((lambda s=s, g=gs: g in s["landed"], eff))
                gs += 1
        progs.append((b, "mma", steps))
        # epilogue
        steps = []
        for it in range(min(2, len(tl))):
            steps.append((lambda s=s, it=it: it in s["sc"], lambda s=s, it=it: s["sf"].add(it)))
        for it in range(len(tl)):
            steps.append((lambda s=s, it=it: it in s["acc_full"], lambda s=s, it=it: s["acc_read"].add(it)))
            nxt = [(lambda s=s, n=it + 2: n in s["sc"], lambda s=s, n=it + 2: s["sf"].add(n))] \
                if it + 2 < len(tl) else []
            if tl[it][0] == "gu":
                def pub(ents=tl[it][1]):
                    for u in ents:
                        count[u] += 1
                publish = [(lambda: True, pub)]
                steps += (nxt + publish) if old_order else (publish + nxt)
            else:
                steps += nxt
        steps.append((lambda: True, lambda: grid.__setitem__(0, grid[0] + 1)))
        progs.append((b, "epilogue", steps))
        # gatekeeper
        steps = [(lambda u=u: count[u] == need[u], lambda s=s, u=u: s["flag"].add(u)) for u in range(U)]
        progs.append((b, "gatekeeper", steps))
        # builders
        steps = []
        for k, it in enumerate(s["dn"]):
            u = tl[it][1]
            steps.append((lambda s=s, u=u, k=k: u in s["flag"] and (k < 2 or (k - 2) in s["b_empty"]),
                          lambda s=s, k=k: s["b_full"].add(k)))
        progs.append((b, "builders", steps))
        progs.append((b, "combine", [(lambda: grid[0] == G, lambda: None)]))

    pc = [0] * len(progs)
    busy = [False] * len(progs)
    ev = []
    t = 0.0
    seq = 0
    while True:
        for i, (_b, _r, steps) in enumerate(progs):
            if not busy[i] and pc[i] < len(steps) and steps[pc[i]][0]():
                busy[i] = True
                heapq.heappush(ev, (t + rng.uniform(0.05, 1.0), seq, i))
                seq += 1
        if not ev:
            break
        t, _, i = heapq.heappop(ev)
        progs[i][2][pc[i]][1]()
        pc[i] += 1
        busy[i] = False
    stuck = [(b, r, pc[i], len(steps)) for i, (b, r, steps) in enumerate(progs) if pc[i] < len(steps)]
    return stuck


CASES = [
    # G, U, upe, tu_max, pairs per entry, RB, gate/up stages, down stages, ring slots
    (8, 8, 12, 16, [12] * 8, 3, 4, 3, 2),                          # few gate/up tiles per CTA, many down tiles
    (8, 8, 12, 16, [32] * 8, 3, 4, 4, 2),                          # two pair groups per expert
    (12, 20, 12, 16, [3, 1, 17, 2, 6, 1, 1, 9, 4, 2, 1, 5, 2, 1, 3, 7, 1, 1, 2, 4], 2, 3, 2, 3),
    (16, 5, 24, 16, [40, 8, 8, 8, 8], 4, 5, 3, 4),
    (6, 12, 8, 8, [1] * 12, 2, 2, 2, 2),
]


@pytest.mark.parametrize("case", CASES)
def test_pipeline_never_deadlocks(case):
    G, U, upe, tu_max, pairs, RB, ng, nd, ns = case
    for seed in range(20):
        stuck = simulate(G, U, upe, tu_max, pairs, RB, ng, nd, ns, random.Random(seed))
        assert not stuck, (seed, stuck[:4])


def test_model_finds_the_old_scale_factor_order_deadlock():
    """Moving tile it+2's scale factors before publishing tile it deadlocks:
    the next scale copy sits behind down stages that fill the ring and wait,
    through their B operand, for this CTA's own publish."""
    G, U, upe, tu_max, pairs, RB, ng, nd, ns = CASES[1]
    found = 0
    for seed in range(10):
        stuck = simulate(G, U, upe, tu_max, pairs, RB, ng, nd, ns, random.Random(seed), old_order=True)
        found += bool(stuck)
    assert found > 0
