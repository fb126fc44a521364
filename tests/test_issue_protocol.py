"""Discrete-event model of the persistent attention kernel's pipeline protocol (CPU only).

The attention kernel hands work between a key-stream builder, two TMA producers (Q and
the K ring; the V ring), two MMA-issuing threads (one per query block, A and B) and two
softmax warpgroups of four warps, through mbarriers that are tested by phase parity. Units follow one another
inside a CTA without a barrier between them. This model replays that protocol on
sequences of units taken from real masks (and on edge cases: a missing query block, query
tiles that retain nothing, odd stream lengths) under random interleavings, and checks that
it always finishes (no deadlock) and that every read sees what it should:

  * each Q K^T product the Q of its own unit and the K tile of its own stream position;
  * each softmax warp the S of its own block, in the S buffer the block went to;
  * each P.V the P of its own block, the V tile of its block, and O holding exactly the
    unit's earlier blocks (the unit's first P.V overwrites O);
  * each rescale O holding exactly the unit's earlier blocks (the softmax waits for the
    previous block's P.V; the one before has completed, since this block's Q K^T went to
    the pipe after it);
  * each epilogue O holding every block of the unit;
  * the next unit's first P.V only after every warp has read O in the epilogue.

mbarrier semantics modelled: a phase completes when its expected arrival count is
reached; a parity test for parity P succeeds when the current phase's parity differs from
P (a barrier two phases behind the awaited one looks complete). Each issuing thread's
products run in its own issue order, the two threads' products interleave arbitrarily,
and a commit arrives once the products its thread issued before it are done. TMA loads
land at a random later time and write their stage when they land.

Deliberately broken variants must be caught, which shows the checker can see the
hazards: a stage reloaded after one issuer's release instead of both, a Q K^T into an S buffer whose
P.V is still pending (overwriting P), a P.V issued before its softmax released P, Q
released at the unit's first product, a rescale without its wait, and an epilogue that
does not wait for the last P.V.
"""
import random

import numpy as np
import pytest

import _cases as C
from oracle import bsa_oracle as O

NS = 4          # ring stages (one key tile each)
WARPS = 4       # softmax warps per query block


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.k = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.k += 1
            self.pending = self.count

    def test(self, parity):
        return (self.k & 1) != parity


class Stale(Exception):
    pass


def units_from_mask(mask):
    """The kernel's units of one (b, h) (dense rows four at a time, then local rows), as
    (q tuple, per-stream-entry retention flags [4 bools]) sorted by decreasing cost."""
    nt = mask.shape[0]
    cnt = mask.sum(-1)
    dense = [i for i in range(nt) if cnt[i] == nt]
    local = [i for i in range(nt) if cnt[i] != nt]
    out = []
    for rows in (dense, local):
        for u0 in range(0, len(rows), 4):
            qs = rows[u0:u0 + 4] + [-1] * (4 - len(rows[u0:u0 + 4]))
            out.append(unit_from_rows(qs, [mask[q] if q >= 0 else np.zeros(nt, bool) for q in qs]))
    out.sort(key=lambda u: -cost(u))
    return out


def unit_from_rows(qs, rows):
    union = np.nonzero(rows[0] | rows[1] | rows[2] | rows[3])[0]
    return (tuple(qs), [[bool(rows[t][j]) for t in range(4)] for j in union])


def cost(unit):
    qs, ent = unit
    return sum(e[0] or e[1] for e in ent) + sum(e[2] or e[3] for e in ent)


def used(ent, c, x):
    return ent[c][2 * x] or ent[c][2 * x + 1]


def run_protocol(units, seed, early_release=False, qk_before_pv=False, early_q=False,
                 no_pfull_wait=False, no_epilogue_wait=False, no_rescale_wait=False):
    """True if every unit finishes; False on deadlock; raises Stale on a wrong read."""
    rng = random.Random(seed)
    nunits = len(units)
    # ------------------------------------------------------------------ barriers
    releases = 1 if early_release else 2        # stage releases before a reload: one per issuer
    kfull, kempty = [Bar(1) for _ in range(NS)], [Bar(releases) for _ in range(NS)]
    vfull, vempty = [Bar(1) for _ in range(NS)], [Bar(releases) for _ in range(NS)]
    qfull, qempty = [Bar(1), Bar(1)], [Bar(1), Bar(1)]
    sfull = [[Bar(1), Bar(1)] for _ in range(2)]            # [query block][S buffer]
    pfull = [[Bar(WARPS), Bar(WARPS)] for _ in range(2)]
    odone = [[Bar(1), Bar(1)] for _ in range(2)]
    lfull, lempty = [Bar(1), Bar(1)], [Bar(2 + 2 + 2 * WARPS), Bar(2 + 2 + 2 * WARPS)]
    # ------------------------------------------------------------------ state
    lists = [None, None]                      # key-stream buffers: unit index or 'end'
    kdata, vdata, qdata = [None] * NS, [None] * NS, [None, None]
    sbuf = [[[None] * WARPS for _ in range(2)] for _ in range(2)]  # [x][buffer][warp]: ('S'|'P', unit, block)
    obuf = [[None, 0], [None, 0]]             # (unit, blocks absorbed)
    epi_done = [[-1] * WARPS for _ in range(2)]   # last unit whose epilogue each warp finished
    inflight = []                             # TMA loads: (barrier, apply)
    pipes = [[], []]                          # per issuer: products / commits in issue order

    bld = {"it": 0, "next": 0, "done": False}
    # two producers: K (Q of each query block, then the K ring) and V (the V ring)
    prods = [{"kind": kind, "it": 0, "state": "list", "unit": None, "c": 0, "qn": [0, 0], "n": 0, "x": 0,
              "done": False} for kind in ("k", "v")]

    def new_cursor():
        return {"it": 0, "have": False, "done": False, "unit": None, "kc": 0, "vc": 0,
                "hasq": False, "qready": False, "qrel": False, "first": True, "gbase": 0, "qn": 0,
                "qk": 0, "pv": 0, "ent": [-1, -1], "nb": 0}
    cur = [new_cursor(), new_cursor()]
    sm = [[{"it": 0, "state": "list", "unit": None, "c": 0, "sidx": 0, "nused": 0, "blocks": 0,
            "done": False} for _ in range(WARPS)] for _ in range(2)]

    def enqueue(x, kind, **kw):
        pipes[x].append(dict(kind=kind, x=x, **kw))

    def unit_of(buf):
        return lists[buf]

    def nblocks(ui):
        return len(units[ui][1])

    # ------------------------------------------------------------------ agents
    def builder_actions():
        if bld["done"]:
            return []
        it = bld["it"]
        buf = it & 1
        if it >= 2 and not lempty[buf].test(((it >> 1) - 1) & 1):
            return []

        def act():
            if bld["next"] >= nunits:
                lists[buf] = "end"
                bld["done"] = True
            else:
                lists[buf] = bld["next"]
                bld["next"] += 1
            lfull[buf].arrive()
            bld["it"] += 1
        return [act]

    def producer_actions(p):
        if p["done"]:
            return []
        if p["state"] == "list":
            buf = p["it"] & 1
            if not lfull[buf].test((p["it"] >> 1) & 1):
                return []

            def act():
                ui = unit_of(buf)
                if ui == "end":
                    p["done"] = True
                    return
                p["unit"], p["x"], p["c"] = ui, 0, 0
                p["state"] = "q" if p["kind"] == "k" else "ring"
            return [act]
        ui = p["unit"]
        qs, ent = units[ui]
        if p["state"] == "q":
            x = p["x"]
            if x == 2:
                def act():
                    p["state"] = "ring"
                return [act]
            if qs[2 * x] < 0:
                def act():
                    p["x"] += 1
                return [act]
            if p["qn"][x] > 0 and not qempty[x].test((p["qn"][x] - 1) & 1):
                return []

            def act():
                inflight.append((qfull[x], lambda x=x, ui=ui: qdata.__setitem__(x, ui)))
                p["qn"][x] += 1
                p["x"] += 1
            return [act]
        nb = nblocks(ui)
        if p["c"] == nb:
            def act():
                lempty[p["it"] & 1].arrive()
                p["it"] += 1
                p["state"] = "list"
            return [act]
        s, ph = p["n"] % NS, ((p["n"] // NS) & 1) ^ 1
        empty, full, data = (kempty, kfull, kdata) if p["kind"] == "k" else (vempty, vfull, vdata)
        if not empty[s].test(ph):
            return []

        def act():
            tag = (ui, p["c"])
            inflight.append((full[s], lambda s=s, tag=tag: data.__setitem__(s, tag)))
            p["n"] += 1
            p["c"] += 1
        return [act]

    def release(empty, x, gi, issued):
        # after a product on the stage, a commit (arrives once the product is done);
        # a tile passed without a product is released at once
        if issued:
            enqueue(x, "commit", bar=empty[gi % NS])
        else:
            empty[gi % NS].arrive()

    def cursor_actions(x):
        cu = cur[x]
        if cu["done"]:
            return []
        acts = []
        if not cu["have"]:
            buf = cu["it"] & 1
            if lfull[buf].test((cu["it"] >> 1) & 1):
                def act():
                    ui = unit_of(buf)
                    if ui == "end":
                        cu["done"] = True
                        return
                    cu.update(have=True, unit=ui, kc=0, vc=0, hasq=units[ui][0][2 * x] >= 0,
                              qready=False, qrel=False, first=True, nb=nblocks(ui))
                acts.append(act)
            return acts
        ui = cu["unit"]
        qs, ent = units[ui]
        nb = cu["nb"]
        if cu["vc"] < cu["kc"]:
            c = cu["vc"]
            gi = cu["gbase"] + c
            s, fph = gi % NS, (gi // NS) & 1
            pending = cu["pv"] != cu["qk"] and c == cu["ent"][cu["pv"] & 1]
            if pending:
                b = cu["pv"] & 1
                ok = (no_pfull_wait or pfull[x][b].test((cu["pv"] >> 1) & 1)) and vfull[s].test(fph)
            else:
                ok = vfull[s].test(fph)
            if ok:
                def act(c=c, gi=gi, s=s, pending=pending):
                    if pending:
                        b = cu["pv"] & 1
                        enqueue(x, "pv", unit=ui, block=c, stage=s, buf=b, first=cu["first"])
                        enqueue(x, "commit", bar=odone[x][b])
                        cu["first"] = False
                        cu["pv"] += 1
                    release(vempty, x, gi, pending)
                    cu["vc"] += 1
                acts.append(act)
        if cu["kc"] < nb:
            c = cu["kc"]
            u = used(ent, c, x) if cu["hasq"] else False
            gi = cu["gbase"] + c
            s, fph = gi % NS, (gi // NS) & 1
            qok = cu["qready"] or qfull[x].test(cu["qn"] & 1)
            if not u:
                ok = kfull[s].test(fph)
            else:
                ok = (cu["qk"] - cu["pv"] < (3 if qk_before_pv else 2)) and qok and kfull[s].test(fph)
            if ok:
                def act(u=u, c=c, gi=gi, s=s):
                    if u:
                        cu["qready"] = True
                        b = cu["qk"] & 1
                        enqueue(x, "qk", unit=ui, block=c, stage=s, buf=b)
                        enqueue(x, "commit", bar=sfull[x][b])
                        cu["ent"][b] = c
                        cu["qk"] += 1
                        if early_q and not cu["qrel"]:
                            enqueue(x, "commit", bar=qempty[x])
                            cu["qrel"] = True
                    release(kempty, x, gi, u)
                    cu["kc"] += 1
                    if cu["kc"] == nb and cu["hasq"] and cu["qready"] and not cu["qrel"]:
                        enqueue(x, "commit", bar=qempty[x])
                        cu["qrel"] = True
                acts.append(act)
        if cu["kc"] == nb and cu["vc"] == nb:
            if not cu["hasq"] or cu["qrel"] or cu["qready"] or qfull[x].test(cu["qn"] & 1):
                def act():
                    if cu["hasq"] and not cu["qrel"]:
                        enqueue(x, "commit", bar=qempty[x])
                        cu["qrel"] = True
                    if cu["hasq"]:
                        cu["qn"] += 1
                    lempty[cu["it"] & 1].arrive()
                    cu["it"] += 1
                    cu["have"] = False
                    cu["gbase"] += nb
                acts.append(act)
        return acts

    def pipe_actions(pipe):
        if not pipe:
            return []

        def act():
            op = pipe.pop(0)
            k = op["kind"]
            if k == "commit":
                op["bar"].arrive()
            elif k == "qk":
                x, ui, c, s = op["x"], op["unit"], op["block"], op["stage"]
                if qdata[x] != ui:
                    raise Stale(f"QK of unit {ui} reads Q of {qdata[x]}")
                if kdata[s] != (ui, c):
                    raise Stale(f"QK of {(ui, c)} reads K {kdata[s]}")
                b = op["buf"]
                for w in range(WARPS):
                    if sbuf[x][b][w] is not None and sbuf[x][b][w][0] == "S":
                        raise Stale(f"S of {sbuf[x][b][w][1:]} overwritten before its softmax read it")
                    sbuf[x][b][w] = ("S", ui, c)
            else:
                x, ui, c, s = op["x"], op["unit"], op["block"], op["stage"]
                if vdata[s] != (ui, c):
                    raise Stale(f"PV of {(ui, c)} reads V {vdata[s]}")
                b = op["buf"]
                for w in range(WARPS):
                    if sbuf[x][b][w] != ("P", ui, c):
                        raise Stale(f"PV of {(ui, c)} reads {sbuf[x][b][w]} (warp {w})")
                if op["first"]:
                    if any(epi_done[x][w] < (obuf[x][0] if obuf[x][0] is not None else -1)
                           for w in range(WARPS)):
                        raise Stale("O overwritten before every warp read the previous unit's O")
                    obuf[x] = [ui, 1]
                else:
                    if obuf[x][0] != ui or obuf[x][1] != op["ordinal_in_unit"]:
                        raise Stale(f"PV of {(ui, c)} adds to O {obuf[x]}")
                    obuf[x][1] += 1
        return [act]

    def softmax_actions(x, w):
        st = sm[x][w]
        if st["done"]:
            return []
        if st["state"] == "list":
            buf = st["it"] & 1
            if not lfull[buf].test((st["it"] >> 1) & 1):
                return []

            def act():
                ui = unit_of(buf)
                if ui == "end":
                    st["done"] = True
                    return
                st.update(unit=ui, c=0, nused=0, blocks=0, state="blocks")
            return [act]
        ui = st["unit"]
        qs, ent = units[ui]
        nb = nblocks(ui)
        if st["state"] == "blocks":
            while st["c"] < nb and (qs[2 * x] < 0 or not used(ent, st["c"], x)):
                st["c"] += 1
            if st["c"] == nb:
                def act():
                    lempty[st["it"] & 1].arrive()
                    st["state"] = "epi"
                return [act]
            b = st["sidx"] & 1
            if not sfull[x][b].test((st["sidx"] >> 1) & 1):
                return []

            def act(b=b):
                c = st["c"]
                if sbuf[x][b][w] != ("S", ui, c):
                    raise Stale(f"softmax {(ui, c)} reads {sbuf[x][b][w]}")
                st["state"] = "resc" if (st["nused"] > 0 and rng.random() < 0.3) else "release"
            return [act]
        if st["state"] == "resc":
            pb = (st["sidx"] - 1) & 1
            if not no_rescale_wait and not odone[x][pb].test(((st["sidx"] - 1) >> 1) & 1):
                return []

            def act():
                if obuf[x] != [ui, st["nused"]]:
                    raise Stale(f"rescale in {(ui, st['c'])} sees O {obuf[x]}")
                st["state"] = "release"
            return [act]
        if st["state"] == "release":
            def act():
                b = st["sidx"] & 1
                sbuf[x][b][w] = ("P", ui, st["c"])
                pfull[x][b].arrive()
                st["sidx"] += 1
                st["nused"] += 1
                st["c"] += 1
                st["state"] = "blocks"
            return [act]
        # epilogue
        pb = (st["sidx"] - 1) & 1
        if st["nused"] > 0 and not no_epilogue_wait and not odone[x][pb].test(((st["sidx"] - 1) >> 1) & 1):
            return []

        def act():
            if st["nused"] > 0 and obuf[x] != [ui, st["nused"]]:
                raise Stale(f"epilogue of unit {ui} sees O {obuf[x]}")
            epi_done[x][w] = ui
            st["it"] += 1
            st["state"] = "list"
        return [act]

    # PV ordinals inside a unit: filled at enqueue time from the cursor's count in the unit
    unit_pv = {}

    def fix_ordinals():
        for op in pipes[0] + pipes[1]:
            if op["kind"] == "pv" and "ordinal_in_unit" not in op:
                key = (op["x"], op["unit"])
                op["ordinal_in_unit"] = unit_pv.get(key, 0)
                unit_pv[key] = op["ordinal_in_unit"] + 1

    for _ in range(2_000_000):
        fix_ordinals()
        acts = builder_actions() + producer_actions(prods[0]) + producer_actions(prods[1]) + \
            cursor_actions(0) + cursor_actions(1) + pipe_actions(pipes[0]) + pipe_actions(pipes[1])
        for x in range(2):
            for w in range(WARPS):
                acts += softmax_actions(x, w)
        if inflight:
            def land():
                i = rng.randrange(len(inflight))
                b, apply = inflight.pop(i)
                apply()
                b.arrive()
            acts.append(land)
        if not acts:
            done = bld["done"] and all(p["done"] for p in prods) and all(c["done"] for c in cur) and \
                all(s["done"] for xs in sm for s in xs) and not pipes[0] and not pipes[1] and not inflight
            return done
        rng.choice(acts)()
    raise AssertionError("model did not terminate")


def _mask_units(name, heads=2, **over):
    w, q, k, v, diff = C.inputs(name, tuple(over.items()))
    qt64, kt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k))
    m = C.oracle_mask(w, qt64[:, :heads], kt64[:, :heads], diff.numpy())["mask"]
    out = []
    for h in range(heads):
        out += units_from_mask(m[0, h])
    return out


def _edge_units():
    nt = 9
    rng = np.random.default_rng(3)
    rows = [rng.random(nt) < 0.4 for _ in range(4)]
    empty = np.zeros(nt, bool)
    one = np.zeros(nt, bool)
    one[4] = True
    return [
        unit_from_rows((0, 1, 2, 3), rows),                       # random rows
        unit_from_rows((0, 1, -1, -1), [rows[0], rows[1], empty, empty]),   # no query block B
        unit_from_rows((0, -1, -1, -1), [one, empty, empty, empty]),        # one tile, one key tile
        unit_from_rows((0, 1, 2, 3), [empty, empty, rows[2], rows[3]]),     # A retains nothing
        unit_from_rows((0, 1, 2, 3), [one, empty, empty, one]),             # odd stream, shared tile
        unit_from_rows((0, 1, 2, -1), [~empty, ~empty, ~empty, empty]),     # dense rows
    ]


@pytest.mark.parametrize("seed", range(6))
def test_protocol_on_real_mask_units(seed):
    units = _mask_units("small128")
    rng = random.Random(seed)
    pick = units[:]
    rng.shuffle(pick)
    assert run_protocol(pick[:10], seed)


@pytest.mark.parametrize("seed", range(8))
def test_protocol_on_edge_units(seed):
    units = _edge_units()
    rng = random.Random(100 + seed)
    seq = [units[rng.randrange(len(units))] for _ in range(8)]
    assert run_protocol(seq, seed)


@pytest.mark.parametrize("seed", range(3))
def test_protocol_budget_units(seed):
    units = _mask_units("budget128", heads=1)
    assert run_protocol(units[:8], seed)


def _catches(**broken):
    units = _mask_units("small128")[:6] + _edge_units()
    for seed in range(40):
        try:
            if not run_protocol(units, seed, **broken):
                return True
        except Stale:
            return True
    return False


def test_model_catches_early_stage_release():
    assert _catches(early_release=True)


def test_model_catches_qk_before_pv():
    assert _catches(qk_before_pv=True)


def test_model_catches_early_q_release():
    assert _catches(early_q=True)


def test_model_catches_pv_before_p():
    assert _catches(no_pfull_wait=True)


def test_model_catches_epilogue_without_wait():
    assert _catches(no_epilogue_wait=True)


def test_model_catches_rescale_without_wait():
    assert _catches(no_rescale_wait=True)
