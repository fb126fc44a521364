"""Discrete-event model of the attention kernel's pipeline protocol (CPU only).

The attention kernel hands work between a TMA producer, one MMA-issuing thread per
sub-unit and two softmax warpgroups through mbarriers that are tested by phase parity.
This model replays that protocol on the unit lists of real masks under random
interleavings and checks that it always finishes (no deadlock) and that every read sees
what it should: each product the key/value tile of its entry (no stale ring stage), the
softmax S of its own block, each P.V the P of its own block, O holding exactly the blocks
before it at each P.V and rescale, and every block at the epilogue.

mbarrier semantics modelled: a phase completes when its expected arrival count is
reached; a parity test for parity P succeeds when the current phase's parity differs from
P, so a barrier two phases behind the awaited one looks complete. Each issuing thread's
products run in its issue order, and its commit arrives once the products it issued
before the commit are done; nothing orders the two issuers' products against each other.

The protocol: S-full barriers per (sub-unit, S buffer), one P-ready and one P.V-done
barrier per sub-unit, and a softmax that waits for the previous block's P.V before it
releases P (and rescales O, when the row max grew). Each sub-unit's softmax runs as four
independent warps, each with its own rows, so warps of one sub-unit may be at different
blocks. Deliberately broken variants must be
caught, which shows the checker can see the hazards: issuers that test only their own next
entries (ring stages), a softmax that releases P without that wait, an epilogue that waits
one block early, and QK products three blocks ahead of P.V.
"""
import random

import numpy as np
import pytest

import _cases as C
from oracle import bsa_oracle as O

NS = 4          # ring stages, one key tile each
WARPS = 4       # softmax warps per sub-unit; each warp's 32 threads arrive on P-ready


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
    """Work units of one (b, h): the kernel's grouping of four consecutive rows per class
    (rows retaining every key tile first), as (union list, used by A, used by B)."""
    nt = mask.shape[0]
    cnt = mask.sum(-1)
    dense = [i for i in range(nt) if cnt[i] == nt]
    local = [i for i in range(nt) if cnt[i] != nt]
    out = []
    for rows in (dense, local):
        for u0 in range(0, len(rows), 4):
            qs = rows[u0:u0 + 4] + [-1] * (4 - len(rows[u0:u0 + 4]))
            mk = [mask[q] if q >= 0 else np.zeros(nt, bool) for q in qs]
            union = np.nonzero(mk[0] | mk[1] | mk[2] | mk[3])[0]
            out.append((len(union), [bool(mk[0][j] or mk[1][j]) for j in union],
                        [bool(mk[2][j] or mk[3][j]) for j in union]))
    return out


def run_protocol(L, need_a, need_b, seed, careless=False, no_wait=False):
    """True if the unit finishes; False on deadlock; raises Stale on a wrong read.

    Besides the ring stages, the model tracks what each S buffer holds (S of block it after
    its QK product, P of block it after the softmax released it) and how many P.V
    products O has absorbed, and checks every read against them: the softmax reads S of
    its own block, a P.V reads P of its own block and adds to O holding exactly the
    blocks before it, a rescale sees O holding exactly the blocks before it, and the
    epilogue sees every block. From its second block on, a softmax waits for the previous
    P.V (then may rescale O) before it releases P.

    careless: one issuer per sub-unit that tests only its own next entries (ring hazard).
    no_wait: the softmax releases P without that wait (it can then run two P-ready phases
    ahead of the issuer).
    """
    rng = random.Random(seed)
    need = [need_a, need_b]
    has = [any(need_a), any(need_b)]
    users = sum(has)
    blk = [[i for i in range(L) if need[u][i]] for u in range(2)]
    n = [len(b) for b in blk]
    kfull, vfull = [Bar(1) for _ in range(NS)], [Bar(1) for _ in range(NS)]
    kempty = [Bar(1 if careless else users) for _ in range(NS)]
    vempty = [Bar(1 if careless else users) for _ in range(NS)]
    sfull = [Bar(1) for _ in range(4)]          # 2u + b
    pfull = [Bar(WARPS) for _ in range(2)]      # u (one arrival per warp stands for its 32)
    odone = [Bar(1) for _ in range(2)]          # u
    pipe, kload, vload = [[], []], [], []     # one product queue per issuing thread
    kdata, vdata = [None] * NS, [None] * NS
    sbuf = [[[None] * WARPS for _ in range(2)] for _ in range(2)]   # per warp's rows: ('S', it) / ('P', it)
    oblocks = [0, 0]                            # P.V products absorbed by O
    prod = [0, 'k']
    ki, vi, qc, pc = [0, 0], [0, 0], [0, 0], [0, 0]
    # one agent per softmax warp: [block, state]; each warp owns a quarter of the rows
    sm = [[[0, 'wait_s'] for _ in range(WARPS)] for _ in range(2)]

    def pbar(u, it):
        return pfull[u], it & 1

    def obar(u, it):
        return odone[u], it & 1

    def actions():
        acts = []
        i = prod[0]
        if i < L:
            s, ph = i % NS, ((i // NS) & 1) ^ 1
            if prod[1] == 'k' and kempty[s].test(ph):
                acts.append(('load_k',))
            if prod[1] == 'v' and vempty[s].test(ph):
                acts.append(('load_v',))
        if kload:
            acts.append(('tma_k',))
        if vload:
            acts.append(('tma_v',))
        for u in range(2):
            if pipe[u]:
                acts.append(('pipe', u))
        for u in range(2):
            if not has[u]:
                continue
            if careless:
                if qc[u] < n[u] and qc[u] - pc[u] < 2:
                    e = blk[u][qc[u]]
                    if kfull[e % NS].test((e // NS) & 1):
                        acts.append(('qk', u))
                bar, par = pbar(u, pc[u])
                if pc[u] < qc[u] and bar.test(par):
                    e = blk[u][pc[u]]
                    if vfull[e % NS].test((e // NS) & 1):
                        acts.append(('pv', u))
            else:
                k = ki[u]
                if k < L and kfull[k % NS].test((k // NS) & 1):
                    if not need[u][k]:
                        acts.append(('k_arrive', u))
                    elif qc[u] - pc[u] < 2:
                        acts.append(('qk', u))
                v = vi[u]
                if v < ki[u] and vfull[v % NS].test((v // NS) & 1):
                    if not need[u][v]:
                        acts.append(('v_arrive', u))
                    else:
                        bar, par = pbar(u, pc[u])
                        if bar.test(par):
                            acts.append(('pv', u))
            for w in range(WARPS):
                it, st = sm[u][w]
                if it < n[u]:
                    if st == 'wait_s' and sfull[2 * u + (it & 1)].test((it >> 1) & 1):
                        acts.append(('softmax_s', u, w))
                    if st == 'wait_o':
                        bar, par = obar(u, it - 1)
                        if bar.test(par):
                            acts.append(('softmax_rescale', u, w))
                    if st == 'release':
                        acts.append(('softmax_p', u, w))
                elif st != 'done':
                    bar, par = obar(u, n[u] - 1)
                    if n[u] == 0 or bar.test(par):
                        acts.append(('epilogue', u, w))
        return acts

    def last_user(u, e, cursor):
        o = 1 - u
        return not need[o][e] or not has[o] or cursor[o] >= n[o] or blk[o][cursor[o]] > e

    while True:
        acts = actions()
        finished = (prod[0] >= L and all(sm[u][w][1] == 'done' or not has[u] for u in range(2) for w in range(WARPS))
                    and all(pc[u] >= n[u] for u in range(2)))
        if finished and not pipe[0] and not pipe[1] and not kload and not vload:
            return True
        if not acts:
            return False
        a = rng.choice(acts)
        kind = a[0]
        if kind == 'load_k':
            kload.append((prod[0] % NS, prod[0]))
            prod[1] = 'v'
        elif kind == 'load_v':
            vload.append((prod[0] % NS, prod[0]))
            prod[1] = 'k'
            prod[0] += 1
        elif kind == 'tma_k':
            s, e = kload.pop(0)
            kdata[s] = e
            kfull[s].arrive()
        elif kind == 'tma_v':
            s, e = vload.pop(0)
            vdata[s] = e
            vfull[s].arrive()
        elif kind == 'pipe':
            op = pipe[a[1]].pop(0)
            if op[0] == 'commit':
                op[1].arrive()
            elif op[0] == 'qk':
                _, u, it, s, e = op
                if kdata[s] != e:
                    raise Stale(f"QK of entry {e} read K stage {s} holding {kdata[s]}")
                if it >= 2 and oblocks[u] < it - 1:
                    raise Stale(f"S of block {it} overwrote P of block {it - 2} before its P.V")
                sbuf[u][it & 1] = [('S', it)] * WARPS
            else:
                _, u, it, s, e = op
                if vdata[s] != e:
                    raise Stale(f"P.V of entry {e} read V stage {s} holding {vdata[s]}")
                if sbuf[u][it & 1] != [('P', it)] * WARPS:
                    raise Stale(f"P.V of block {it} read {sbuf[u][it & 1]}")
                if oblocks[u] != it:
                    raise Stale(f"P.V of block {it} added to O holding {oblocks[u]} blocks")
                oblocks[u] += 1
        elif kind == 'qk':
            u = a[1]
            e = blk[u][qc[u]]
            s = e % NS
            pipe[u] += [('qk', u, qc[u], s, e), ('commit', sfull[2 * u + (qc[u] & 1)])]
            qc[u] += 1
            if careless:
                if last_user(u, e, qc):
                    pipe[u].append(('commit', kempty[s]))
            else:
                pipe[u].append(('commit', kempty[s]))
                ki[u] += 1
        elif kind == 'k_arrive':
            u = a[1]
            kempty[ki[u] % NS].arrive()
            ki[u] += 1
        elif kind == 'pv':
            u = a[1]
            e = blk[u][pc[u]]
            s = e % NS
            pipe[u] += [('pv', u, pc[u], s, e), ('commit', obar(u, pc[u])[0])]
            pc[u] += 1
            if careless:
                if last_user(u, e, pc):
                    pipe[u].append(('commit', vempty[s]))
            else:
                pipe[u].append(('commit', vempty[s]))
                vi[u] += 1
        elif kind == 'v_arrive':
            u = a[1]
            vempty[vi[u] % NS].arrive()
            vi[u] += 1
        elif kind == 'softmax_s':
            u, w = a[1], a[2]
            it = sm[u][w][0]
            if sbuf[u][it & 1][w] != ('S', it):
                raise Stale(f"softmax warp {w} of block {it} read {sbuf[u][it & 1][w]}")
            sm[u][w][1] = 'wait_o' if it > 0 and not no_wait else 'release'
        elif kind == 'softmax_rescale':
            u, w = a[1], a[2]
            if oblocks[u] != sm[u][w][0]:
                raise Stale(f"rescale at block {sm[u][w][0]} saw O holding {oblocks[u]} blocks")
            sm[u][w][1] = 'release'
        elif kind == 'softmax_p':
            u, w = a[1], a[2]
            it = sm[u][w][0]
            sbuf[u][it & 1][w] = ('P', it)
            bar, _ = pbar(u, it)
            bar.arrive()
            sm[u][w] = [it + 1, 'wait_s']
        elif kind == 'epilogue':
            u, w = a[1], a[2]
            if oblocks[u] != n[u]:
                raise Stale(f"epilogue read O holding {oblocks[u]} of {n[u]} blocks")
            sm[u][w][1] = 'done'


def _case_units(name):
    w, q, k, v, diff = C.inputs(name)
    ref = C.oracle_mask(w, O.reorder(O.to_f64(q), w.T, w.Hs, w.Ws),
                        O.reorder(O.to_f64(k), w.T, w.Hs, w.Ws), diff.numpy())
    m = ref["mask"]
    return [u for b in range(m.shape[0]) for h in range(m.shape[1]) for u in units_from_mask(m[b, h])]


@pytest.mark.parametrize("name", ["tiny", "tiny_ragged", "small128", "ragged128", "budget128"])
def test_two_issuer_protocol_finishes_and_reads_the_right_tiles(name):
    for L, na, nb in _case_units(name):
        for seed in range(12):
            assert run_protocol(L, na, nb, seed), (name, L, seed)


def test_random_sparse_unit_lists():
    rng = np.random.default_rng(7)
    for trial in range(150):
        L = int(rng.integers(1, 40))
        na = list(rng.random(L) < rng.uniform(0.1, 0.9))
        nb = list(rng.random(L) < rng.uniform(0.1, 0.9))
        for j in range(L):                       # every union entry has a user
            if not (na[j] or nb[j]):
                (na if rng.random() < 0.5 else nb)[j] = True
        if trial % 5 == 0:                       # units without a second sub-unit
            na, nb = [True] * L, [False] * L
        for seed in range(4):
            assert run_protocol(L, na, nb, seed), (trial, L, seed)


def test_careless_protocol_is_caught():
    """Testing only a sub-unit's own next entries lets it run two ring phases ahead of
    the producer: the checker must report a deadlock or a stale-tile read."""
    caught = 0
    for L, na, nb in _case_units("budget128"):
        for seed in range(12):
            try:
                caught += not run_protocol(L, na, nb, seed, careless=True)
            except Stale:
                caught += 1
    assert caught > 0


def test_release_without_waiting_is_caught():
    """Without the wait for the previous P.V, a softmax can complete two phases of its
    single P-ready barrier before the issuer tests the first: the parity test aliases, and
    the checker must report a deadlock or a wrong read."""
    caught = 0
    for L, na, nb in _case_units("budget128"):
        for seed in range(12):
            try:
                caught += not run_protocol(L, na, nb, seed, no_wait=True)
            except Stale:
                caught += 1
    assert caught > 0


@pytest.mark.parametrize("mutation", ["epilogue_one_block_early", "qk_three_blocks_ahead"])
def test_broken_waits_are_caught(mutation):
    """The same checker on two one-line mistakes: an epilogue that waits for the last P.V
    but one, and QK products allowed three blocks ahead of P.V (S would overwrite P before
    its product)."""
    import inspect
    import textwrap
    src = inspect.getsource(run_protocol)
    a, b = {
        "epilogue_one_block_early": ("bar, par = obar(u, n[u] - 1)", "bar, par = obar(u, max(n[u] - 2, 0))"),
        "qk_three_blocks_ahead": ("elif qc[u] - pc[u] < 2:", "elif qc[u] - pc[u] < 3:"),
    }[mutation]
    assert a in src
    ns = dict(globals())
    exec(textwrap.dedent(src.replace(a, b)), ns)
    caught = 0
    for L, na, nb in _case_units("budget128"):
        for seed in range(12):
            try:
                caught += not ns["run_protocol"](L, na, nb, seed)
            except Stale:
                caught += 1
    assert caught > 0
