"""A model of the forward kernel's synchronisation, run on the CPU.

The agents follow fwd_kernel's code: the TMA producer (per-warpgroup release
barriers), the MMA issuer (polling at d = 64 with separate P columns,
fixed order with flushes at d = 128 with P over S) and the two softmax
warpgroups. mbarriers are modelled by their completed-phase count and the
hardware's one-bit parity test; TMA landings and MMA completions are
asynchronous events (MMAs complete in issue order, like the tensor pipe).
Random interleavings are explored on the workloads' key schedules and on
random ones. Checked:

* no deadlock: some agent can always move until all are done;
  (schedules: the SD3-1024-like arrow CTAs, C3-like pooled top-30% CTAs,
  random ones with long per-warpgroup gaps)
* no stale data: every QK^T / PV finds its own tile in the K / V stage it
  reads, no stage is reloaded while an issued MMA still reads it, and the
  softmax never overwrites P that a pending PV reads.

The producer's K and V loads run as two independent agents (one lane each).
Three planted mistakes must be caught: the fixed order without the
cross-warpgroup PV order the split producer needs, the fixed order without
the flushes an earlier single-loop producer needed, and the polling issuer
testing K without walking the tiles in order.
"""
import random

import numpy as np
import pytest

from oracle import masks as OM


class Bar:
    def __init__(self, count=1):
        self.count, self.arrived, self.done = count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count
        if self.arrived == self.count:
            self.arrived, self.done = 0, self.done + 1

    def test(self, parity):  # mbarrier.try_wait.parity / test_wait.parity
        return (self.done & 1) != parity


class Stale(AssertionError):
    pass


def run(need, S, sep_p, seed, plant=None, max_steps=400000, split=True):
    """need[t]: bit w = warpgroup w needs tile t. Returns 'ok' or 'deadlock'.

    split: the producer's K and V loads run as two independent agents (one lane
    each), as in the kernel; False models the earlier single loop that loaded
    K(t) then V(t)."""
    rng = random.Random(seed)
    T = len(need)
    B = {}

    def bar(name, count=1):
        if name not in B:
            B[name] = Bar(count)
        return B[name]

    stage_k = [None] * S  # tile held, or None
    stage_v = [None] * S
    landed_k = [False] * S
    landed_v = [False] * S
    events = []           # TMA landings (any order)
    pipe = []             # issued MMAs, completing in order
    reading_p = [False, False]

    def tma(kind, st, t):
        def land():
            (landed_k if kind == 'k' else landed_v)[st] = True
            bar(f'{kind}_full{st}').arrive()
        events.append(land)

    def wait(cond):
        while not cond():
            yield False
        yield True

    # ---------------------------------------------------------------- producer
    def load(kind, t, par):
        st = t % S
        stage, landed = (stage_k, landed_k) if kind == 'k' else (stage_v, landed_v)
        prev = need[t - S] if t >= S else 0
        for w in range(2):
            if (prev >> w) & 1:
                b = f'{kind}_empty{st}_{w}'
                p = par.get(b, 0)
                yield from wait(lambda b=b, p=p: bar(b).test(p))
                par[b] = p ^ 1
        if any(op['reads'] == (kind, st) for op in pipe):
            raise Stale(f'{kind} stage {st} reloaded while an MMA reads it')
        stage[st] = t
        landed[st] = False
        tma(kind, st, t)

    def producer():
        for w in range(2):
            if any((n >> w) & 1 for n in need):
                events.append(lambda w=w: bar(f'q_full{w}').arrive())
        par = {}
        for t in range(T):
            for kind in (('k',) if split else ('k', 'v')):
                yield from load(kind, t, par)

    def producer_v():  # the V lane of the split producer
        par = {}
        for t in range(T):
            yield from load('v', t, par)

    def issue(w, kind, t, j):
        st = t % S
        stage, landed = (stage_k, landed_k) if kind == 'qk' else (stage_v, landed_v)
        if stage[st] != t or not landed[st]:
            raise Stale(f'{kind} of tile {t} (warpgroup {w}) found {stage[st]} landed={landed[st]}')
        if kind == 'pv':
            reading_p[w] = True
        pipe.append(dict(w=w, kind=kind, t=t, reads=('k' if kind == 'qk' else 'v', st)))

    def complete(op):
        st = op['reads'][1]
        if op['kind'] == 'qk':
            bar(f's_full{op["w"]}').arrive()
            bar(f'k_empty{st}_{op["w"]}').arrive()
        else:
            reading_p[op['w']] = False
            bar(f'o_ready{op["w"]}').arrive()
            bar(f'v_empty{st}_{op["w"]}').arrive()

    # ---------------------------------------------------------------- issuers
    def issuer_poll():  # separate P columns
        def next_tile(t, w):
            while t < T and not ((need[t] >> w) & 1):
                t += 1
            return t
        g = [dict(next=next_tile(0, w), cnt=0, f0=-1, j0=0, f1=-1, j1=0, q=False) for w in range(2)]
        seen = {'k': 0, 'v': 0}

        def walk(kind, upto):
            while seen[kind] <= upto and bar(f'{kind}_full{seen[kind] % S}').test((seen[kind] // S) & 1):
                seen[kind] += 1
            return seen[kind] > upto

        def try_pv(w):
            G = g[w]
            if G['f0'] < 0:
                return False
            u = G['f0']
            if not walk('v', u) or not bar(f'p_full{w}', 1).test(G['j0'] & 1):
                return False
            issue(w, 'pv', u, G['j0'])
            G['f0'], G['j0'], G['f1'] = G['f1'], G['j1'], -1
            return True

        def try_qk(w):
            G = g[w]
            if G['next'] >= T or G['f1'] >= 0:
                return False
            t = G['next']
            if not G['q']:
                if not bar(f'q_full{w}').test(0):
                    return False
                G['q'] = True
            if not (G['cnt'] == 0 or bar(f's_free{w}').test((G['cnt'] - 1) & 1)):
                return False
            if plant == 'no_k_walk':
                if not bar(f'k_full{t % S}').test((t // S) & 1):
                    return False
            elif not walk('k', t):
                return False
            issue(w, 'qk', t, G['cnt'])
            if G['f0'] < 0:
                G['f0'], G['j0'] = t, G['cnt']
            else:
                G['f1'], G['j1'] = t, G['cnt']
            G['cnt'] += 1
            G['next'] = next_tile(t + 1, w)
            return True

        while any(G['next'] < T or G['f0'] >= 0 for G in g):
            moved = False
            for w in range(2):
                q = try_qk(w)
                moved |= try_pv(w) or q
            yield moved

    def issuer_fixed():  # P over S
        pt, pj, c, q = [-1, -1], [0, 0], [0, 0], [False, False]
        v_seen = [0]

        def pv(w):
            u = pt[w]
            while v_seen[0] <= u:  # V tiles observed in tile order, as in the kernel
                x = v_seen[0]
                yield from wait(lambda x=x: bar(f'v_full{x % S}').test((x // S) & 1))
                v_seen[0] += 1
            yield from wait(lambda: bar(f'p_full{w}', 1).test(pj[w] & 1))
            issue(w, 'pv', u, pj[w])
            pt[w] = -1

        def flush_below(limit):
            order = sorted((pt[w], w) for w in range(2) if 0 <= pt[w] < limit)
            for _, w in order:
                yield from pv(w)

        for t in range(T):
            # single-loop producer: K(t) waits behind V(t - 1), which needs every
            # PV of tile t - 1 - S
            if not split and plant != 'no_flush':
                yield from flush_below(t - S)
            yield from wait(lambda t=t: bar(f'k_full{t % S}').test((t // S) & 1))
            for w in range(2):
                if (need[t] >> w) & 1:
                    if not q[w]:
                        yield from wait(lambda w=w: bar(f'q_full{w}').test(0))
                        q[w] = True
                    if pt[w] >= 0:
                        # split producer: V(u) reuses the stage of tile u - S, so the
                        # other warpgroup's PV of a tile <= u - S goes first
                        o = 1 - w
                        if split and plant != 'no_v_order' and 0 <= pt[o] <= pt[w] - S:
                            yield from pv(o)
                        yield from pv(w)
                    issue(w, 'qk', t, c[w])
            for w in range(2):
                if (need[t] >> w) & 1:
                    pt[w], pj[w] = t, c[w]
                    c[w] += 1
        yield from flush_below(T)

    # ---------------------------------------------------------------- softmax
    def softmax(w):
        j = 0
        for t in range(T):
            if not ((need[t] >> w) & 1):
                continue
            yield from wait(lambda j=j: bar(f's_full{w}').test(j & 1))
            if sep_p:
                bar(f's_free{w}').arrive()
            if j > 0:
                yield from wait(lambda j=j: bar(f'o_ready{w}').test((j - 1) & 1))
            if reading_p[w]:
                raise Stale(f'warpgroup {w} overwrites P while its PV is pending')
            bar(f'p_full{w}', 1).arrive()
            j += 1
            yield True

    live = {'producer': producer(), 'issuer': issuer_poll() if sep_p else issuer_fixed(),
            'wg0': softmax(0), 'wg1': softmax(1)}
    if split:
        live['producer_v'] = producer_v()
    idle = {k: 0 for k in live}
    for _ in range(max_steps):
        if not live and not events and not pipe:
            return 'ok'
        choices = list(live) + (['event'] if events else []) + (['pipe'] if pipe else [])
        c = rng.choice(choices)
        if c == 'event':
            events.pop(rng.randrange(len(events)))()
            idle = {k: 0 for k in live}
            continue
        if c == 'pipe':
            complete(pipe.pop(0))
            idle = {k: 0 for k in live}
            continue
        try:
            moved = next(live[c])
        except StopIteration:
            del live[c]
            idle.pop(c, None)
            continue
        if moved:
            idle = {k: 0 for k in live}
        else:
            idle[c] += 1
        if not events and not pipe and live and all(idle[k] >= 3 for k in live):
            return 'deadlock'
    return 'too long'


def tile_needs(keep, p, nQB):
    """need bits of the CTA covering query blocks 4p..4p+3 (block 64)."""
    ents = []
    for J in range(keep.shape[1]):
        gb = 0
        for g in range(4):
            I = 4 * p + g
            if I < nQB and keep[I, J]:
                gb |= 1 << g
        if gb:
            ents.append(gb)
    need = []
    for t in range(0, len(ents), 2):
        g = ents[t] | (ents[t + 1] if t + 1 < len(ents) else 0)
        need.append((1 if g & 3 else 0) | (2 if g & 12 else 0))
    return need


def arrow_needs(N=4352, n_text=256, bs=64, windows=(1, 2, 4)):
    nb = N // bs
    out = []
    for w in windows:
        tm = OM.arrow_token_mask(N, n_text, bs, 1, w)
        keep = tm.reshape(nb, bs, nb, bs).any(axis=(1, 3))
        out += [tile_needs(keep, p, nb) for p in range(nb // 4)]
    return out


def pooled_needs():
    """C3-like schedules: content-driven top-30% at block 128 (a CTA's two
    warpgroups serve different query blocks, so their kept sets differ)."""
    import workloads as W
    from oracle import select as OS
    w = W.content_case(B=1, H=2, n_text=256, grid_hw=(64, 64), d=64, block=128, seed=5)
    shp = w["shape"]
    ntb = -(-shp.n_text // shp.block_k)
    groups = [(ntb, shp.n_kb, (30 * (shp.n_kb - ntb) + 99) // 100)]
    out = []
    for h in range(shp.H):
        cls, _ = OS.pooled_select(w["q"][0, h].double().numpy(), w["k"][0, h].double().numpy(), 128, 128,
                                  shp.n_text, groups, True)
        for I in range(0, shp.n_qb, 2):  # CTA rows: warpgroup 0 = block I, warpgroup 1 = block I + 1
            need = []
            for J in range(shp.n_kb):  # a 128-key tile is one block (two 64-key segments)
                b0 = cls[I, J] > 0
                b1 = I + 1 < shp.n_qb and cls[I + 1, J] > 0
                if b0 or b1:
                    need.append((1 if b0 else 0) | (2 if b1 else 0))
            out.append(need)
    return out


def random_needs(seed, n=40):
    rng = random.Random(seed)
    out = []
    for _ in range(n):
        T = rng.randint(1, 24)
        mode = rng.random()
        if mode < 0.3:  # long gaps for one warpgroup
            need = [3 if rng.random() < 0.2 else rng.choice([1, 2]) for _ in range(T)]
        else:
            need = [rng.choice([1, 2, 3, 3, 3]) for _ in range(T)]
        out.append(need)
    return out


@pytest.mark.parametrize("sep_p,S", [(True, 4), (False, 2), (False, 4), (True, 2)])
def test_protocol_on_arrow_schedules(sep_p, S):
    for need in arrow_needs():
        for seed in range(6):
            assert run(need, S, sep_p, seed) == 'ok', need


@pytest.mark.parametrize("sep_p,S", [(True, 4), (False, 2)])
def test_protocol_on_pooled_selection_schedules(sep_p, S):
    needs = pooled_needs()
    assert any(0 < sum(1 for n in need if n != 3) for need in needs)  # the warpgroups' sets differ
    for need in needs:
        for seed in range(4):
            assert run(need, S, sep_p, seed) == 'ok', need


@pytest.mark.parametrize("sep_p,S", [(True, 4), (False, 2)])
def test_protocol_on_random_schedules(sep_p, S):
    for k, need in enumerate(random_needs(5)):
        for seed in range(8):
            assert run(need, S, sep_p, 100 * k + seed) == 'ok', need


def test_planted_missing_flush_deadlocks_the_single_loop_producer():
    # a producer that loads K(t) only after V(t - 1): warpgroup 0 waits for K of
    # a far tile while its own PV of an old tile, which the producer needs
    # released first, is still unissued
    need = [3, 2, 2, 2, 2, 2, 3]
    results = {run(need, 2, False, seed, plant='no_flush', split=False) for seed in range(30)}
    assert 'deadlock' in results
    assert all(run(need, 2, False, seed, split=False) == 'ok' for seed in range(30))


def test_planted_missing_v_order_deadlocks_the_split_producer():
    # split producer: warpgroup 1's PV of tile 0 is pending while warpgroup 0
    # waits for V(2), which reuses tile 0's stage
    need = [3, 1, 1, 1, 2]
    results = {run(need, 2, False, seed, plant='no_v_order') for seed in range(60)}
    assert 'deadlock' in results
    assert all(run(need, 2, False, seed) == 'ok' for seed in range(60))


@pytest.mark.parametrize("S", [2, 4])
def test_split_producer_on_one_group_runs(S):
    # long runs of tiles only one warpgroup needs, alternating: the case the
    # split producer is for
    for k in range(6):
        rng = random.Random(k)
        need = []
        while len(need) < 40:
            need += [rng.choice([1, 2])] * rng.randint(1, 6) + [3] * rng.randint(0, 2)
        for seed in range(8):
            assert run(need, S, False, 10 * k + seed) == 'ok', need


def test_planted_unordered_k_test_reads_stale_data():
    # warpgroup 0 skips tiles 1..4; tested directly, K(5)'s one-bit parity
    # can pass while the stage still holds tile 1
    need = [3, 2, 2, 2, 2, 1, 3]
    caught = False
    for seed in range(200):
        try:
            run(need, 4, True, seed, plant='no_k_walk')
        except Stale:
            caught = True
            break
    assert caught
    for seed in range(50):
        assert run(need, 4, True, seed) == 'ok'
