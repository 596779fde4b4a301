"""The block-sparse forward's lockstep schedule.  The steps come from the
library's own walk (attn_schedule_sparse_steps runs on the host the
sparse_next_step code that the kernel's loader, MMA issuer and softmax warps
call) and must equal a Python statement of the walk; a model of the MMA
issuer's order then checks, over random mask pairs, that every K/V stream position is loaded
once, in order, each Q tile sees exactly its own tiles in increasing order,
every stage is released exactly once and after its last reader, the Q tile
that zeroes a V tile's padded rows is the first to read it, and no load waits
for a release that comes after the load's first use in the MMA order (the
ring cannot deadlock).  The kernel's own results are checked against the
oracle in test_blocksparse_gpu.py."""
import random

import pytest

from io_aware_exact_29_b200 import attn


def _run(m0, m1, nt0, nt1, j00=0, j01=0, KST=2, VST=3):
    use = lambda a, j: (j >= (j00 if a == 0 else j01) and j < (nt0 if a == 0 else nt1)) and (m0 if a == 0 else m1)[j]
    n0 = sum(use(0, j) for j in range(j00, nt0)); n1 = sum(use(1, j) for j in range(j01, nt1))
    nsteps = max(n0, n1)
    def gen():
        c = [j00, j01]; pos = 0
        for si in range(nsteps):
            st = dict(has0=si < n0, has1=si < n1, x0=-1, x1=-1, pos0=-1, pos1=-1)
            for a in (0, 1):
                if st['has%d' % a]:
                    while c[a] < (nt0 if a == 0 else nt1) - 1 and not use(a, c[a]): c[a] += 1
                    st['x%d' % a] = c[a]; c[a] += 1
            st['shared'] = st['has0'] and st['has1'] and st['x0'] == st['x1']
            if st['has0']: st['pos0'] = pos; pos += 1
            if st['has1']:
                if st['shared']: st['pos1'] = st['pos0']
                else: st['pos1'] = pos; pos += 1
            yield st
    steps = list(gen())
    lib_steps = attn.schedule_sparse_steps([bool(x) for x in m0], [bool(x) for x in m1],
                                           nt0, nt1, j00, j01)
    assert lib_steps == steps, (lib_steps, steps)
    # loader
    loads = []
    for st in steps:
        if st['has0']: loads.append((st['pos0'], st['x0']))
        if st['has1'] and not st['shared']: loads.append((st['pos1'], st['x1']))
    assert [p for p, _ in loads] == list(range(len(loads)))
    tile_of = dict(loads)
    # MMA events in issue order
    ev = []; prev = None
    for i in range(nsteps + 1):
        st = steps[i] if i < nsteps else None
        if st and st['has0']:
            ev.append(('S', 0, st['pos0']))
            if not st['shared']: ev.append(('Krel', st['pos0']))
        if prev and prev['has1']:
            ev.append(('PV', 1, prev['pos1'], i - 1)); ev.append(('Vrel', prev['pos1']))
        if st:
            if st['has1']:
                ev.append(('S', 1, st['pos1'])); ev.append(('Krel', st['pos1']))
            if st['has0']:
                ev.append(('PV', 0, st['pos0'], i))
                if not st['shared']: ev.append(('Vrel', st['pos0']))
        prev = st
    # each position released once, after all uses
    for kind, use_kind in (('Krel', 'S'), ('Vrel', 'PV')):
        for p in range(len(loads)):
            rel = [k for k, e in enumerate(ev) if e[0] == kind and e[1] == p]
            assert len(rel) == 1, (kind, p, rel)
            uses = [k for k, e in enumerate(ev) if e[0] == use_kind and e[2] == p]
            assert uses and max(uses) < rel[0], (kind, p)
    # per Q tile: tiles in increasing order, exactly its mask's tiles
    for a, n in ((0, n0), (1, n1)):
        s_list = [tile_of[e[2]] for e in ev if e[0] == 'S' and e[1] == a]
        pv_list = [tile_of[e[2]] for e in ev if e[0] == 'PV' and e[1] == a]
        want = [j for j in range((j00, j01)[a], (nt0, nt1)[a]) if use(a, j)]
        assert s_list == want and pv_list == want, (a, s_list, want)
        # PV ia index = step index, last at n-1
        ias = [e[3] for e in ev if e[0] == 'PV' and e[1] == a]
        assert ias == list(range(n))
    # first reader of each V position is the one whose softmax zeroes it
    for st in steps:
        for a in (0, 1):
            if not st['has%d' % a]: continue
            first_user = a == 0 or not st['shared']
            p = st['pos%d' % a]
            first_pv = next(e for e in ev if e[0] == 'PV' and e[2] == p)
            assert (first_pv[1] == a) == first_user
    # ring: a load of position p needs the release of p - KST (K) / p - VST (V) earlier in the
    # MMA order than the first use of position p (no use-before-release cycle)
    for p in range(len(loads)):
        first_use = min(k for k, e in enumerate(ev) if e[0] in ('S',) and e[2] == p)
        if p >= KST:
            relk = next(k for k, e in enumerate(ev) if e[0] == 'Krel' and e[1] == p - KST)
            assert relk < first_use, ('K ring', p)
        first_pv = min(k for k, e in enumerate(ev) if e[0] == 'PV' and e[2] == p)
        if p >= VST:
            relv = next(k for k, e in enumerate(ev) if e[0] == 'Vrel' and e[1] == p - VST)
            assert relv < first_pv, ('V ring', p)
    # the loader issues K(p), V(p), K(p+1), ...: the S of position p+1 also waits
    # for V(p)'s load, i.e. for the release of V(p - VST)
    for p in range(len(loads) - 1):
        if p >= VST:
            relv = next(k for k, e in enumerate(ev) if e[0] == 'Vrel' and e[1] == p - VST)
            first_s_next = min(k for k, e in enumerate(ev) if e[0] == 'S' and e[2] == p + 1)
            assert relv < first_s_next, ('V before next K', p)
    return len(loads), nsteps


@pytest.mark.parametrize("kst,vst", [(2, 3), (3, 4)])
def test_lockstep_schedule_bookkeeping(kst, vst):
    rng = random.Random(kst * 10 + vst)
    for _ in range(3000):
        nk = rng.randint(1, 20)
        d0, d1 = rng.random(), rng.random()
        m0 = [rng.random() < d0 for _ in range(nk)]
        m1 = [rng.random() < d1 for _ in range(nk)]
        nt0, nt1 = rng.randint(0, nk), rng.randint(0, nk)
        j00 = rng.randint(0, max(0, nt0 - 1)) if rng.random() < 0.3 else 0
        j01 = max(j00, rng.randint(0, max(0, nt1 - 1))) if rng.random() < 0.3 else 0
        _run(m0, m1, nt0, nt1, j00, j01, KST=kst, VST=vst)


def test_identical_masks_share_every_tile():
    m = [True, False, True, True, False, True]
    loads, steps = _run(m, m, 6, 6)
    assert loads == steps == 4
