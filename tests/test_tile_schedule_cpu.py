"""Host-side checks of the job lists of the TILES path's single launch (no GPU
needed): every K block of every projection is covered exactly once, the end
of each neuron tile's gate sits with the start of its up range (the MAIN
job), helper and z pieces are numbered as the kernel reads them, and the
waits between the CTAs' lists always resolve (a step-by-step simulation in
which each CTA finishes its jobs in order and a job waits for what the kernel
waits for)."""
from __future__ import annotations

import ctypes

import pytest

from activation_sparse_gated_relu_b200 import binding as B
from activation_sparse_gated_relu_b200.build import build

Z, MAIN, HELP, DOWN, GHELP = 0, 1, 2, 3, 4


@pytest.fixture(scope="module")
def lib():
    build()
    return B.load_library()


def schedule(lib, d, F, R, n):
    nj = ctypes.c_int(0)
    st = lib.sffn_debug_tile_schedule(d, F, R, n, None, 0, None, ctypes.byref(nj))
    assert st == B.SFFN_ERR_INVALID_ARG and nj.value > 0
    jobs = (ctypes.c_int * (4 * nj.value))()
    off = (ctypes.c_int * (n + 1))()
    assert lib.sffn_debug_tile_schedule(d, F, R, n, jobs, nj.value, off, ctypes.byref(nj)) == B.SFFN_OK
    recs = []
    for i in range(nj.value):
        x, y, z, w = jobs[4 * i:4 * i + 4]
        recs.append(dict(type=x & 15, fin=(x >> 4) & 1, count=(x >> 8) & 0xFF, gcount=(x >> 16) & 0xFF, tile=y,
                         k0=z & 0xFFFF, k1=(z >> 16) & 0xFFFF, id=w))
    lists = [recs[off[c]:off[c + 1]] for c in range(n)]
    assert off[0] == 0 and off[n] == nj.value
    return lists


def cover(ranges, total):
    """The ranges tile [0, total) exactly once."""
    ranges = sorted(ranges)
    pos = 0
    for a, b in ranges:
        assert a == pos and b > a, (ranges, total)
        pos = b
    assert pos == total


SHAPES = [
    # d, F, rank, CTAs
    (4096, 14336, 512, 148), (4096, 14336, 0, 148), (4096, 14336, 512, 149), (4096, 14336, 0, 149),
    (2048, 8192, 256, 148), (4096, 28672, 1024, 148), (256, 1024, 64, 148), (256, 1024, 0, 148),
    (264, 384, 192, 7), (4096, 14336, 512, 1), (1024, 4096, 0, 32), (512, 2048, 128, 3),
]


@pytest.mark.parametrize("d,F,R,n", SHAPES)
def test_lists_cover_every_block_once(lib, d, F, R, n):
    check_cover(schedule(lib, d, F, R, n), d, F, R, n)


def check_cover(lists, d, F, R, n):
    # the kernel's unit is a pair of 128-row tiles
    kd, P, Rt, Md, Kf = -(-d // 64), -(-(F // 128) // 2), -(-R // 256), -(-d // 256), F // 64
    jobs = [j for L in lists for j in L]
    # z: the pieces of each rank pair, slots consecutive in K order, each
    # knowing its index; the last min(4, pieces) finish the pair's parts
    for r in range(Rt):
        zs = sorted((j for j in jobs if j["type"] == Z and j["tile"] == r), key=lambda j: j["k0"])
        cover([(j["k0"], j["k1"]) for j in zs], kd)
        assert all(j["count"] == len(zs) for j in zs)
        assert [j["id"] for j in zs] == list(range(zs[0]["id"], zs[0]["id"] + len(zs)))
        assert [j["gcount"] for j in zs] == list(range(len(zs)))
        nfin = min(4, len(zs))
        assert [j["fin"] for j in zs] == [0] * (len(zs) - nfin) + [1] * nfin
    assert not any(j["type"] == Z for j in jobs) if R == 0 else True
    # each tile: one MAIN holding the end of the gate and the start of the up
    # range; gate helpers before it, up helpers after it, slots consecutive
    kg = R // 64 if R else kd
    for p in range(P):
        mains = [j for j in jobs if j["type"] == MAIN and j["tile"] == p]
        assert len(mains) == 1
        m = mains[0]
        assert 0 <= m["k0"] < kg and m["k1"] >= 1
        gs = sorted((j for j in jobs if j["type"] == GHELP and j["tile"] == p), key=lambda j: j["k0"])
        cover([(j["k0"], j["k1"]) for j in gs] + [(m["k0"], kg)], kg)
        hs = sorted((j for j in jobs if j["type"] == HELP and j["tile"] == p), key=lambda j: j["k0"])
        cover([(0, m["k1"])] + [(j["k0"], j["k1"]) for j in hs], kd)
        assert m["gcount"] == len(gs) and m["count"] == len(hs)
        ids = [j["id"] for j in gs + hs]
        assert ids == list(range(m["id"], m["id"] + len(ids)))
    # down: every output tile's K range
    for t in range(Md):
        cover([(j["k0"], j["k1"]) for j in jobs if j["type"] == DOWN and j["tile"] == t], Kf)
    # a CTA's list: z pieces, then phase 1, then the down ranges
    rank = {Z: 0, MAIN: 1, HELP: 1, GHELP: 1, DOWN: 2}
    for L in lists:
        ph = [rank[j["type"]] for j in L]
        assert ph == sorted(ph)
    # the z pieces are short and spread over the CTAs
    if R:
        zl = [sum(j["k1"] - j["k0"] for j in L if j["type"] == Z) for L in lists]
        assert max(zl) <= max(8, -(-Rt * kd // n) + 8) and max(j["count"] for L in lists for j in L if j["type"] == Z) <= 8


@pytest.mark.parametrize("d,F,R,n", SHAPES)
def test_waits_resolve(lib, d, F, R, n):
    check_waits(schedule(lib, d, F, R, n), R, n)


def check_waits(lists, R, n):
    """Each CTA finishes its jobs in order; a job finishes once what the kernel
    makes it wait for has finished: a z finisher every piece of its rank pair
    (the z pieces, first in every list, publish their partial sums before
    any of them waits), a gate piece (MAIN, GHELP) every part of z (low
    rank), a MAIN its helpers, a DOWN the MAINs of its K range.  Every CTA's
    zeroing of out comes first in its list."""
    Rt = -(-R // 256)
    done_z, done_zt, done_help, done_main = set(), set(), set(), set()
    fin_done = {}
    for L in lists:
        for j in L:
            if j["type"] == Z:
                done_z.add(j["id"])
    pos = [0] * n
    progress = True
    while progress:
        progress = False
        for c in range(n):
            while pos[c] < len(lists[c]):
                j = lists[c][pos[c]]
                if j["type"] == Z:
                    first = j["id"] - j["gcount"]
                    if j["fin"]:
                        if not all(q in done_z for q in range(first, first + j["count"])):
                            break
                        fin_done.setdefault(j["tile"], set()).add(j["id"])
                        if len(fin_done[j["tile"]]) == min(4, j["count"]):
                            done_zt.add(j["tile"])
                elif j["type"] == MAIN:
                    if R and len(done_zt) < Rt:
                        break
                    if not all(q in done_help for q in range(j["id"], j["id"] + j["gcount"] + j["count"])):
                        break
                    done_main.add(j["tile"])
                elif j["type"] == GHELP:
                    if R and len(done_zt) < Rt:
                        break
                    done_help.add(j["id"])
                elif j["type"] == HELP:
                    done_help.add(j["id"])
                else:
                    need = set(range(j["k0"] // 4, (j["k1"] + 3) // 4))  # 4 blocks of 64 per pair
                    if not need <= done_main:
                        break
                pos[c] += 1
                progress = True
    assert all(pos[c] == len(lists[c]) for c in range(n)), "a wait never resolves"


def test_balance_at_the_lopa_shape(lib):
    """At d 4096, d_ff 14336 on 148 CTAs the heaviest list holds at most 8 %
    more K blocks than the mean (the launch is as slow as it), with the
    low-rank gate (rank 512) and with the dense one."""
    for R in (512, 0):
        lists = schedule(lib, 4096, 14336, R, 148)
        kg = R // 64 if R else 64
        loads = [sum((kg - j["k0"] + j["k1"]) if j["type"] == MAIN else (j["k1"] - j["k0"]) for j in L)
                 for L in lists]
        mean = sum(loads) / len(loads)
        assert max(loads) <= 1.08 * mean, (R, max(loads), mean)


def test_rejects_bad_sizes(lib):
    nj = ctypes.c_int(0)
    for args in [(0, 1024, 0, 4), (4096, 1000, 0, 4), (4096, 1024, 65, 4), (4096, 1024, 0, 0), (4100, 1024, 0, 4)]:
        assert lib.sffn_debug_tile_schedule(*args, None, 0, None, ctypes.byref(nj)) == B.SFFN_ERR_INVALID_ARG


def test_random_shapes(lib):
    """Seeded sizes across the accepted range (d a multiple of 8 up to 4096,
    d_ff a multiple of 128, rank 0 or a multiple of 64, 1 to 160 CTAs): the
    builder accepts each, every block is covered once and the waits resolve."""
    import random
    rng = random.Random(20241203)
    for _ in range(150):
        d = 8 * rng.randint(1, 512)
        F = 128 * rng.randint(1, 224)
        R = rng.choice([0, 0, 64 * rng.randint(1, 16)])
        n = rng.choice([1, 2, 3, 7, 32, 64, 100, 132, 148, 149, 160])
        lists = schedule(lib, d, F, R, n)
        check_cover(lists, d, F, R, n)
        check_waits(lists, R, n)
