"""Index arithmetic of the staged score kernel, checked on the CPU.

The staged kernel streams a warp's batches of KB consecutive key records
through a private ring of STAGES shared-memory slots with bulk copies.  Its
span partition, batch grid, slot/parity sequence, copy ranges and shared-memory
carve-up are restated here from its source constants and checked for every
instantiation the library launches: the copies stay inside K and pos, start on
16-byte boundaries and move whole 16-byte units; every key is staged and stored
exactly once; a slot is refilled only after its batch was consumed; the ring
and the barriers stay inside the dynamic shared memory, which fits an SM at the
kernel's occupancy.
"""
import pytest

THREADS = 256
WARPS = THREADS // 32
SMEM_PER_SM = 228 * 1024
RESERVED_PER_CTA = 1024


def shape(lpk, pre):
    ng = 32 // lpk
    u = 4 if (lpk == 4 or pre) else 8
    return ng, u, ng * u, 8 * lpk


def staging(pre, elem, lpk):
    ng, u, kb, f = shape(lpk, pre)
    rb = 2 * f * elem
    key_bytes = kb * rb
    slot = key_bytes + (kb * 4 if pre else 0)
    budget = 13312 if pre else 8192
    stages = max(2, min(4, budget // slot))
    header = (WARPS * stages * 8 + 127) // 128 * 128
    smem = header + WARPS * stages * slot
    return dict(ng=ng, u=u, kb=kb, rb=rb, key_bytes=key_bytes, slot=slot, stages=stages, header=header, smem=smem,
                ctas=3 if (elem == 1 and not pre) else 2)


# The instantiations the dispatch launches: pre-RoPE caches of both element
# types, and post-RoPE fp8 caches, at head dims 64 / 128 / 256 (lanes per key 4 / 8 / 16).
CONFIGS = [(pre, elem, lpk) for lpk in (4, 8, 16) for (pre, elem) in ((True, 2), (True, 1), (False, 1))]


@pytest.mark.parametrize("pre,elem,lpk", CONFIGS)
def test_shared_memory_fits_the_occupancy(pre, elem, lpk):
    st = staging(pre, elem, lpk)
    assert st["slot"] % 16 == 0 and st["key_bytes"] % 16 == 0 and st["header"] % 128 == 0
    assert st["kb"] % 4 == 0
    assert st["ctas"] * (st["smem"] + RESERVED_PER_CTA) <= SMEM_PER_SM, st
    assert st["key_bytes"] < (1 << 20)  # an mbarrier's transaction count


def schedule(total, grid, st, pos_aligned=True):
    """Yields (warp, batch i, b0, n, slot, parity, copies) in the kernel's order;
    copies = [(kind, byte offset in the source array, bytes, ring offset)]."""
    kb, rb, stages = st["kb"], st["rb"], st["stages"]
    nwarps = grid * WARPS
    per = (total + nwarps - 1) // nwarps
    per = (per + kb - 1) // kb * kb
    for wid in range(nwarps):
        beg = wid * per
        end = min(total, beg + per)
        if beg >= end:
            continue
        nb = (end - beg + kb - 1) // kb
        warp = wid % WARPS
        issued = {}

        def issue(i):
            b0 = beg + i * kb
            n = min(kb, end - b0)
            s = i % stages
            ring = st["header"] + (warp * stages + s) * st["slot"]
            copies = [("K", b0 * rb, n * rb, ring)]
            pb = (n & ~3) * 4 if (pos_aligned and st["slot"] > st["key_bytes"]) else 0
            if pb:
                copies.append(("pos", b0 * 4, pb, ring + st["key_bytes"]))
            assert s not in issued, "slot refilled before its batch was consumed"
            issued[s] = i
            return copies

        pending = {}
        for i in range(min(nb, stages)):
            pending[i] = issue(i)
        for i in range(nb):
            s = i % stages
            assert issued.get(s) == i
            del issued[s]
            b0 = beg + i * kb
            n = min(kb, end - b0)
            yield wid, i, b0, n, s, (i // stages) & 1, pending.pop(i), beg, end
            if i + stages < nb:
                pending[i + stages] = issue(i + stages)
        assert not pending and not issued


def grid_for(total, kb, sms=148, occ=2):
    want = (total + kb * WARPS - 1) // (kb * WARPS)
    return max(1, min(sms * occ, want))


@pytest.mark.parametrize("pre,elem,lpk", CONFIGS)
@pytest.mark.parametrize("total", [1, 3, 7, 8, 15, 16, 17, 31, 33, 100, 4095, 4096, 4097, 65536 + 5, 300001])
def test_copies_cover_every_key_once_in_bounds(pre, elem, lpk, total):
    st = staging(pre, elem, lpk)
    grid = grid_for(total, st["kb"], occ=st["ctas"])
    covered = bytearray(total)
    stored = bytearray(total)
    for wid, i, b0, n, s, parity, copies, beg, end in schedule(total, grid, st):
        assert beg <= b0 < end and 0 < n <= st["kb"] and b0 + n <= end
        assert (b0 - beg) % st["kb"] == 0 and b0 % st["kb"] == 0  # the global batch grid
        for kind, off, nbytes, ring in copies:
            size = total * (st["rb"] if kind == "K" else 4)
            assert off % 16 == 0 and nbytes % 16 == 0 and ring % 16 == 0, (kind, off, nbytes, ring)
            assert 0 <= off and off + nbytes <= size
            assert st["header"] <= ring and ring + nbytes <= st["smem"]
        for k in range(b0, b0 + n):
            covered[k] += 1
        # lane l < KB stores key b0 + l when it is inside the batch
        for lane in range(32):
            if lane < st["kb"] and b0 + lane < b0 + n:
                stored[b0 + lane] += 1
        # barriers of this warp: indices warp*STAGES + s inside the header
        assert ((wid % WARPS) * st["stages"] + s + 1) * 8 <= st["header"]
    assert all(c == 1 for c in covered) and all(c == 1 for c in stored)


@pytest.mark.parametrize("pre,elem,lpk", CONFIGS)
def test_lane_reads_stay_in_their_slot(pre, elem, lpk):
    """Lane (q, gl) reads key NG*u + q of the slot at byte offsets below the record length."""
    st = staging(pre, elem, lpk)
    ng, u, kb, rb = st["ng"], st["u"], st["kb"], st["rb"]
    f = rb // (2 * elem)
    for lane in range(32):
        q, gl = lane // lpk, lane % lpk
        for uu in range(u):
            idx = ng * uu + q
            assert idx < kb
            base = idx * rb
            # rotate-half: real part at e*8*gl (16 B for bf16, 8 for fp8), imaginary F elements later;
            # interleaved: 32*gl (bf16, two 16-B reads) or 16*gl (fp8)
            for off, width in ([(16 * gl, 16), (2 * f + 16 * gl, 16)] if elem == 2 else
                               [(8 * gl, 8), (f + 8 * gl, 8)]) + \
                              ([(32 * gl, 16), (32 * gl + 16, 16)] if elem == 2 else [(16 * gl, 16)]):
                assert off % width == 0 and off + width <= rb
                assert base + off + width <= st["key_bytes"]
        if pre:
            assert kb * 4 + st["key_bytes"] <= st["slot"]


def test_large_totals_last_batches():
    """Full-size caches (up to the 128K workload's 268 M keys): the last warp's span and
    its final batch stay in bounds, analytically."""
    for pre, elem, lpk in CONFIGS:
        st = staging(pre, elem, lpk)
        for total in (9437184, 268435456, 268435456 + 13, 2 ** 31 + 7):
            grid = grid_for(total, st["kb"], occ=st["ctas"])
            nwarps = grid * WARPS
            per = ((total + nwarps - 1) // nwarps + st["kb"] - 1) // st["kb"] * st["kb"]
            last = (total - 1) // per
            beg, end = last * per, total
            nb = (end - beg + st["kb"] - 1) // st["kb"]
            b0 = beg + (nb - 1) * st["kb"]
            n = min(st["kb"], end - b0)
            assert 0 < n <= st["kb"] and b0 + n == total
            assert (b0 + n) * st["rb"] <= total * st["rb"] and b0 * st["rb"] % 16 == 0


# ---------------------------------------------------------------- key centres

KC_CHUNKS = 16


def kc_staging(post, elem, lpk):
    ng, u, f = 32 // lpk, 4, 8 * lpk
    kb, rb = ng * u, 2 * f * elem
    key_bytes = kb * rb
    pos_cap = kb + 4 if post else 0
    slot = key_bytes + pos_cap * 4
    acc = 24 * WARPS * lpk * 8
    header = 256
    per_cta = (228 * 1024 - 2 * 1024) // 2
    fit = (per_cta - acc - header) // (WARPS * slot)
    stages = max(2, min(4, fit))
    smem = header + acc + WARPS * stages * slot
    return dict(ng=ng, u=u, kb=kb, rb=rb, key_bytes=key_bytes, pos_cap=pos_cap, slot=slot, acc=acc,
                header=header, stages=stages, smem=smem)


KC_CONFIGS = [(post, elem, lpk) for lpk in (4, 8, 16) for post in (True, False) for elem in (2, 1)]


@pytest.mark.parametrize("post,elem,lpk", KC_CONFIGS)
def test_key_centre_shared_memory(post, elem, lpk):
    st = kc_staging(post, elem, lpk)
    assert st["slot"] % 16 == 0 and st["acc"] % 16 == 0 and st["kb"] % 4 == 0
    assert WARPS * st["stages"] * 8 <= st["header"]
    assert 2 * (st["smem"] + RESERVED_PER_CTA) <= SMEM_PER_SM, st


def kc_batches(lo, hi, chunk, warp, st):
    n = hi - lo
    beg = lo + n * chunk // KC_CHUNKS
    end = lo + n * (chunk + 1) // KC_CHUNKS
    first = beg + warp * st["kb"]
    nbw = (end - first + WARPS * st["kb"] - 1) // (WARPS * st["kb"]) if first < end else 0
    for t in range(nbw):
        b0 = first + t * WARPS * st["kb"]
        yield t, b0, min(st["kb"], end - b0), beg, end


@pytest.mark.parametrize("post,elem,lpk", KC_CONFIGS)
@pytest.mark.parametrize("rows", [[0], [1], [5], [17, 0, 3], [4096, 4097, 33], [1000, 2049, 7, 65536 + 3]])
def test_key_centre_copies_in_bounds_and_cover_rows(post, elem, lpk, rows):
    st = kc_staging(post, elem, lpk)
    offs = [0]
    for n in rows:
        offs.append(offs[-1] + n)
    total = offs[-1]
    seen = bytearray(total)
    for r in range(len(rows)):
        lo, hi = offs[r], offs[r + 1]
        for chunk in range(KC_CHUNKS):
            for warp in range(WARPS):
                slots = {}
                for t, b0, n, beg, end in kc_batches(lo, hi, chunk, warp, st):
                    assert beg <= b0 and b0 + n <= end and n > 0
                    # records
                    assert (b0 * st["rb"]) % 16 == 0 and (n * st["rb"]) % 16 == 0
                    assert b0 * st["rb"] + n * st["rb"] <= total * st["rb"]
                    ring = st["header"] + st["acc"] + (warp * st["stages"] + t % st["stages"]) * st["slot"]
                    assert ring % 16 == 0 and ring + st["slot"] <= st["smem"]
                    # the positions window [a0, a1) inside the array, 16-byte aligned
                    if post:
                        a0 = b0 & ~3
                        a1 = min((b0 + n + 3) & ~3, total & ~3)
                        if a1 > a0:
                            assert (a0 * 4) % 16 == 0 and ((a1 - a0) * 4) % 16 == 0
                            assert 0 <= a0 and a1 <= total and a1 - a0 <= st["pos_cap"]
                        # every key k of the batch reads spos[k - a0] when k < a1, else global memory
                        for k in range(b0, b0 + n):
                            if k < a1:
                                assert 0 <= k - a0 < a1 - a0
                    for k in range(b0, b0 + n):
                        seen[k] += 1
                    slots[t % st["stages"]] = t
    assert all(c == 1 for c in seen)
