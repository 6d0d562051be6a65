"""Event simulations of the mbarrier protocols of two kernel families, run on
the CPU: the TMA ring of the FP4 quantizer and the column statistics (one
producer, 8 consumer warps taking tiles in turn), and the FP4 GEMM's producer /
scale-copy warp / MMA warp (per-stage scale columns in the 128x256 kernel, two
alternating TMEM slots in the 256x192 kernel, low-rank steps between tiles).

An mbarrier is modelled by its phase count; a parity wait passes when the
current (incomplete) phase's parity differs from the parity asked for, as
`mbarrier.try_wait.parity` does.  Loads land after random delays, so out of
order.  The protocols the kernels use must never read a stage or a TMEM slot
that holds another step's data and must never stall; the earlier forms of both
(a consumer that only waits on its own tiles' full barrier; a scale warp that
waits on the operand barrier and skips the low-rank steps) must be caught."""
import random


class Bar:
    def __init__(self):
        self.phase = 0

    def complete(self):
        self.phase += 1

    def done(self, parity):
        return (self.phase & 1) != parity


def ring(S, C, ntiles, wait_previous_round, seed, skew=(1, 2, 3, 20, 40)):
    """Producer + C consumer warps over an S-stage ring; returns (wrong reads, stalled)."""
    rng = random.Random(seed)
    full = [Bar() for _ in range(S)]
    empty = [Bar() for _ in range(S)]
    content = [None] * S
    pending = []
    nextq = 0
    cons = [{"q": w, "until": 0, "stage": None} for w in range(C)]
    errors = done = t = 0
    while done < ntiles and t < 100000:
        if nextq < ntiles:
            s, ph = nextq % S, (nextq // S) & 1
            if empty[s].done(ph ^ 1):
                content[s] = None
                pending.append((t + rng.choice(skew), s, nextq))
                nextq += 1
        for item in [p for p in pending if p[0] <= t]:
            pending.remove(item)
            content[item[1]] = item[2]
            full[item[1]].complete()
        for c in cons:
            q = c["q"]
            if q >= ntiles or c["stage"] is not None:
                continue
            s, sph = q % S, (q // S) & 1
            if wait_previous_round and not empty[s].done(sph ^ 1):
                continue
            if not full[s].done(sph):
                continue
            errors += content[s] != q
            c["stage"], c["until"] = s, t + rng.choice([1, 5, 10])
        for c in cons:
            if c["stage"] is not None and c["until"] <= t:
                empty[c["stage"]].complete()
                c["stage"] = None
                c["q"] += C
                done += 1
        t += 1
    return errors, done < ntiles


def gemm(S, num_kt, nlr, tiles, two_slots, own_scale_barrier, seed):
    """Producer, scale warp and MMA warp of the FP4 GEMM; returns (wrong reads, stalled)."""
    rng = random.Random(seed)
    steps = []
    for tile in range(tiles):
        steps += ["fp4"] * num_kt + ["lr"] * nlr
    n = len(steps)
    fp4 = {}
    for i, kind in enumerate(steps):
        if kind == "fp4":
            fp4[i] = len(fp4)
    full = [Bar() for _ in range(S)]
    empty = [Bar() for _ in range(S)]
    sf_full = [Bar() for _ in range(S)]
    nsl = 2 if two_slots else S
    sf_ready = [Bar() for _ in range(nsl)]
    sf_free = [Bar() for _ in range(2)]
    ops, sfs, tmem = [None] * S, [None] * S, [None] * nsl
    events = []
    prod_i, sf = 0, {"i": 0, "ph": 0, "busy": False}
    mma = {"i": 0, "ph": 0, "busy": False}
    errors = t = 0
    while mma["i"] < n and t < 200000:
        for ev in [e for e in events if e[0] <= t]:
            events.remove(ev)
            kind, pl = ev[1], ev[2]
            if kind == "ops":
                ops[pl[0]] = pl[1]
                full[pl[0]].complete()
            elif kind == "sf":
                sfs[pl[0]] = pl[1]
                sf_full[pl[0]].complete()
            elif kind == "copied":
                tmem[pl[0]] = pl[1]
                sf_ready[pl[0]].complete()
                sf["busy"] = False
            else:
                s, slot, g = pl
                if g is not None:
                    errors += tmem[slot] != g       # the slot changed under the MMA
                    if two_slots:
                        sf_free[slot].complete()
                empty[s].complete()
                mma["busy"] = False
        if prod_i < n:
            s, ph = prod_i % S, (prod_i // S) & 1
            if empty[s].done(ph ^ 1):
                ops[s] = None
                d = rng.choice([1, 2, 8, 30])
                if steps[prod_i] == "fp4":
                    sfs[s] = None
                    ds = rng.choice([1, 2, 8, 30]) if own_scale_barrier else d - 0.5
                    events.append((t + ds, "sf", (s, fp4[prod_i])))
                events.append((t + d, "ops", (s, prod_i)))
                prod_i += 1
        i = sf["i"]
        if i < n and not sf["busy"]:
            s = i % S
            if steps[i] == "lr":
                sf["i"] += 1
            else:
                g = fp4[i]
                slot = g & 1 if two_slots else s
                ok = not (two_slots and g >= 2 and not sf_free[slot].done(((g >> 1) - 1) & 1))
                if own_scale_barrier:
                    ok = ok and sf_full[s].done((sf["ph"] >> s) & 1)
                else:
                    ok = ok and full[s].done((i // S) & 1)
                if ok:
                    errors += sfs[s] != g
                    sf["ph"] ^= 1 << s
                    sf["busy"] = True
                    events.append((t + rng.choice([1, 3, 10]), "copied", (slot, sfs[s])))
                    sf["i"] += 1
        i = mma["i"]
        if i < n and not mma["busy"]:
            s, ph = i % S, (i // S) & 1
            g = fp4.get(i)
            slot = None if g is None else (g & 1 if two_slots else s)
            ok = full[s].done(ph)
            if ok and g is not None:
                par = (g >> 1) & 1 if two_slots else (mma["ph"] >> s) & 1
                ok = sf_ready[slot].done(par)
            if ok:
                errors += ops[s] != i
                if g is not None:
                    errors += tmem[slot] != g
                    if not two_slots:
                        mma["ph"] ^= 1 << s
                mma["busy"] = True
                events.append((t + rng.choice([2, 5]), "mma", (s, slot, g)))
                mma["i"] += 1
        t += 1
    return errors, mma["i"] < n


def _total(fn, seeds, *args):
    errors = stalls = 0
    for seed in range(seeds):
        e, s = fn(*args, seed)
        errors += e
        stalls += s
    return errors, stalls


def test_ring_protocol_of_the_tma_consumers():
    # the stage counts the kernels use: 12 (rows), 16 and 8 (columns)
    for S in (8, 12, 16):
        assert _total(ring, 40, S, 8, 240, True) == (0, 0), S
    # the earlier consumer wait is caught at 12 stages, where a stage's
    # rounds alternate between two warps
    assert _total(ring, 40, 12, 8, 240, False)[0] > 0


def test_ring_protocol_with_loads_in_order_needs_no_extra_wait():
    # with loads landing in issue order both forms are correct
    for S in (8, 12, 16):
        for seed in range(20):
            assert ring(S, 8, 240, False, seed, skew=(5,)) == (0, False)


def test_gemm_scale_warp_protocol():
    for two_slots, S in ((False, 4), (True, 3)):
        for nlr in (0, 2, 4, 5, 8):
            assert _total(gemm, 25, S, 6, nlr, 4, two_slots, True) == (0, 0), (two_slots, nlr)
    # the earlier scale warp (operand barrier, low-rank steps skipped) is caught
    for two_slots, S in ((False, 4), (True, 3)):
        assert _total(gemm, 25, S, 6, 4, 4, two_slots, False)[0] > 0
