"""Exhaustive check of the decode kernel's synchronization protocol (no GPU).

A model of one CTA of ``csrc/decode.cuh``, explored over every interleaving
of its warps' steps for small shapes.  The weight stream itself needs no
model: every lane loads its own operands into its own registers.  What the
warps share is the row-block hand-off through shared memory:

* a CTA's work has F row-block parts (flushes).  At the end of part f every
  warp writes its accumulators into slot set f mod 2;
* from part 2 on, a warp first waits on FREE[f mod 2] (bar.sync) unless it
  finished part f - 2 itself: that finisher arrived on FREE[f mod 2] once it
  had read the set, and it does not wait there again;
* warp f mod NW finishes part f: after writing its own slot it waits on
  FULL[f mod 2] (bar.sync), reads every slot of the set and, if part f + 2
  exists, arrives on FREE[f mod 2]; the other warps arrive on FULL[f mod 2]
  after writing and carry on.

Named barriers are modelled with hardware generations: an arrival counts
toward the barrier's current generation, whichever part the arriving warp
means, and a generation completes once all NW warps have arrived.  The model
asserts at every step:
- no slot is overwritten before the finisher of its previous part read it;
- the finisher reads every slot holding its own part;
- every arrival lands in the generation of the part it belongs to;
- and the protocol cannot deadlock.

Planted protocol mistakes must each be caught.
"""
import pytest


def explore(nw, F, mutation=None):
    """Depth-first search over all reachable states of nw warps and F parts.
    Returns (violations found, states visited)."""

    def finisher(f):
        return f % nw

    def waits_free(w, f):
        if f < 2:
            return False
        if mutation == "skip_free_wait":
            return False
        return w != finisher(f - 2)

    def slot_set(f):
        return 0 if mutation == "one_slot_set" else f & 1

    # warp state: (f, pc, gen) with pc in
    #   "FW"  wait on FREE (arrive done), "WR" write slot, "FA" FULL step,
    #   "FS"  finisher waiting on FULL, "RD" finisher reads, "DONE"
    # barrier state: tuple of (gen, count) for FULL[0], FULL[1], FREE[0], FREE[1]
    # slots: per set, per warp, part index held (-1 none)
    # read: frozenset of parts whose slots the finisher has read
    def start_pc(w, f):
        return "FREE" if waits_free(w, f) else "WR"

    init = (tuple((0, start_pc(w, 0), -1) for w in range(nw)), ((0, 0),) * 4, ((-1,) * nw,) * 2, frozenset())
    seen = set()
    stack = [init]
    errors = []

    def arrive(bars, idx, intended_gen, what):
        bl = list(bars)
        gen, cnt = bl[idx]
        if gen != intended_gen:
            errors.append(f"{what}: arrival for generation {intended_gen} counted in {gen}")
        cnt += 1
        if cnt == nw:
            bl[idx] = (gen + 1, 0)
        else:
            bl[idx] = (gen, cnt)
        return tuple(bl), gen

    while stack and len(errors) < 5:
        st = stack.pop()
        if st in seen:
            continue
        seen.add(st)
        warps, bars, slots, read = st
        succ = []
        for w, (f, pc, gen) in enumerate(warps):
            if pc == "DONE":
                continue

            def put(new, bars_=bars, slots_=slots, read_=read):
                wl = list(warps)
                wl[w] = new
                succ.append((tuple(wl), bars_, slots_, read_))

            s = slot_set(f)
            if pc == "FREE":  # bar.sync FREE[s]: arrive, then wait for the generation
                nb, g = arrive(bars, 2 + s, (f - 2) // 2 if mutation != "one_slot_set" else f - 2,
                               f"warp {w} FREE part {f}")
                put((f, "FW", g), bars_=nb)
            elif pc == "FW":
                if bars[2 + s][0] > gen:
                    put((f, "WR", -1))
            elif pc == "WR":
                prev = slots[s][w]
                if prev >= 0 and prev not in read:
                    errors.append(f"warp {w} overwrites slot of part {prev} (set {s}) before its finisher read it")
                sl = [list(x) for x in slots]
                sl[s][w] = f
                put((f, "FA", -1), slots_=tuple(tuple(x) for x in sl))
            elif pc == "FA":
                fin = finisher(f)
                if w == fin and mutation != "finisher_does_not_wait":
                    nb, g = arrive(bars, s, f // 2 if mutation != "one_slot_set" else f, f"finisher {w} FULL {f}")
                    put((f, "FS", g), bars_=nb)
                elif w == fin:
                    put((f, "RD", -1))
                else:
                    nb, _ = arrive(bars, s, f // 2 if mutation != "one_slot_set" else f, f"warp {w} FULL {f}")
                    nxt = f + 1
                    put((nxt, start_pc(w, nxt) if nxt < F else "DONE", -1), bars_=nb)
            elif pc == "FS":
                if bars[s][0] > gen:
                    put((f, "RD", -1))
            elif pc == "RD":
                for ww in range(nw):
                    if slots[s][ww] != f:
                        errors.append(f"finisher of part {f} reads warp {ww}'s slot holding part {slots[s][ww]}")
                nread = read | {f}
                nb = bars
                if f + 2 < F and mutation != "finisher_skips_free":
                    nb, _ = arrive(bars, 2 + s, f // 2 if mutation != "one_slot_set" else f,
                                   f"finisher {w} FREE after part {f}")
                nxt = f + 1
                put((nxt, start_pc(w, nxt) if nxt < F else "DONE", -1), bars_=nb, read_=nread)
        if not succ:
            if not all(wst[1] == "DONE" for wst in warps):
                errors.append(f"deadlock: warps={warps} bars={bars}")
        stack.extend(succ)
    return errors, len(seen)


# ---------------------------------------------------------------- the shipped protocol is safe
@pytest.mark.parametrize("nw,F", [(2, 1), (2, 3), (2, 6), (3, 4), (3, 7), (4, 5), (4, 6)])
def test_protocol_has_no_race_or_deadlock(nw, F):
    errors, states = explore(nw, F)
    assert errors == [], errors[:3]
    assert states > 10


# ---------------------------------------------------------------- each planted mistake is caught
@pytest.mark.parametrize("mutation", ["skip_free_wait", "finisher_skips_free", "finisher_does_not_wait",
                                      "one_slot_set"])
def test_planted_protocol_mistakes_are_caught(mutation):
    errors, _ = explore(3, 5, mutation)
    assert errors, f"mutation {mutation} was not caught"
