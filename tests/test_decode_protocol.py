"""Exhaustive check of the decode kernel's synchronization protocol (no GPU).

A model of one CTA of ``csrc/decode.cuh``, explored over every interleaving
of its warps' steps for small shapes.  The weight stream itself needs no
model: every lane loads its own operands into its own registers.  What the
warps share is the row-block hand-off through shared memory:

* a CTA's work has F row-block parts (flushes).  With S slot sets (1 or 2)
  every warp writes its accumulators at the end of part f into set f mod S;
* from part S on, every warp first waits on FREE[f mod S] (bar.sync); the
  finisher of part f - S gets there only after it has read that set;
* warp f mod NW finishes part f: after writing its own slot it waits on
  FULL[f mod S] (bar.sync) and reads every slot of the set; the other warps
  arrive on FULL[f mod S] after writing and carry on.

(An earlier form, in which the finisher arrived on FREE and then skipped its
own wait there, is kept as a planted mistake: with one slot set it lets a
warp arrive on the next FREE generation before the current one completes.)

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


def explore(nw, F, mutation=None, sets=2):
    """Depth-first search over all reachable states of nw warps and F parts
    with `sets` slot sets.  Returns (violations found, states visited)."""
    S = sets
    # "one_slot_set": the slots of a single set reused while waits assume two
    reuse = 2 if mutation == "one_slot_set" else S

    def finisher(f):
        return f % nw

    def waits_free(w, f):
        if f < reuse:
            return False
        if mutation == "skip_free_wait":
            return False
        if mutation == "finisher_arrives_and_skips":
            return w != finisher(f - reuse)
        return True

    def slot_set(f):
        return 0 if mutation == "one_slot_set" else f % S

    def gen_free(f):  # generation of FREE[f mod S] that part f waits on
        return (f - reuse) // reuse if mutation != "one_slot_set" else f - reuse

    def gen_full(f):
        return f // S if mutation != "one_slot_set" else f

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
                nb, g = arrive(bars, 2 + s, gen_free(f), f"warp {w} FREE part {f}")
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
                    nb, g = arrive(bars, s, gen_full(f), f"finisher {w} FULL {f}")
                    put((f, "FS", g), bars_=nb)
                elif w == fin:
                    put((f, "RD", -1))
                else:
                    nb, _ = arrive(bars, s, gen_full(f), f"warp {w} FULL {f}")
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
                if mutation == "finisher_arrives_and_skips" and f + reuse < F:
                    nb, _ = arrive(bars, 2 + s, f // reuse, f"finisher {w} FREE after part {f}")
                nxt = f + 1
                put((nxt, start_pc(w, nxt) if nxt < F else "DONE", -1), bars_=nb, read_=nread)
        if not succ:
            if not all(wst[1] == "DONE" for wst in warps):
                errors.append(f"deadlock: warps={warps} bars={bars}")
        stack.extend(succ)
    return errors, len(seen)


# ---------------------------------------------------------------- the shipped protocol is safe
@pytest.mark.parametrize("sets", [1, 2])
@pytest.mark.parametrize("nw,F", [(2, 1), (2, 3), (2, 6), (3, 4), (3, 7), (4, 5), (4, 6)])
def test_protocol_has_no_race_or_deadlock(nw, F, sets):
    errors, states = explore(nw, F, sets=sets)
    assert errors == [], errors[:3]
    assert states > 10


# ---------------------------------------------------------------- each planted mistake is caught
@pytest.mark.parametrize("sets", [1, 2])
@pytest.mark.parametrize("mutation", ["skip_free_wait", "finisher_does_not_wait"])
def test_planted_protocol_mistakes_are_caught(mutation, sets):
    errors, _ = explore(3, 5, mutation, sets=sets)
    assert errors, f"mutation {mutation} was not caught"


def test_one_set_reused_as_if_two_is_caught():
    errors, _ = explore(3, 5, "one_slot_set")
    assert errors


def test_finisher_that_arrives_and_skips_its_wait_races_with_one_set():
    errors, _ = explore(2, 3, "finisher_arrives_and_skips", sets=1)
    assert any("overwrites" in e or "generation" in e for e in errors)
