"""Exhaustive check of the decode kernel's synchronization protocol (no GPU).

A model of one CTA of ``csrc/decode.cuh``, explored over every interleaving
of its warps' steps for small shapes.  The weight stream itself needs no
model: every lane loads its own operands into its own registers.  What the
warps share is the row-block hand-off through shared memory:

* a CTA's work has F row-block parts (flushes).  With S slot sets (1 or 2)
  every warp writes its accumulators at the end of part f into set f mod S;
* from part S on, every warp except the finisher of part f - S first waits
  on FREE[f mod 2] (bar.sync); that finisher arrived on FREE[f mod 2] as soon
  as it had read the set, and does not wait there;
* warp f mod NW finishes part f: after writing its own slot it waits on
  FULL[f mod S] (bar.sync), reads every slot of the set and, if part f + S
  exists, arrives on FREE[(f + S) mod 2]; the other warps arrive on
  FULL[f mod S] after writing and carry on.

The FREE barrier alternates by part, not by slot set: with one set, a barrier
per set would let the early-released finisher arrive on the next generation
before the current one completes (kept as a planted mistake).

Named barriers are modelled with hardware generations: an arrival counts
toward the barrier's current generation, whichever part the arriving warp
means, and a generation completes once all NW warps have arrived.  The model
asserts at every step:
- no slot is overwritten before the finisher of its previous part read it;
- the finisher reads every slot holding its own part;
- every arrival lands in the generation of the part it belongs to;
- and the protocol cannot deadlock.

Planted protocol mistakes must each be caught.

The instances for 8 and 16 tokens finish cooperatively instead (explore_coop):
one slot set, the first R warps reduce (one thread per output), every part
ends with a bar.sync of all warps on FULL, the reducers meet on READ after
reading (twice more for a row block split between CTAs) and release the set
on FREE, on which the other warps wait before writing the next part.
"""
import pytest


def explore(nw, F, mutation=None, sets=2):
    """Depth-first search over all reachable states of nw warps and F parts
    with `sets` slot sets.  Returns (violations found, states visited)."""
    S = sets

    def finisher(f):
        return f % nw

    def free_bar(f):  # the FREE barrier guarding the writes of part f
        return f % S if mutation == "free_id_by_set" else f % 2

    def waits_free(w, f):
        if f < S or mutation == "skip_free_wait":
            return False
        return w != finisher(f - S)

    def slot_set(f):
        return f % S

    def gen_free(f):  # generation of FREE[free_bar(f)] that part f uses
        return (f - S) // 2 if mutation != "free_id_by_set" else (f - S) // S

    def gen_full(f):
        return f // S

    # warp state: (f, pc, gen) with pc in
    #   "FREE" arrive on FREE then "FW" wait for its generation, "WR" write the
    #   slot, "FA" the FULL step, "FS" the finisher waiting on FULL, "RD" the
    #   finisher reading the set, "DONE"
    # barrier state: (gen, count) for FULL[0], FULL[1], FREE[0], FREE[1]
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
            if pc == "FREE":  # bar.sync FREE: arrive, then wait for the generation
                nb, g = arrive(bars, 2 + free_bar(f), gen_free(f), f"warp {w} FREE part {f}")
                put((f, "FW", g), bars_=nb)
            elif pc == "FW":
                if bars[2 + free_bar(f)][0] > gen:
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
                if f + S < F and mutation != "finisher_skips_free":
                    # released as soon as the set is read, for part f + S
                    nb, _ = arrive(bars, 2 + free_bar(f + S), gen_free(f + S), f"finisher {w} FREE after part {f}")
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
@pytest.mark.parametrize("mutation", ["skip_free_wait", "finisher_skips_free", "finisher_does_not_wait"])
def test_planted_protocol_mistakes_are_caught(mutation, sets):
    errors, _ = explore(3, 5, mutation, sets=sets)
    assert errors, f"mutation {mutation} was not caught"


def test_free_barrier_chosen_by_slot_set_races_with_one_set():
    """With one slot set, a FREE barrier per set (instead of alternating by
    part) lets the early-released finisher arrive on the next generation
    before the current one completes."""
    errors, _ = explore(2, 3, "free_id_by_set", sets=1)
    assert any("generation" in e or "overwrites" in e for e in errors)


# ---------------------------------------------------------------- cooperative finishing
def explore_coop(nw, R, F, mutation=None, split=(0,)):
    """The protocol of the token-capacity 8 and 16 instances: one slot set,
    the first R warps are reducers.  Per part f every warp writes its slot
    (non-reducers first wait on FREE from part 1 on), all warps bar.sync on
    FULL, then each reducer reads every slot, the reducers bar.sync on READ
    (three times in parts listed in `split`, which publish a partial to the
    other CTAs) and, if a later part exists and R < nw, arrive on FREE.
    Returns (violations found, states visited)."""
    extra = {f: 2 for f in split}  # the two further READ syncs of a split part

    def read_syncs(f):
        return 1 + extra.get(f, 0)

    # warp: (f, pc, k, gen); pc in FREE, FW, WR, FULL, FULLW, RD, RS, RSW, DONE
    # bars: (gen, count) for FULL, READ, FREE
    # slots: part held per warp; readers: frozenset of (part, reducer) reads done
    def is_red(w):
        return w < R

    def start(w, f):
        if f >= F:
            return (f, "DONE", 0, -1)
        waits = f >= 1 and not is_red(w) and mutation != "nonreducer_skips_free"
        return (f, "FREE" if waits else "WR", 0, -1)

    counts = {0: nw, 1: R, 2: nw}
    read_gen_base = [0]
    for f in range(F):
        read_gen_base.append(read_gen_base[-1] + read_syncs(f))

    init = (tuple(start(w, 0) for w in range(nw)), ((0, 0),) * 3, (-1,) * nw, frozenset())
    seen, stack, errors = set(), [init], []

    def arrive(bars, idx, intended, what):
        bl = list(bars)
        gen, cnt = bl[idx]
        if gen != intended:
            errors.append(f"{what}: arrival for generation {intended} counted in {gen}")
        cnt += 1
        bl[idx] = (gen + 1, 0) if cnt == counts[idx] else (gen, cnt)
        return tuple(bl), gen

    while stack and len(errors) < 5:
        st = stack.pop()
        if st in seen:
            continue
        seen.add(st)
        warps, bars, slots, readers = st
        succ = []
        for w, (f, pc, k, gen) in enumerate(warps):
            if pc == "DONE":
                continue

            def put(new, bars_=bars, slots_=slots, readers_=readers):
                wl = list(warps)
                wl[w] = new
                succ.append((tuple(wl), bars_, slots_, readers_))

            if pc == "FREE":
                nb, g = arrive(bars, 2, f - 1, f"warp {w} FREE part {f}")
                put((f, "FW", 0, g), bars_=nb)
            elif pc == "FW":
                if bars[2][0] > gen:
                    put((f, "WR", 0, -1))
            elif pc == "WR":
                prev = slots[w]
                if prev >= 0 and any((prev, r) not in readers for r in range(R)):
                    errors.append(f"warp {w} overwrites its slot of part {prev} before every reducer read it")
                sl = list(slots)
                sl[w] = f
                put((f, "FULL", 0, -1), slots_=tuple(sl))
            elif pc == "FULL":
                if is_red(w) and mutation == "reducer_does_not_wait_full":
                    nb, _ = arrive(bars, 0, f, f"reducer {w} FULL {f}")
                    put((f, "RD", 0, -1), bars_=nb)
                else:
                    nb, g = arrive(bars, 0, f, f"warp {w} FULL {f}")
                    put((f, "FULLW", 0, g), bars_=nb)
            elif pc == "FULLW":
                if bars[0][0] > gen:
                    put((f, "RD", 0, -1) if is_red(w) else start(w, f + 1))
            elif pc == "RD":
                for ww in range(nw):
                    if slots[ww] != f:
                        errors.append(f"reducer {w} of part {f} reads warp {ww}'s slot holding part {slots[ww]}")
                nr = readers | {(f, w)}
                if mutation == "no_read_sync":
                    nb = bars
                    if f + 1 < F and R < nw:
                        nb, _ = arrive(bars, 2, f, f"reducer {w} FREE after part {f}")
                    put(start(w, f + 1), bars_=nb, readers_=nr)
                else:
                    put((f, "RS", 0, -1), readers_=nr)
            elif pc == "RS":
                nb, g = arrive(bars, 1, read_gen_base[f] + k, f"reducer {w} READ {f}.{k}")
                put((f, "RSW", k, g), bars_=nb)
            elif pc == "RSW":
                if bars[1][0] > gen:
                    nb = bars
                    if k == 0 and f + 1 < F and R < nw and mutation != "reducer_skips_free":
                        nb, _ = arrive(bars, 2, f, f"reducer {w} FREE after part {f}")
                    if k + 1 < read_syncs(f):
                        put((f, "RS", k + 1, -1), bars_=nb)
                    else:
                        put(start(w, f + 1), bars_=nb)
        if not succ and not all(x[1] == "DONE" for x in warps):
            errors.append(f"deadlock: warps={warps} bars={bars}")
        stack.extend(succ)
    return errors, len(seen)


@pytest.mark.parametrize("nw,R,F,split", [(2, 1, 4, (0,)), (3, 1, 4, (0, 3)), (3, 2, 4, (1,)), (4, 2, 3, (0, 2)),
                                          (3, 3, 4, (0,)), (4, 1, 3, (0,))])
def test_cooperative_protocol_has_no_race_or_deadlock(nw, R, F, split):
    errors, states = explore_coop(nw, R, F, split=split)
    assert errors == [], errors[:3]
    assert states > 10


@pytest.mark.parametrize("mutation", ["nonreducer_skips_free", "reducer_does_not_wait_full", "no_read_sync",
                                      "reducer_skips_free"])
def test_cooperative_planted_mistakes_are_caught(mutation):
    errors, _ = explore_coop(3, 2, 4, mutation, split=(0,))
    assert errors, f"mutation {mutation} was not caught"
