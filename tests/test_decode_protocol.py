"""Exhaustive check of the decode kernel's synchronization protocol (no GPU).

A model of one CTA of ``csrc/decode.cuh``, explored over every interleaving
of its threads' steps for small shapes:

* the producer issues stage loads into a ring of S stages. Iteration i may be
  issued once every consumer warp has released iteration i - S (the empty
  barrier). A load writes its stage at any time between issue and landing,
  and landing completes the stage's full barriers;
* each consumer warp waits for its stage, reads it (the read spans two
  steps), then releases it. At the end of a row block it waits on FREE (from
  its second flush on), writes its accumulator slot and arrives on FULL;
* the finisher syncs on FULL, reads every slot, then arrives on FREE (except
  after the last flush).

Named barriers are modelled with hardware generations: an arrival counts
toward the barrier's current generation, whichever flush the arriving warp
means. The model asserts at every step:
- no stage is written while a consumer is reading it;
- no consumer reads a stage holding another iteration's data;
- no slot is overwritten before the finisher has read it;
- every arrival lands in the generation of the flush it belongs to;
- and the protocol cannot deadlock.

Planted protocol mistakes must each be caught.
"""
import pytest

# ---------------------------------------------------------------- the model


def explore(n_cons, n_stages, flushes, mutation=None):
    """Depth-first search over all reachable states. `flushes`: the units at
    which a row block ends (the last unit must be one). Returns the list of
    violations found (empty when the protocol is safe)."""
    N = flushes[-1] + 1
    F = len(flushes)
    flush_of = {u: k for k, u in enumerate(flushes)}
    BAR = n_cons + 1  # named-barrier thread count: consumers + finisher (per warp)

    # state fields
    # prod: next iteration to issue
    # pending: tuple of issued-not-landed iterations
    # landed: per stage, iteration whose data sits there (-1: none)
    # writing: per stage, iteration whose load may be writing it (-1: none)
    # released: per iteration, consumer releases
    # cons: per consumer (i, pc, nflush, arrived_gen) ; pc in W, R, E, F1, F1w, F2, F3, DONE
    # fin: (f, pc, gen)  pc in A (arrive on FULL), Aw (wait, then read the slots), C (arrive on FREE), DONE
    # full: (gen, count) ; free: (gen, count)
    # slot: per consumer, flush index written (-1 none) ; fin_read: last flush read (-1)
    init = (0, (), (-1,) * n_stages, (-1,) * n_stages, (0,) * N,
            tuple((0, "W", 0, -1) for _ in range(n_cons)), (0, "A", -1), (0, 0), (0, 0), (-1,) * n_cons, -1)
    seen = set()
    stack = [init]
    errors = []

    def arrive(bar, intended_gen, what):
        gen, cnt = bar
        if gen != intended_gen:
            errors.append(f"{what}: arrival for generation {intended_gen} counted in {gen}")
        cnt += 1
        if cnt == BAR:
            return (gen + 1, 0), gen
        return (gen, cnt), gen

    while stack and len(errors) < 5:
        st = stack.pop()
        if st in seen:
            continue
        seen.add(st)
        prod, pending, landed, writing, released, cons, fin, full, free, slot, fin_read = st
        succ = []

        # producer: issue iteration prod
        if prod < N:
            s = prod % n_stages
            need = n_cons if mutation != "release_one_short" else n_cons - 1
            if prod < n_stages or released[prod - n_stages] >= need:
                for c, (ci, cpc, _, _) in enumerate(cons):
                    if cpc == "E" and ci % n_stages == s and ci != prod:
                        errors.append(f"stage {s} overwritten (iteration {prod}) while consumer {c} reads {ci}")
                wr = list(writing)
                wr[s] = prod
                succ.append((prod + 1, pending + (prod,), landed, tuple(wr), released, cons, fin, full, free, slot,
                             fin_read))
        # a pending load lands (any order)
        for it in pending:
            s = it % n_stages
            ld = list(landed)
            ld[s] = it
            wr = list(writing)
            wr[s] = -1
            succ.append((prod, tuple(p for p in pending if p != it), tuple(ld), tuple(wr), released, cons, fin,
                         full, free, slot, fin_read))

        # consumers
        for c, (ci, cpc, nfl, agen) in enumerate(cons):
            def with_cons(new, **kw):
                cl = list(cons)
                cl[c] = new
                d = dict(zip(("prod", "pending", "landed", "writing", "released", "cons", "fin", "full", "free",
                              "slot", "fin_read"), st))
                d["cons"] = tuple(cl)
                d.update(kw)
                return (d["prod"], d["pending"], d["landed"], d["writing"], d["released"], d["cons"], d["fin"],
                        d["full"], d["free"], d["slot"], d["fin_read"])

            if cpc == "DONE":
                continue
            s = ci % n_stages
            if cpc == "W":
                if landed[s] == ci or (mutation == "no_full_wait" and prod > ci):
                    succ.append(with_cons((ci, "R", nfl, agen)))
            elif cpc == "R":  # loads issued
                if landed[s] != ci or writing[s] != -1:
                    errors.append(f"consumer {c} reads stage {s} for {ci} holding {landed[s]} "
                                  f"(load writing {writing[s]})")
                if mutation == "release_before_loads_return":
                    rel = list(released)
                    rel[ci] += 1
                    succ.append(with_cons((ci, "E", nfl, agen), released=tuple(rel)))
                else:
                    succ.append(with_cons((ci, "E", nfl, agen)))
            elif cpc == "E":  # loads returned: release the stage
                if writing[s] != -1 and writing[s] != ci:
                    errors.append(f"consumer {c} still reading stage {s} ({ci}) while {writing[s]} writes it")
                rel = list(released)
                if mutation != "release_before_loads_return":
                    rel[ci] += 1
                nxt = "F1" if ci in flush_of else "W"
                nci = ci if ci in flush_of else ci + 1
                if nxt == "W" and nci == N:
                    nxt = "DONE"
                succ.append(with_cons((nci, nxt, nfl, agen), released=tuple(rel)))
            elif cpc == "F1":  # FREE: arrive then wait (from the second flush on)
                if nfl > 0 and mutation != "skip_free_wait":
                    nb, g = arrive(free, nfl - 1, f"consumer {c} FREE")
                    succ.append(with_cons((ci, "F1w", nfl, g), free=nb))
                else:
                    succ.append(with_cons((ci, "F2", nfl, agen)))
            elif cpc == "F1w":
                if free[0] > agen:
                    succ.append(with_cons((ci, "F2", nfl, agen)))
            elif cpc == "F2":  # write the slot
                if slot[c] >= 0 and fin_read < slot[c]:
                    errors.append(f"consumer {c} overwrites slot of flush {slot[c]} before the finisher read it")
                sl = list(slot)
                sl[c] = nfl
                succ.append(with_cons((ci, "F3", nfl, agen), slot=tuple(sl)))
            elif cpc == "F3":  # arrive FULL
                nb, _ = arrive(full, nfl, f"consumer {c} FULL")
                nxt = "W" if ci + 1 < N else "DONE"
                succ.append(with_cons((ci + 1, nxt, nfl + 1, agen), full=nb))

        # finisher
        f, fpc, fgen = fin
        if fpc == "A":  # bar.sync FULL: arrive, then wait for the generation
            nb, g = arrive(full, f, "finisher FULL")
            succ.append((prod, pending, landed, writing, released, cons, (f, "Aw", g), nb, free, slot, fin_read))
        elif fpc == "Aw":
            if full[0] > fgen:
                for c in range(n_cons):
                    if slot[c] != f:
                        errors.append(f"finisher reads flush {f} but consumer {c}'s slot holds {slot[c]}")
                succ.append((prod, pending, landed, writing, released, cons, (f, "C", -1), full, free, slot, f))
        elif fpc == "C":
            if f < F - 1 and mutation != "finisher_skips_free":
                nb, _ = arrive(free, f, "finisher FREE")
                succ.append((prod, pending, landed, writing, released, cons, (f + 1, "A", -1), full, nb, slot,
                             fin_read))
            else:
                nxt = (f + 1, "A", -1) if f < F - 1 else (f, "DONE", -1)
                succ.append((prod, pending, landed, writing, released, cons, nxt, full, free, slot, fin_read))

        if not succ:
            done = all(c[1] == "DONE" for c in cons) and fin[1] == "DONE" and prod == N and not pending
            if not done:
                errors.append(f"deadlock: prod={prod} pending={pending} cons={cons} fin={fin} "
                              f"full={full} free={free}")
        stack.extend(succ)
    return errors, len(seen)


# ---------------------------------------------------------------- the shipped protocol is safe
@pytest.mark.parametrize("n_cons,n_stages,flushes", [
    (2, 2, [1, 3]),         # two row blocks of two stages
    (2, 3, [0, 2, 3]),      # a split row block at each end, as stream-K shares have
    (3, 2, [1, 2]),
    (2, 2, [0, 1, 2]),      # a flush after every stage
    (3, 3, [1, 3, 5]),      # three warps, three stages, three row blocks (about 40 000 states)
])
def test_protocol_has_no_race_or_deadlock(n_cons, n_stages, flushes):
    errors, states = explore(n_cons, n_stages, flushes)
    assert errors == [], errors[:3]
    assert states > 100


# ---------------------------------------------------------------- each planted mistake is caught
@pytest.mark.parametrize("mutation", ["release_one_short", "no_full_wait", "release_before_loads_return",
                                      "skip_free_wait", "finisher_skips_free"])
def test_planted_protocol_mistakes_are_caught(mutation):
    errors, _ = explore(2, 2, [1, 3], mutation)
    assert errors, f"mutation {mutation} was not caught"
