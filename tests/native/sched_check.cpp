// Host check of the decode kernel's work split (masked_glu_b200/csrc/sched.cuh)
// over many shapes and grid sizes: every (row block, k-stage) unit is done by
// exactly one CTA; a row block is either finished inside one CTA or is a
// stream-K row block whose contributors (counted by Sched::contributors) are
// exactly the CTAs that flush a part of it; their scratch slots are distinct
// and each CTA uses each of its two slots for at most one row block; and
// Sched::flushes() counts a CTA's flushes exactly.
// Prints "ok" and exits 0 on success.
#include <cstdio>
#include <map>
#include <set>
#include <vector>

#include "sched.cuh"

using mglu::dec::ROWS;
using mglu::dec::Sched;

static int check(int rows, int d, int ks_width, int G)
{
    Sched ref;
    ref.init(rows, d, ks_width, G, 0);
    const int RB = ref.RB, nst = ref.nst;
    std::vector<int> seen((size_t)RB * nst, 0);
    std::map<int, std::set<int>> flushers;        // stream-K row block -> CTAs flushing it
    std::map<int, int> slot_owner;                // slot -> row block
    std::set<int> complete;                       // row blocks finished inside one CTA
    for (int c = 0; c < G; ++c) {
        Sched sc;
        sc.init(rows, d, ks_width, G, c);
        int rb, ks, cur_rb = -1, seg_start = 0, nflush = 0;
        sc.start(rb, ks);
        for (int i = 0; i < sc.n; sc.next(i, rb, ks), ++i) {
            nflush += sc.flush_at(i, ks) ? 1 : 0;
            if (rb < 0 || rb >= RB || ks < 0 || ks >= nst) {
                std::printf("unit out of range rows=%d d=%d G=%d c=%d rb=%d ks=%d\n", rows, d, G, c, rb, ks);
                return 1;
            }
            seen[(size_t)rb * nst + ks]++;
            if (rb != cur_rb) {  // a new row-block segment of this CTA
                cur_rb = rb;
                seg_start = ks;
            }
            if (!sc.flush_at(i, ks))
                continue;
            const bool whole = seg_start == 0 && ks == nst - 1;
            if (i < sc.n_sk) {
                int cf, cl;
                const int np = sc.contributors(rb, cf, cl);
                if (cf == cl) {
                    if (!whole || cf != c) {
                        std::printf("stream-K row block %d owned by one CTA but not whole (c=%d)\n", rb, c);
                        return 1;
                    }
                    complete.insert(rb);
                } else {
                    flushers[rb].insert(c);
                    const int sl = sc.slot(c, rb);
                    if (sl != 2 * c && sl != 2 * c + 1) {
                        std::printf("slot %d not owned by CTA %d\n", sl, c);
                        return 1;
                    }
                    if (slot_owner.count(sl) && slot_owner[sl] != rb) {
                        std::printf("slot %d used for row blocks %d and %d\n", sl, slot_owner[sl], rb);
                        return 1;
                    }
                    slot_owner[sl] = rb;
                    (void)np;
                }
            } else {
                if (!whole) {
                    std::printf("data-parallel row block %d not whole in CTA %d\n", rb, c);
                    return 1;
                }
                complete.insert(rb);
            }
            cur_rb = -1;  // the next unit starts a new segment
        }
        if (nflush != sc.flushes()) {
            std::printf("CTA %d flushes %d times, flushes() says %d (rows=%d d=%d ks=%d G=%d)\n", c, nflush,
                        sc.flushes(), rows, d, ks_width, G);
            return 1;
        }
    }
    for (size_t u = 0; u < seen.size(); ++u)
        if (seen[u] != 1) {
            std::printf("unit %zu done %d times (rows=%d d=%d ks=%d G=%d)\n", u, seen[u], rows, d, ks_width, G);
            return 1;
        }
    for (auto &kv : flushers) {
        int cf, cl;
        const int np = ref.contributors(kv.first, cf, cl);
        std::set<int> want;
        for (int cc = cf; cc <= cl; ++cc)
            if (ref.contributes(cc))
                want.insert(cc);
        if ((int)kv.second.size() != np || kv.second != want) {
            std::printf("row block %d: %zu CTAs flush it, contributors says %d (rows=%d d=%d G=%d)\n", kv.first,
                        kv.second.size(), np, rows, d, G);
            return 1;
        }
        if (complete.count(kv.first)) {
            std::printf("row block %d both split and complete\n", kv.first);
            return 1;
        }
    }
    if ((int)(complete.size() + flushers.size()) != RB) {
        std::printf("row blocks accounted %zu of %d (rows=%d d=%d G=%d)\n", complete.size() + flushers.size(), RB,
                    rows, d, G);
        return 1;
    }
    return 0;
}

int main()
{
    const int rows_list[] = {1, 16, 40, 200, 1024, 4096, 8192, 14336, 2000};
    const int d_list[] = {8, 128, 200, 640, 2048, 4096, 14336};
    const int ks_list[] = {256, 384, 512, 768, 1024};
    const int g_list[] = {1, 7, 64, 148, 296, 320};
    for (int rows : rows_list)
        for (int d : d_list)
            for (int ks : ks_list)
                for (int G : g_list)
                    if (check(rows, d, ks, G))
                        return 1;
    std::printf("ok\n");
    return 0;
}
