// Host check of the decode kernel's work split (masked_glu_b200/csrc/sched.cuh)
// over many shapes and grid sizes, following the kernel's own steps:
//  - every (row block, unit) is streamed by exactly one warp;
//  - a warp's range meets each row block in one segment; only its first
//    segment can go to the head slot and only its last stays as the tail;
//  - after the stream, the CTA's combine for a row block adds exactly the
//    partial segments its warps hold of it (head or tail as the kernel picks
//    them), and publishes to a scratch slot that no other row block uses;
//  - split_kernel's chosen CTA adds exactly the CTAs that published that
//    row block;
//  - every row block's outputs are written exactly once.
// Prints "ok" and exits 0 on success.
#include <cstdio>
#include <map>
#include <set>
#include <vector>

#include "sched.cuh"

using mglu::dec::Plan;

static int fail(const char *what, int rows, int d, int G, int NW, int a, int b)
{
    std::printf("%s (rows=%d d=%d grid=%d nw=%d: %d %d)\n", what, rows, d, G, NW, a, b);
    return 1;
}

static int check(int rows, int d, int step, int G, int NW)
{
    Plan pl;
    pl.init(rows, d, step, G, NW);
    const int RB = pl.RB, nsw = pl.nsw;
    std::vector<int> seen((size_t)pl.U, 0), written(RB, 0);
    // partial segments: row block -> warps holding one, and which slot kind
    std::map<int, std::map<int, char>> partial;  // rb -> (warp -> 'h' or 't')
    for (int gw = 0; gw < pl.GW; ++gw) {
        const uint32_t u0 = pl.begin(gw), u1 = pl.begin(gw + 1);
        const int n = (int)(u1 - u0);
        int rb = (int)(u0 / nsw), s = (int)(u0 % nsw), seg_start = s;
        for (int i = 0; i < n; ++i) {
            const uint32_t u = u0 + (uint32_t)i;
            if (u != (uint32_t)rb * nsw + (uint32_t)s || rb >= RB)
                return fail("unit numbering", rows, d, G, NW, gw, i);
            if (pl.owner(u) != gw)
                return fail("owner() disagrees with begin()", rows, d, G, NW, gw, (int)u);
            seen[u]++;
            if (s == nsw - 1 || i == n - 1) {
                if (seg_start == 0 && s == nsw - 1) {
                    if (!pl.covers(gw, rb))
                        return fail("whole segment not covered", rows, d, G, NW, gw, rb);
                    written[rb]++;
                } else if (i < n - 1) {
                    if (rb != (int)(u0 / nsw))
                        return fail("head slot used by a later segment", rows, d, G, NW, gw, rb);
                    partial[rb][gw] = 'h';
                } else {
                    partial[rb][gw] = 't';
                }
                seg_start = 0;
            }
            if (++s == nsw)
                s = 0, ++rb;
        }
    }
    for (uint32_t u = 0; u < pl.U; ++u)
        if (seen[u] != 1)
            return fail("unit not streamed exactly once", rows, d, G, NW, (int)u, seen[u]);
    std::map<int, int> slot_rb;                 // scratch slot -> row block
    std::map<int, std::set<int>> published;     // row block -> CTAs that stored sums
    for (int c = 0; c < G; ++c) {
        if (!pl.cta_has_units(c))
            continue;
        const int w0 = c * NW;
        for (int rb = pl.first_rb(c); rb <= pl.last_rb(c); ++rb) {
            const uint32_t ub = (uint32_t)rb * nsw, ue = ub + nsw;
            int w_lo = pl.owner(ub), w_hi = pl.owner(ue - 1u);
            if (w_lo == w_hi) {
                if (partial.count(rb))
                    return fail("row block skipped but has partial segments", rows, d, G, NW, c, rb);
                continue;
            }
            w_lo = w_lo > w0 ? w_lo : w0;
            w_hi = w_hi < w0 + NW - 1 ? w_hi : w0 + NW - 1;
            std::set<int> used;
            for (int w = w_lo; w <= w_hi; ++w) {
                if (pl.begin(w + 1) == pl.begin(w))
                    continue;  // an empty range holds nothing (its slots are never read)
                const int first = (int)(pl.begin(w) / nsw), last = (int)((pl.begin(w + 1) - 1u) / nsw);
                const char kind = (rb == first && first != last) ? 'h' : 't';
                auto it = partial.find(rb);
                if (it == partial.end() || !it->second.count(w) || it->second.at(w) != kind)
                    return fail("combine reads a slot that does not hold this row block", rows, d, G, NW, w, rb);
                used.insert(w);
            }
            for (auto &kv : partial[rb])
                if (kv.first / NW == c && !used.count(kv.first))
                    return fail("combine misses a partial segment", rows, d, G, NW, kv.first, rb);
            int cf, cl;
            pl.ctas_of(rb, cf, cl);
            if (cf == cl) {
                written[rb]++;
            } else {
                const int sl = pl.slot(c, rb);
                if (sl != 2 * c && sl != 2 * c + 1)
                    return fail("slot outside the CTA's pair", rows, d, G, NW, c, sl);
                if (slot_rb.count(sl) && slot_rb[sl] != rb)
                    return fail("slot reused for two row blocks", rows, d, G, NW, sl, rb);
                slot_rb[sl] = rb;
                published[rb].insert(c);
            }
        }
    }
    for (int c = 0; c < G; ++c) {  // split_kernel
        if (!pl.cta_has_units(c))
            continue;
        const int rb = pl.last_rb(c);
        int cf, cl;
        pl.ctas_of(rb, cf, cl);
        if (cf == cl || cf != c)
            continue;
        std::set<int> adds;
        for (int cc = cf; cc <= cl; ++cc)
            if (pl.cta_has_units(cc)) {
                adds.insert(cc);
                if (slot_rb.count(pl.slot(cc, rb)) == 0 || slot_rb[pl.slot(cc, rb)] != rb)
                    return fail("split adds a slot that holds another row block", rows, d, G, NW, cc, rb);
            }
        if (adds != published[rb])
            return fail("split adds a different set of CTAs than published", rows, d, G, NW, c, rb);
        written[rb]++;
    }
    for (int rb = 0; rb < RB; ++rb)
        if (written[rb] != 1)
            return fail("row block not written exactly once", rows, d, G, NW, rb, written[rb]);
    return 0;
}

int main()
{
    const int rows_list[] = {1, 7, 16, 17, 33, 100, 256, 1000, 2048, 8192, 14336};
    const int d_list[] = {8, 64, 72, 200, 512, 1000, 2048, 4096};
    const int grids[] = {1, 2, 3, 7, 148, 320};
    const int nws[] = {8, 12, 16};
    const int steps[] = {64, 128};
    for (int rows : rows_list)
        for (int d : d_list)
            for (int step : steps)
                for (int G : grids)
                    for (int NW : nws) {
                        Plan pl;
                        pl.init(rows, d, step, G, NW);
                        if ((uint32_t)G > pl.U)
                            continue;  // the host caps the grid at the number of units
                        if (check(rows, d, step, G, NW))
                            return 1;
                    }
    std::printf("ok\n");
    return 0;
}
