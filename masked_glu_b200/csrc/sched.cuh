// sched.cuh -- how the decode kernel splits its work over a persistent grid.
//
// A unit is (row block of ROWS rows of W, step of k: 32 k per MMA unit
// times the MMA units a warp takes at once).  The units
// are numbered row block by row block, u = rb * nsw + s, and every warp of the
// grid gets an equal contiguous range of them (warp-level stream-K): warp gw
// of GW does [begin(gw), begin(gw + 1)).  A warp never waits for another while
// it streams.  Its range meets a row block in one segment: a middle segment
// covers the whole row block and the warp finishes it alone; the first and
// the last segment of the range may be partial, and partial segments are
// combined after the stream, inside the CTA (its warps' ranges are adjacent)
// and, for the first and last row block of a CTA's range, across CTAs.
// Plain integer code, also compiled for the host by the test suite.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace mglu {
namespace dec {

constexpr int ROWS = 16;

struct Plan {
    int nsw;     // units per row block (ceil(d / step))
    int RB;      // row blocks
    uint32_t U;  // units, RB * nsw (the host keeps it below 2^31)
    int GW;      // warps of the grid
    int NW;      // warps per CTA

    MGLU_HD void init(int rows, int d, int step, int grid, int nw)
    {
        nsw = (d + step - 1) / step;
        RB = (rows + ROWS - 1) / ROWS;
        U = (uint32_t)RB * (uint32_t)nsw;
        NW = nw;
        GW = grid * nw;
    }
    // first unit of warp gw (gw = GW gives U)
    MGLU_HD uint32_t begin(int gw) const { return (uint32_t)((uint64_t)gw * U / (uint64_t)GW); }
    // warp whose range holds unit u
    MGLU_HD int owner(uint32_t u) const { return (int)(((uint64_t)(u + 1) * (uint64_t)GW - 1u) / U); }
    MGLU_HD int cta_owner(uint32_t u) const { return owner(u) / NW; }
    // row blocks touched by CTA c: [first_rb(c), last_rb(c)] (c must have units)
    MGLU_HD int first_rb(int c) const { return (int)(begin(c * NW) / (uint32_t)nsw); }
    MGLU_HD int last_rb(int c) const { return (int)((begin((c + 1) * NW) - 1u) / (uint32_t)nsw); }
    MGLU_HD bool cta_has_units(int c) const { return begin((c + 1) * NW) > begin(c * NW); }
    // does warp gw's range cover every unit of row block rb?
    MGLU_HD bool covers(int gw, int rb) const
    {
        return begin(gw) <= (uint32_t)rb * (uint32_t)nsw && begin(gw + 1) >= (uint32_t)(rb + 1) * (uint32_t)nsw;
    }
    // CTAs whose ranges meet row block rb: [c_first, c_last]
    MGLU_HD void ctas_of(int rb, int &c_first, int &c_last) const
    {
        c_first = cta_owner((uint32_t)rb * (uint32_t)nsw);
        c_last = cta_owner((uint32_t)(rb + 1) * (uint32_t)nsw - 1u);
    }
    // global partial slot of CTA c for row block rb (rb is c's first or last)
    MGLU_HD int slot(int c, int rb) const { return 2 * c + (rb == first_rb(c) ? 0 : 1); }
};

}  // namespace dec
}  // namespace mglu
