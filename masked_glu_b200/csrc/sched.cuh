// sched.cuh -- how the decode kernel splits its work over a persistent grid.
//
// A unit is (row block of ROWS rows of W, k-stage).  Every CTA gets the same
// number of whole row blocks (data-parallel part) plus an equal contiguous
// share of the units of the remaining row blocks (stream-K part); it does its
// stream-K share first.  Plain integer code, also compiled for the host by
// the test suite.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace mglu {
namespace dec {

constexpr int ROWS = 16;

// The work of one CTA: first its stream-K share (units of the last RB_sk row
// blocks, split evenly over the grid), then its whole row blocks.  Every
// role of the CTA walks the same sequence with the same counters; no
// division happens per unit.
struct Sched {
    // 32-bit arithmetic throughout (the host keeps d < 2^22 and rows < 2^27,
    // so every product below fits): the integer divisions run once per CTA.
    int nst;          // k-stages per row block
    int G, cta;       // grid size, this CTA
    int RB;           // row blocks
    int q;            // whole row blocks per CTA
    int rb_sk0;       // first stream-K row block
    uint32_t U_sk;    // stream-K units
    uint32_t sk_b;    // first stream-K unit of this CTA
    int n_sk, n;      // units of this CTA: stream-K, all

    MGLU_HD void init(int rows, int d, int ks_width, int grid, int block)
    {
        nst = (d + ks_width - 1) / ks_width;
        G = grid;
        cta = block;
        RB = (rows + ROWS - 1) / ROWS;
        q = RB / G;
        rb_sk0 = q * G;
        U_sk = (uint32_t)(RB - rb_sk0) * (uint32_t)nst;
        sk_b = sk_begin(cta);
        n_sk = (int)(sk_begin(cta + 1) - sk_b);
        n = n_sk + q * nst;
    }
    // (row block, stage) of the first unit of this CTA
    MGLU_HD void start(int &rb, int &ks) const
    {
        if (n_sk > 0) {
            rb = rb_sk0 + (int)(sk_b / (uint32_t)nst);
            ks = (int)(sk_b % (uint32_t)nst);
        } else {
            rb = cta * q;
            ks = 0;
        }
    }
    // advance after unit i (0-based) of this CTA
    MGLU_HD void next(int i, int &rb, int &ks) const
    {
        if (i + 1 == n_sk) {
            rb = cta * q;
            ks = 0;
        } else if (++ks == nst) {
            ks = 0;
            ++rb;
        }
    }
    // does unit i end this CTA's part of its row block?
    MGLU_HD bool flush_at(int i, int ks) const
    {
        return ks == nst - 1 || i == n_sk - 1 || i == n - 1;
    }
    // CTA whose stream-K share holds stream-K unit v
    MGLU_HD int sk_owner(uint32_t v) const { return (int)(((v + 1) * (uint32_t)G + U_sk - 1) / U_sk) - 1; }
    MGLU_HD uint32_t sk_begin(int c) const { return (uint32_t)c * U_sk / (uint32_t)G; }
    // A stream-K row block rb: the CTAs that hold its units are those of
    // [c_first, c_last] whose share is not empty; returns how many there are.
    MGLU_HD int contributors(int rb, int &c_first, int &c_last) const
    {
        const uint32_t v0 = (uint32_t)(rb - rb_sk0) * (uint32_t)nst;
        c_first = sk_owner(v0);
        c_last = sk_owner(v0 + (uint32_t)nst - 1);
        int n = 0;
        for (int cc = c_first; cc <= c_last; ++cc)
            n += sk_begin(cc + 1) > sk_begin(cc) ? 1 : 0;
        return n;
    }
    // scratch slot of CTA c's partial of stream-K row block rb: each CTA has
    // one for the first row block of its share and one for the last
    MGLU_HD int slot(int c, int rb) const
    {
        return 2 * c + ((uint32_t)(rb - rb_sk0) * (uint32_t)nst <= sk_begin(c) ? 0 : 1);
    }
    MGLU_HD bool contributes(int c) const { return sk_begin(c + 1) > sk_begin(c); }
    // number of units i at which flush_at(i, .) holds: the row blocks the
    // stream-K share touches plus the whole row blocks
    MGLU_HD int flushes() const
    {
        int f = q;
        if (n_sk > 0)
            f += (int)((sk_b + (uint32_t)n_sk - 1u) / (uint32_t)nst - sk_b / (uint32_t)nst) + 1;
        return f;
    }
};

}  // namespace dec
}  // namespace mglu
