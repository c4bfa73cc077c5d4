// tfa_sched.h -- how the persistent grid divides the work (host and device).
//
// An *item* is (batch b, query head h, pair qp of 128-row query tiles), or with
// head pairs (batch b, heads 2h and 2h+1, query tile qp); its work is the union
// of the two tiles' key-tile ranges (tfa_plan.h), one *step* per key tile.
// Items are ordered by that group qp (longest first when causal), then batch,
// then head, so the heads of one KV group -- which read the same K/V -- sit
// next to each other.
//
// Split schedule (the default): the concatenated steps of all items are cut
// into `grid` contiguous ranges of (almost) equal length, one per CTA, so every
// CTA gets the same amount of key-tile work whatever the item sizes.  A range
// boundary may cut an item; each piece of a query tile's key range is then a
// separate online-softmax pass whose partial (row max m, row sum l, unscaled
// accumulator a) is merged exactly as tiny-llm "Week 2 Day 5: Tiled Dense
// Prefill Attention", Task 1 merges tile statistics:
//   m' = max(m, m_b),  l' = e^(m-m') l + e^(m_b-m') l_b,  a' = e^(m-m') a + e^(m_b-m') a_b.
// The piece holding the tile's first key tile (its *finalizer*) merges the
// others and writes the output.  Every other piece of the tile is the FIRST
// piece of a later CTA's range, so partials are produced early, and a
// finalizer only ever waits for CTAs after its own: no cycle is possible.
//
// Whole-item schedule (when the estimate favours it, varlen, no-allocation
// entry, debug flag): items go out in snake order; nothing is split or merged.
#pragma once

#include "tfa_plan.h"

namespace tfa {

// Packed variable-length batches: sequence b has q_len[b] query rows from
// packed row q_start[b] and k_len[b] keys from packed row k_start[b] (a
// sequence whose lengths failed validation has q_len 0 and is skipped).
// With `order` set, only the items that exist are dealt: order[i] low 10 bits
// = 1023 - b, high bits = b's item groups (query-tile pairs, or query tiles
// with head pairs), sorted in decreasing order
// (longest sequences first, then by index), and group_start[rr] = the items
// of the groups before group rr (the groups' order as for fixed lengths).
// Group rr holds, for each of its first n sequences of `order`, every head
// (or head pair).
constexpr int kMaxVarlenGroups = 1024;  // item groups for the compact deal
struct SeqTable {
    const int *q_start, *q_len, *k_start, *k_len;
    const unsigned *order;
    const int *group_start;
};

struct Shape {
    int B, Hq, L, S, causal, window;  // varlen: L = longest query, S unused
    unsigned flags;
    int n_qp;   // query-tile pairs per head: ceil(L / 256); with head pairs, ceil(L / 128)
    int grid;   // CTAs
    int split;  // 1: split schedule; 0: whole items in snake order
    // Head pairs: an item's two tiles are the same 128-row query tile of two
    // query heads of one KV group (Hq here counts the pairs), so both visit
    // the same key tiles; otherwise they are two consecutive query tiles of
    // one head, whose key ranges differ at the causal diagonal and the window.
    int hp = 0;
};

TFA_HD int shape_n_qp(int L, int hp = 0) {
    return hp ? (L + kBlockQ - 1) / kBlockQ : (L + 2 * kBlockQ - 1) / (2 * kBlockQ);
}

// Key-tile ranges of the two query tiles of item group qp (a query-tile pair,
// or with head pairs one query tile of both heads).
struct ItemSpan {
    int jl, jh;     // union range
    int lo[2], hi[2];
    bool present[2];
};

TFA_HD ItemSpan item_span_ls(const Shape &s, int L, int S, int qp) {
    ItemSpan sp;
    sp.jl = 0x7fffffff;
    sp.jh = -1;
    for (int t = 0; t < 2; ++t) {
        const int q0 = s.hp ? qp * kBlockQ : qp * 2 * kBlockQ + t * kBlockQ;
        sp.present[t] = q0 < L;
        const KeyRange kr = qtile_key_range(L, S, s.causal, s.window, q0, s.flags);
        sp.lo[t] = kr.lo;
        sp.hi[t] = sp.present[t] ? kr.hi : -1;
        if (sp.present[t]) {
            sp.jl = imin(sp.jl, kr.lo);
            sp.jh = imax(sp.jh, kr.hi);
        }
    }
    return sp;
}

TFA_HD ItemSpan item_span(const Shape &s, int qp) { return item_span_ls(s, s.L, s.S, qp); }

// Items of group r all have query-tile pair (or query tile) group_qp(r).
TFA_HD int group_qp(const Shape &s, int r) { return s.causal ? s.n_qp - 1 - r : r; }

TFA_HD int item_steps(const Shape &s, int qp) {
    const ItemSpan sp = item_span(s, qp);
    return sp.jh - sp.jl + 1;
}

TFA_HD long long total_steps(const Shape &s) {
    long long w = 0;
    for (int r = 0; r < s.n_qp; ++r) w += static_cast<long long>(item_steps(s, group_qp(s, r)));
    return w * s.B * s.Hq;
}

// First global step of CTA c's range (c == grid gives the end).
TFA_HD long long cta_begin(long long W, int grid, int c) { return (W * c) / grid; }

struct Segment {
    int item;       // r * (B * Hq) + b * Hq + h
    int qp, b, h;
    int jb, je;     // key tiles [jb, je] of this piece
    long long x0;   // global index of the item's first step (split schedule)
    int L, S;       // the item's query rows and keys (the call's, or its sequence's)
    int q_base, k_base;  // varlen: first packed query / key row of the sequence
};

// Key-tile ranges of the segment's two tiles, for its own lengths.
TFA_HD ItemSpan seg_span(const Shape &s, const Segment &seg) { return item_span_ls(s, seg.L, seg.S, seg.qp); }

// Per-CTA iterator over its pieces, identical on every role of the CTA.
struct SegIter {
    long long pos, end;   // split: current / end global step
    long long gstart;     // split: first global step of group r
    int r, gsteps, bh;    // split: current group, steps per item in it, items per group
    // whole-item schedule: CTA c visits items c, 2G - 1 - c, 2G + c, 4G - 1 - c,
    // ... (G CTAs): the step alternates between 2G - 1 - 2c and 2c + 1, which sum
    // to 2G.  Items come largest first (causal item groups in decreasing order),
    // so alternating the direction pairs a CTA's large items with small ones.
    // Once a CTA's item is past the end, so are all its later ones.
    int item, stride, n_items;
    SeqTable seq;  // varlen batches (whole-item schedule only); q_start == nullptr otherwise

    TFA_HD void init(const Shape &s, long long W, int c) {
        seq.q_start = seq.q_len = seq.k_start = seq.k_len = nullptr;
        seq.order = nullptr;
        seq.group_start = nullptr;
        bh = s.B * s.Hq;
        n_items = s.n_qp * bh;
        item = c;
        stride = 2 * s.grid - 1 - 2 * c;
        pos = cta_begin(W, s.grid, c);
        end = cta_begin(W, s.grid, c + 1);
        r = 0;
        gstart = 0;
        gsteps = item_steps(s, group_qp(s, 0));
        if (s.split) {
            while (r + 1 < s.n_qp && pos >= gstart + static_cast<long long>(bh) * gsteps) {
                gstart += static_cast<long long>(bh) * gsteps;
                ++r;
                gsteps = item_steps(s, group_qp(s, r));
            }
        }
    }

    TFA_HD bool next(const Shape &s, Segment &seg) {
        if (!s.split) {
            for (;;) {
                if (item >= n_items) return false;
                if (seq.order) {  // varlen, existing items only
                    int lo = 0, hi = s.n_qp - 1;  // last group starting at or before item
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (seq.group_start[mid] <= item) lo = mid;
                        else hi = mid - 1;
                    }
                    const int idx = item - seq.group_start[lo], bi = idx / s.Hq;
                    seg.qp = group_qp(s, lo);
                    seg.b = 1023 - static_cast<int>(seq.order[bi] & 1023u);
                    seg.h = idx - bi * s.Hq;
                } else {
                    const int rr = item / bh, rem = item - rr * bh;
                    seg.qp = group_qp(s, rr);
                    seg.b = rem / s.Hq;
                    seg.h = rem - seg.b * s.Hq;
                }
                seg.item = item;
                item += stride;
                stride = 2 * s.grid - stride;
                seg.L = s.L;
                seg.S = s.S;
                seg.q_base = 0;
                seg.k_base = 0;
                if (seq.q_start) {  // varlen: the sequence's own lengths
                    seg.L = seq.q_len[seg.b];
                    seg.S = seq.k_len[seg.b];
                    seg.q_base = seq.q_start[seg.b];
                    seg.k_base = seq.k_start[seg.b];
                    if (seg.qp * (s.hp ? 1 : 2) * kBlockQ >= seg.L) continue;  // no such tile (pair)
                }
                const ItemSpan sp = seg_span(s, seg);
                seg.jb = sp.jl;
                seg.je = sp.jh;
                seg.x0 = 0;
                return true;
            }
        }
        if (pos >= end) return false;
        while (pos >= gstart + static_cast<long long>(bh) * gsteps) {
            gstart += static_cast<long long>(bh) * gsteps;
            ++r;
            gsteps = item_steps(s, group_qp(s, r));
        }
        const long long in_group = (pos - gstart) / gsteps;
        const long long x0 = gstart + in_group * gsteps;
        const long long stop = end < x0 + gsteps ? end : x0 + gsteps;
        const int rem = static_cast<int>(in_group);
        seg.item = r * bh + rem;
        seg.qp = group_qp(s, r);
        seg.b = rem / s.Hq;
        seg.h = rem - seg.b * s.Hq;
        seg.L = s.L;
        seg.S = s.S;
        seg.q_base = 0;
        seg.k_base = 0;
        const ItemSpan sp = item_span(s, seg.qp);
        seg.jb = sp.jl + static_cast<int>(pos - x0);
        seg.je = sp.jl + static_cast<int>(stop - x0) - 1;
        seg.x0 = x0;
        pos = stop;
        return true;
    }
};

// What a piece does for query tile t.
struct TileRole {
    bool active;     // the piece holds at least one of the tile's key tiles
    int lo, hi;      // those key tiles
    bool finalizer;  // holds the tile's first key tile: writes the output
    bool complete;   // holds all of them: nothing to merge
};

TFA_HD TileRole tile_role(const Shape &s, const Segment &seg, const ItemSpan &sp, int t) {
    TileRole tr;
    tr.lo = imax(sp.lo[t], seg.jb);
    tr.hi = imin(sp.hi[t], seg.je);
    tr.active = sp.present[t] && tr.lo <= tr.hi;
    tr.finalizer = seg.jb <= sp.lo[t];
    tr.complete = !s.split || (tr.finalizer && seg.je >= sp.hi[t]);
    return tr;
}

// For a finalizer piece of tile t cut from its later pieces: the CTAs after
// `c` whose first piece holds some of the tile's key tiles are c+1 .. c_last.
TFA_HD int last_contributor(long long W, int grid, int c, const Segment &seg,
                            const ItemSpan &sp, int t) {
    const long long t_last = seg.x0 + (sp.hi[t] - sp.jl);  // global step of the tile's last key tile
    int cl = c;
    while (cl + 1 < grid && cta_begin(W, grid, cl + 1) <= t_last) ++cl;
    return cl;
}

// Host-side choice between the two schedules: the estimated makespan of each,
// in key-tile steps, counting kPieceCostSteps for every piece a CTA starts
// (pipeline refill, epilogue, and for split pieces the partial merge).  The
// split schedule balances steps exactly but can give some CTAs many small
// pieces; the whole-item schedule has one piece per item but deals whole items.
constexpr int kPieceCostSteps = 6;

inline long long makespan_estimate(Shape s, long long W) {
    long long worst = 0;
    for (int c = 0; c < s.grid; ++c) {
        SegIter it;
        it.init(s, W, c);
        Segment seg;
        long long cost = 0;
        while (it.next(s, seg)) cost += (seg.je - seg.jb + 1) + kPieceCostSteps;
        if (cost > worst) worst = cost;
    }
    return worst;
}

}  // namespace tfa
