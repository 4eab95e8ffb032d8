// ksplit.cuh -- the work schedule of the persistent GEMM kernels, with the
// tiles of the last, partial wave split along K.
//
// A GEMM of T output tiles on P workers (CTAs, or CTA pairs) runs whole tiles
// c, c + P, ... on worker c.  When T is not a multiple of P the last wave
// leaves P - (T mod P) workers idle for a whole tile.  With the split, the
// first T_dp = T - (T mod P) tiles still run whole (T_dp / P per worker); the
// remaining R = T mod P tiles are cut into groups of two K stages (the scale
// tiles travel two stages per copy), R * ng groups in all (ng = ceil(KT / 2)),
// and worker c takes the contiguous groups [c S / P, (c + 1) S / P) of that
// sequence (S = R * ng, S >= P so that no range is empty).
//
// A range is shorter than a tile (R < P), so it holds at most two pieces: the
// end of one tile (stages up to KT: the tile's finishing piece) and the start
// of the next (a partial piece); a range inside one tile is a single piece.
// Every worker whose range ends inside a tile leaves one partial sum, so the
// partial sums fit one slot per worker, and the worker index is the slot.  The
// finishing piece's worker adds the partial sums of workers first .. c - 1 (in
// that order) to its own accumulator and runs the epilogue.
//
// Each worker runs its whole tiles first and then its pieces in reverse order:
// its partial piece before its finishing piece.  A partial piece therefore is
// the first split work of its worker and never waits for anything, and a
// finishing piece comes last, so by the time it needs the partial sums of the
// workers before it they have normally been written.
//
// Host and device share these functions: the host plans the split and tests
// the schedule (mx_debug_split_units), the kernels walk it.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define MX_HD __host__ __device__ __forceinline__
#else
#define MX_HD inline
#endif

namespace mx {

enum : int { kUnitWhole = 0, kUnitPartial = 1, kUnitFinish = 2 };

// Slots of partial sums a workspace provides: one per CTA of the largest grid
// (148 SMs: 148 single CTAs or 74 pairs of two).
constexpr int kSplitSlots = 148;
// Most workers that share one tile (its finishing worker adds the others'
// partial sums one after the other).
constexpr int kSplitWorkersPerTile = 8;

struct KSplitPlan {
    int on;          // 0: whole tiles c, c + workers, ... only
    int workers;     // P
    int tiles;       // T
    int kt;          // K stages per tile
    int dp_tiles;    // tiles run whole before the split (a multiple of workers)
    int groups;      // two-stage groups per tile (ceil(kt / 2))
    int64_t total;   // groups of the split tiles (S)
};

struct KUnit {
    int tile;    // output tile index (the kernels' tile order)
    int kb, ke;  // K stages [kb, ke)
    int kind;    // kUnitWhole, kUnitPartial or kUnitFinish
    int first;   // kUnitFinish: the first worker holding a partial sum of this tile
};

// First group of worker c's range.
MX_HD int64_t ks_begin(const KSplitPlan &s, int c) { return (int64_t)c * s.total / s.workers; }

// The worker whose range holds group x: the largest c with ks_begin(c) <= x.
MX_HD int ks_worker_of(const KSplitPlan &s, int64_t x) {
    return (int)(((x + 1) * s.workers + s.total - 1) / s.total) - 1;
}

// Work units of worker c.
MX_HD int ks_units(const KSplitPlan &s, int c) {
    if (!s.on) return c < s.tiles ? (s.tiles - c + s.workers - 1) / s.workers : 0;
    const int64_t g0 = ks_begin(s, c), g1 = ks_begin(s, c + 1);
    const int pieces = (int)((g1 - 1) / s.groups - g0 / s.groups) + 1;
    return s.dp_tiles / s.workers + pieces;
}

// Unit u of worker c (0 <= u < ks_units(s, c)).
MX_HD KUnit ks_unit(const KSplitPlan &s, int c, int u) {
    KUnit r;
    r.first = c;
    const int nd = s.on ? s.dp_tiles / s.workers : (1 << 30);
    if (u < nd) {
        r.tile = c + u * s.workers;
        r.kb = 0;
        r.ke = s.kt;
        r.kind = kUnitWhole;
        return r;
    }
    const int64_t g0 = ks_begin(s, c), g1 = ks_begin(s, c + 1);
    const int64_t t = (g1 - 1) / s.groups - (u - nd);  // pieces in reverse order
    const int64_t tg = t * s.groups;
    const int64_t kb = (g0 > tg ? g0 : tg) - tg, ke = (g1 < tg + s.groups ? g1 : tg + s.groups) - tg;
    r.tile = s.dp_tiles + (int)t;
    r.kb = (int)(2 * kb);
    r.ke = (int)(2 * ke) < s.kt ? (int)(2 * ke) : s.kt;
    if (r.kb == 0 && r.ke == s.kt) {
        r.kind = kUnitWhole;
    } else if (r.ke == s.kt) {
        r.kind = kUnitFinish;
        r.first = ks_worker_of(s, tg);
    } else {
        r.kind = kUnitPartial;
    }
    return r;
}

// Total K stages of worker c's units.
MX_HD int ks_stages(const KSplitPlan &s, int c) {
    const int n = ks_units(s, c);
    int total = 0;
    for (int u = 0; u < n; ++u) {
        const KUnit x = ks_unit(s, c, u);
        total += x.ke - x.kb;
    }
    return total;
}

// The plan for T tiles of kt stages on at most `workers` workers.  mode 0:
// split when there are at most half as many tiles as workers and each
// worker's share is 16 K stages or more (a GEMM with few output tiles and a
// long K, such as a decode-time projection with a small N); 1: never; 2:
// whenever possible (also the last wave of a GEMM of several waves).  At most kSplitWorkersPerTile workers share a tile.
// `allowed`: the caller has the slots.  Without a split the grid has
// min(T, workers) workers.
inline KSplitPlan ks_plan(int64_t tiles, int workers, int kt, int mode, bool allowed) {
    KSplitPlan s;
    s.on = 0;
    s.tiles = (int)tiles;
    s.kt = kt;
    s.workers = (int)(tiles < workers ? tiles : workers);
    s.dp_tiles = s.tiles;
    s.groups = (kt + 1) / 2;
    s.total = 0;
    if (!allowed || mode == 1 || workers < 2 || workers > kSplitSlots || kt < 4 || tiles <= 0) return s;
    if (mode == 0 && tiles * 2 > workers) return s;
    if (tiles * kSplitWorkersPerTile < workers) workers = (int)(tiles * kSplitWorkersPerTile);
    // and only with K long enough that each worker's share (8 groups, 16
    // stages or more) outweighs the partial sums' round trips
    if (mode == 0 && tiles * (int64_t)s.groups < 8 * (int64_t)workers) return s;
    const int64_t rem = tiles % workers;
    if (rem == 0) return s;
    const int64_t total = rem * s.groups;
    if (total < workers) return s;
    s.on = 1;
    s.workers = workers;
    s.dp_tiles = (int)(tiles - rem);
    s.total = total;
    return s;
}

}  // namespace mx
