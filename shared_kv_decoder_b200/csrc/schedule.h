// Work schedules of the persistent kernels: which work tile a CTA takes in
// which round, the KV tile range of a prefill work tile, which of those tiles
// need the mask, and how a decode sequence splits into units.  The kernels
// and the host-side schedule dump (yoco_debug_tile_schedule) both call these
// functions, so the dump shows the kernels' own index arithmetic.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define YOCO_HD __host__ __device__ __forceinline__
#else
#define YOCO_HD inline
#endif

namespace yoco {
namespace sched {

constexpr int kPrefillBM = 128;  // query rows per work tile
constexpr int kPrefillBN = 128;  // keys per KV tile

YOCO_HD int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
YOCO_HD int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Prefill work tiles are numbered heaviest causal tile first: all (head,
// batch) pairs of the last query tile, then of the one before, and so on.
struct PrefillWork {
    int qt, h, b, g;              // query tile, query head, batch, KV head
    int64_t i0;                   // first query row
    int64_t p_first, p_last;      // absolute positions of the first / last real row
    int jt_lo, n_kv;              // first KV tile, number of KV tiles
};

struct PrefillShape {
    int32_t B, Hq, Hkv;
    int64_t Tq, Tkv, q_pos0;
    int32_t window;               // 0: causal
    int32_t n_qtiles;
};

// The KV range of query tile qt of (batch b, query head h).
YOCO_HD PrefillWork prefill_work_at(const PrefillShape &s, int qt, int h, int b) {
    PrefillWork x;
    x.qt = qt;
    x.h = h;
    x.b = b;
    x.g = x.h / (s.Hq / s.Hkv);
    x.i0 = (int64_t)x.qt * kPrefillBM;
    const int64_t i_last = min64(x.i0 + kPrefillBM, s.Tq) - 1;
    x.p_first = s.q_pos0 + x.i0;
    x.p_last = s.q_pos0 + i_last;
    // visible keys of the tile: j <= p (and j > p - window), j < Tkv
    const int64_t j_lo = s.window > 0 ? max64(0, x.p_first - s.window + 1) : 0;
    const int64_t j_hi = min64(s.Tkv - 1, x.p_last);
    x.jt_lo = (int)(j_lo / kPrefillBN);
    x.n_kv = (int)(j_hi / kPrefillBN) - x.jt_lo + 1;
    return x;
}

// One query head per work tile (any group size).
YOCO_HD PrefillWork prefill_work(const PrefillShape &s, int w) {
    const int per = s.Hq * s.B;
    return prefill_work_at(s, s.n_qtiles - 1 - w / per, (w % per) % s.Hq, (w % per) / s.Hq);
}

// Two query heads per work tile, 2hp and 2hp + 1, which share their KV head
// when the group size Hq / Hkv is even: n_work = n_qtiles * (Hq / 2) * B.
// The returned h is the first head of the pair.
YOCO_HD PrefillWork prefill_pair_work(const PrefillShape &s, int w) {
    const int hp = s.Hq / 2, per = hp * s.B;
    return prefill_work_at(s, s.n_qtiles - 1 - w / per, 2 * ((w % per) % hp), (w % per) / hp);
}

// The paired kernel serves bf16 shapes whose group size is even.
YOCO_HD bool prefill_pairs_heads(int Hq, int Hkv) { return (Hq / Hkv) % 2 == 0; }

// Work tile of round r for CTA c of a G-CTA grid: rounds alternate direction
// (snake order), so with the works sorted heaviest first every CTA gets a
// similar total.  Values >= n_work mean the CTA is done.
YOCO_HD int prefill_work_index(int r, int c, int G) { return r * G + ((r & 1) ? G - 1 - c : c); }

// Does KV tile t of work x hold a (row, key) pair that is not visible, or a
// key past Tkv?  Only such tiles run the per-element mask.
YOCO_HD bool prefill_tile_masked(const PrefillShape &s, const PrefillWork &x, int t) {
    const int64_t j0 = (int64_t)(x.jt_lo + t) * kPrefillBN;
    return (j0 + kPrefillBN - 1 > x.p_first) || (j0 + kPrefillBN > s.Tkv) ||
           (s.window > 0 && j0 <= x.p_last - s.window);
}

// Decode units of a sequence of len tokens: ceil(len / split) contiguous
// ranges of split tokens, never more than the n_split the workspace holds.
YOCO_HD int64_t decode_units(int64_t len, int64_t split, int64_t n_split) {
    return len > 0 ? min64((len + split - 1) / split, n_split) : 0;
}

}  // namespace sched
}  // namespace yoco
