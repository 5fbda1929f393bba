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

// Prefill work order.  A K/V "stream" is one batch entry's keys and values of
// one KV head; the work tiles of a query tile and stream are its query heads
// (or head pairs).  Work tiles are numbered in bands of `band` query tiles,
// the band of the last (heaviest causal) query tiles first; inside a band,
// stream by stream; inside a stream, query tile descending, then the heads.
// The host sets band so that one stream's share of a band holds about as many
// work tiles as the persistent grid has CTAs: each round of the grid then
// reads ONE stream, and CTAs that drift a round apart read at most a few, so
// the K/V tiles they stream stay in L2 instead of the whole K/V of every
// stream being live at once.  Consecutive bands are each lighter than the
// last, and within a band every stream repeats the same lengths, so the
// snake dealing below still balances the CTAs' totals.
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
    int32_t band;                 // query tiles per band of the work order (>= 1)
};

// K/V bytes (all streams) up to which the whole K/V stays in L2 anyway; then
// the band is one query tile, which is the plain heaviest-first order (all
// streams' work tiles of the last query tile, then of the one before, ...).
constexpr int64_t kPrefillBandMinKVBytes = (int64_t)32 << 20;

// Streams one round of the grid covers (a build-time tuning constant): one
// keeps the fewest K/V bytes live, more spread the CTAs that read the same
// tile at the same moment over more of L2.
#ifndef YOCO_BAND_STREAMS
#define YOCO_BAND_STREAMS 1
#endif
constexpr int kPrefillBandStreams = YOCO_BAND_STREAMS;

// Query tiles per band for a grid of `grid` CTAs, `per` work tiles per (query
// tile, stream), kv_bytes of K and V over all streams and the attention
// window.  A sliding window needs no bands: its work tiles read only the
// window's few KV tiles, which neighbouring query tiles share, so each tile
// comes from DRAM about once in any order, and one stream per round would
// only crowd all CTAs onto the same few tiles.
YOCO_HD int32_t prefill_band(int grid, int per, int64_t kv_bytes, int32_t window) {
    if (window > 0 || kv_bytes <= kPrefillBandMinKVBytes) return 1;
    const int b = per > 0 ? grid / (per * kPrefillBandStreams) : 1;
    return b > 0 ? b : 1;
}

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

// Work tile w of the banded order when each (query tile, stream) has `per`
// work tiles of `heads` consecutive query heads.
YOCO_HD PrefillWork prefill_work_banded(const PrefillShape &s, int w, int per, int heads) {
    const int streams = s.B * s.Hkv;
    const int64_t band_works = (int64_t)s.band * streams * per;
    const int j = (int)(w / band_works);
    const int64_t off = w - (int64_t)j * band_works;
    const int nb = (int)min64(s.band, (int64_t)s.n_qtiles - (int64_t)j * s.band);
    const int64_t stream_works = (int64_t)nb * per;
    const int stream = (int)(off / stream_works);
    const int rem = (int)(off - (int64_t)stream * stream_works);
    const int qt = s.n_qtiles - 1 - (j * s.band + rem / per);
    const int b = stream / s.Hkv, g = stream - b * s.Hkv;
    return prefill_work_at(s, qt, g * (s.Hq / s.Hkv) + (rem % per) * heads, b);
}

// One query head per work tile (any group size): n_work = n_qtiles * Hq * B.
YOCO_HD PrefillWork prefill_work(const PrefillShape &s, int w) {
    return prefill_work_banded(s, w, s.Hq / s.Hkv, 1);
}

// Two query heads per work tile, 2hp and 2hp + 1, which share their KV head
// when the group size Hq / Hkv is even: n_work = n_qtiles * (Hq / 2) * B.
// The returned h is the first head of the pair.
YOCO_HD PrefillWork prefill_pair_work(const PrefillShape &s, int w) {
    return prefill_work_banded(s, w, s.Hq / s.Hkv / 2, 2);
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

// A decode sequence's arguments are in range when 1 <= len <= max_len (the
// length the split plan was sized for) and its rows [start, start + len) lie
// inside the cache's rows [0, cache_rows).  A sequence out of range gets no
// units: it reads nothing, its output is 0 and its lse -inf, and the kernels
// report it through the status word.
YOCO_HD bool decode_seq_ok(int64_t start, int64_t len, int64_t max_len, int64_t cache_rows) {
    return len >= 1 && len <= max_len && start >= 0 && start <= cache_rows - len;
}

}  // namespace sched
}  // namespace yoco
