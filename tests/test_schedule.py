"""The kernels' work plans (yoco_debug_tile_schedule), checked on the host
against the oracle's visibility rule, bit-exact: the prefill visits exactly
the KV tiles that hold a visible (query, key) pair, masks exactly the tiles
that also hold an invisible pair or a key past the end, and covers every
work tile once; the decode units partition every sequence.  No GPU needed:
the plan is computed by the same schedule functions the kernels run."""
import numpy as np
import pytest
import torch

import oracle
import shared_kv_decoder_b200 as yoco

BM = BN = 128

PREFILL_CASES = [
    # B, Hq, Hkv, Tq, Tkv, q_pos0, window, n_cta
    (1, 4, 2, 300, 300, 0, 0, 5),        # causal, ragged last query tile
    (2, 8, 2, 256, 256, 0, 0, 148),      # more CTAs than work tiles
    (1, 2, 1, 200, 777, 577, 0, 3),      # chunk offset, tail KV tile
    (1, 4, 4, 640, 640, 0, 100, 7),      # window smaller than a tile
    (3, 2, 2, 513, 513, 0, 300, 4),      # window spanning tile edges, B > 1
    (1, 2, 1, 129, 1000, 871, 256, 2),   # chunked window, tile-boundary offsets
    (1, 1, 1, 1, 1, 0, 0, 1),            # a single query and key
    (1, 2, 1, 384, 384, 0, 128, 3),      # window equal to the tile size
    (2, 8, 8, 300, 300, 0, 0, 5),        # group size 1: one head per work tile
    (1, 16, 2, 520, 520, 0, 200, 6),     # group size 8
]


def _prefill(B, Hq, Hkv, Tq, Tkv, q_pos0, W, n_cta):
    return yoco.debug_tile_schedule(yoco.SCHEDULE_PREFILL, Hq, Hkv, 64, B=B, Tq=Tq, Tkv=Tkv,
                                    q_pos0=q_pos0, window=W, n_cta=n_cta)


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tkv,q_pos0,W,n_cta", PREFILL_CASES)
def test_prefill_plan_matches_visibility(B, Hq, Hkv, Tq, Tkv, q_pos0, W, n_cta):
    rec = _prefill(B, Hq, Hkv, Tq, Tkv, q_pos0, W, n_cta)
    vis = oracle.visibility(Tq, Tkv, q_pos0, W)
    n_qt = -(-Tq // BM)
    n_kt = -(-Tkv // BN)
    # expected per query tile: KV tiles with a visible pair, and which need a mask
    want = {}
    for qt in range(n_qt):
        rows = vis[qt * BM:min((qt + 1) * BM, Tq)]
        tiles = {}
        for kt in range(n_kt):
            blk = rows[:, kt * BN:(kt + 1) * BN]
            if blk.any():
                # masked: an invisible pair among real rows, or keys past Tkv
                tiles[kt] = int((not blk.all()) or (kt + 1) * BN > Tkv)
        want[qt] = tiles
    seen = {}
    for cta, b, h, qt, kt, masked in rec.tolist():
        assert 0 <= cta < n_cta and 0 <= b < B and 0 <= h < Hq
        seen.setdefault((b, h, qt), []).append((cta, kt, masked))
    assert set(seen) == {(b, h, qt) for b in range(B) for h in range(Hq) for qt in range(n_qt)}
    for (b, h, qt), visits in seen.items():
        assert len({c for c, _, _ in visits}) == 1, "a work tile is split over CTAs"
        kts = [kt for _, kt, _ in visits]
        assert kts == sorted(want[qt]), (b, h, qt)      # exactly the visible tiles, in order
        assert {kt: m for _, kt, m in visits} == want[qt], (b, h, qt)


@pytest.mark.parametrize("B,Hq,Hkv,Tq,Tkv,q_pos0,W,n_cta", PREFILL_CASES)
def test_prefill_plan_order_and_balance(B, Hq, Hkv, Tq, Tkv, q_pos0, W, n_cta):
    rec = _prefill(B, Hq, Hkv, Tq, Tkv, q_pos0, W, n_cta)
    heads = 2 if (Hq // Hkv) % 2 == 0 else 1          # heads per work tile
    n_qt = -(-Tq // BM)
    # work tiles: (cta, b, head pair, query tile); the heads of a pair visit
    # the same KV tiles in lockstep, and each work tile's visits are one run
    runs = []
    for cta, b, h, qt, kt, _ in rec.tolist():
        key = (cta, b, h // heads, qt)
        if not runs or runs[-1][0] != key:
            runs.append([key, []])
        runs[-1][1].append((h, kt))
    assert len(runs) == len({k for k, _ in runs})
    for (cta, b, hp, qt), visits in runs:
        per_head = [[kt for h, kt in visits if h == heads * hp + e] for e in range(heads)]
        assert all(v == per_head[0] for v in per_head)
        if heads == 2:
            assert [h for h, _ in visits] == [2 * hp, 2 * hp + 1] * len(per_head[0])
    # each CTA starts with a heaviest work tile (the last query tile), and the
    # per-CTA totals stay within one work tile's worth of each other
    firsts = {}
    for (cta, _, _, qt), _ in runs:
        firsts.setdefault(cta, qt)
    assert all(qt == n_qt - 1 for qt in firsts.values()) or len(firsts) > B * Hq // heads
    tot = np.zeros(max(firsts) + 1)
    for (cta, _, _, _), v in runs:
        tot[cta] += len(v)
    heaviest = max(len(v) for _, v in runs)
    if len(runs) >= 2 * len(tot):
        assert tot.max() - tot.min() <= heaviest


@pytest.mark.parametrize("lens,max_len,Hq,Hkv,D,n_cta", [
    ([1000, 17, 3000], 3000, 32, 8, 128, 4),
    ([1, 2, 3, 130, 4097], 5000, 8, 1, 64, 148),
    ([65536, 70001, 131072, 100000], 131072, 32, 8, 128, 148),
    ([0, 5, 0, 300], 300, 4, 2, 64, 3),
    ([100, 5000, 7, 1000], 1000, 32, 8, 128, 16),   # 5000 > max_len: out of range, no units
])
def test_decode_plan_partitions_sequences(lens, max_len, Hq, Hkv, D, n_cta):
    starts = np.cumsum([0] + [l + 7 for l in lens[:-1]])
    rec = yoco.debug_tile_schedule(yoco.SCHEDULE_DECODE, Hq, Hkv, D, B=len(lens), seq_start=starts,
                                   seq_len=lens, max_len=max_len, n_cta=n_cta)
    stage = 128 // Hkv
    covered = {b: [] for b in range(len(lens))}
    per_cta_units = {}
    for cta, b, s, row0, n_tok, n_st in rec.tolist():
        assert 0 <= cta < n_cta
        assert n_tok >= 1 and n_st == -(-n_tok // stage)
        covered[b].append((row0 - starts[b], n_tok, s))
        per_cta_units[cta] = per_cta_units.get(cta, 0) + 1
    for b, L in enumerate(lens):
        segs = sorted(covered[b])
        pos = 0
        for k, (off, n, s) in enumerate(segs):
            assert off == pos and s == k         # consecutive, no gap or overlap
            pos += n
        # the whole sequence, nothing past it; none of a sequence out of range
        assert pos == (L if 1 <= L <= max_len else 0)
        if len(segs) > 1:                        # equal splits, a multiple of the stage
            split = segs[0][1]
            assert split % stage == 0 and all(n == split for _, n, _ in segs[:-1])
    # the compact unit list is dealt round-robin over the CTAs
    if per_cta_units:
        assert max(per_cta_units.values()) - min(per_cta_units.values()) <= 1


@pytest.mark.parametrize("lens,max_len,max_units", [
    ([1 << 20], 1 << 20, 296),                       # one 1M-token sequence: two units an SM at most
    ([32768], 32768, 296),                           # one 32K sequence: ~2 MB units
    ([65536 + 4096 * i for i in range(16)], 131072, 1776),   # 16 long sequences: the call's maximum
])
def test_decode_plan_unit_counts(lens, max_len, max_units):
    # a sequence gets at most 296 units (its merge folds them in one CTA per
    # query head) and a call at most 12 per SM; the 1M-token sequence's split
    # is set by that cap (14 MB units), the others' by the call's unit count
    starts = np.cumsum([0] + lens[:-1])
    rec = yoco.debug_tile_schedule(yoco.SCHEDULE_DECODE, 32, 8, 128, B=len(lens), seq_start=starts,
                                   seq_len=lens, max_len=max_len, n_cta=148)
    per_seq = np.bincount(rec[:, 1], minlength=len(lens))
    assert per_seq.max() <= 296
    assert len(rec) <= max_units
    tok_bytes = 2 * 8 * 128 * 2
    split = int(rec[0, 4])
    if len(lens) == 1 and lens[0] == (1 << 20):
        assert per_seq[0] == 296 or per_seq[0] == -(-lens[0] // split)
        assert split * tok_bytes > (2 << 20)          # the cap, not the 2 MB target, sets the split
    else:
        assert split * tok_bytes < 5 * (1 << 20)


def test_schedule_rejects_bad_arguments():
    with pytest.raises(yoco.YocoError):
        _prefill(1, 4, 2, 100, 50, 0, 0, 4)      # q_pos0 + Tq > Tkv
    with pytest.raises(yoco.YocoError):
        yoco.debug_tile_schedule(7, 4, 2, 64)
    with pytest.raises(yoco.YocoError):
        yoco.debug_tile_schedule(yoco.SCHEDULE_PREFILL, 3, 2, 64, Tq=1, Tkv=1)   # Hq % Hkv


def test_prefill_banded_order_reads_one_stream_per_round():
    # K/V beyond 32 MB (here 67 MB: T=16384, 8 KV heads, D=128, bf16): the work
    # order goes in bands, so that each round of the 148-CTA grid streams the
    # K/V of ONE KV head (two head pairs x 74 query tiles) and the tiles the
    # CTAs read stay in L2.  Checked: every work tile once, on one CTA, over
    # exactly KV tiles 0..qt (causal); each round's CTAs on one KV head; the
    # bands heaviest first; per-CTA totals within one work tile.
    B, Hq, Hkv, T, n_cta = 1, 32, 8, 16384, 148
    rec = yoco.debug_tile_schedule(yoco.SCHEDULE_PREFILL, Hq, Hkv, 128, B=B, Tq=T, Tkv=T, n_cta=n_cta)
    n_qt = T // BM
    works = {}
    order = []
    for cta, b, h, qt, kt, masked in rec.tolist():
        key = (b, h // 2, qt)
        if key not in works:
            works[key] = [cta, []]
            order.append((cta, key))
        assert works[key][0] == cta
        works[key][1].append((h, kt, masked))
    assert len(works) == n_qt * Hq // 2 * B
    for (b, hp, qt), (cta, visits) in works.items():
        assert [kt for h, kt, _ in visits if h == 2 * hp] == list(range(qt + 1))
        assert all(m == (kt == qt) for _, kt, m in visits)     # only the diagonal tile is masked
    # round r of CTA c is its r-th work tile; each round is one KV head
    per_cta = {}
    for cta, key in order:
        per_cta.setdefault(cta, []).append(key)
    G = Hq // Hkv
    n_rounds = max(len(v) for v in per_cta.values())
    for r in range(n_rounds):
        heads = {(2 * k[1]) // G for v in per_cta.values() if r < len(v) for k in [v[r]]}
        qts = [v[r][2] for v in per_cta.values() if r < len(v)]
        assert len(heads) <= 3, (r, heads)    # the last, shorter band mixes streams
        if r == 0:
            assert len(heads) == 1 and min(qts) >= n_qt - 74      # the heaviest band first
    tot = {c: sum(k[2] + 1 for k in v) for c, v in per_cta.items()}
    assert max(tot.values()) - min(tot.values()) <= n_qt
