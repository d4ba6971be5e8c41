"""The list-merging algorithms the LM-head kernels use, modelled step by step
in Python and checked against a full sort of every candidate (no GPU).

- threshold-and-rank merge (merge kernel): tau = max(16th largest of the
  records' leading entries, largest 16th entry of any record) is a lower
  bound on the row's 16th best value, so gathering the entries >= tau and
  ranking them under (value desc, index asc) yields the exact top-16;
- bitonic merge of two sorted 16-lists (the epilogue's half merge): the
  elementwise better of a[k] and b[15-k], then four half-cleaner stages;
- the 16-element bitonic sorting network that fills an empty list;
- the weight-streaming tile plan: every tile width a CTA runs is one of the
  at most four widths the host builds tensor maps for, including the narrow
  last tile of a long range.
Ties, duplicate values, records with empty slots and few records are all
exercised; the GPU tests check the kernels themselves."""
import numpy as np
import pytest

K = 16
EMPTY_I = 0x7FFFFFFF


def _key(v, i):
    return (-v, i)                                  # smaller key = better entry


def _better(a, b):
    return _key(*a) < _key(*b)


def _exact(records):
    allv = [(v, i) for rec in records for (v, i) in rec if i != EMPTY_I]
    allv.sort(key=lambda e: _key(*e))
    return allv[:K]


def _merge_threshold_rank(records):
    P = len(records)
    J = 1 if P >= K else -(-K // P)
    heads = [rec[j][0] for rec in records for j in range(J)]
    th = -np.inf
    for h in heads:
        if sum(1 for x in heads if x >= h) >= K:
            th = max(th, h)
    tau = max(th, max(rec[K - 1][0] for rec in records))
    gathered = [(v, i) for rec in records for (v, i) in rec if v >= tau and i != EMPTY_I]
    out = [None] * K
    for e in gathered:
        rank = sum(1 for f in gathered if _better(f, e))
        if rank < K:
            out[rank] = e
    return [e for e in out if e is not None], len(gathered)


def _random_records(rng, P, n_valid_max, tie_levels):
    """P sorted records of 16 entries over distinct indices; values drawn
    from a few levels (many ties) or continuous; some records part-empty."""
    idx = rng.permutation(P * K * 4)[: P * K]
    records = []
    for r in range(P):
        n_valid = rng.integers(0, n_valid_max + 1)
        vals = rng.choice(tie_levels, size=K) if tie_levels is not None else rng.standard_normal(K)
        ents = [(float(vals[k]), int(idx[r * K + k])) for k in range(K)]
        ents = sorted(ents[:n_valid], key=lambda e: _key(*e)) + [(-np.inf, EMPTY_I)] * (K - n_valid)
        records.append(ents)
    return records


@pytest.mark.parametrize("P", [1, 2, 3, 5, 15, 16, 17, 37, 148])
@pytest.mark.parametrize("ties", [False, True])
def test_threshold_rank_merge_is_exact(P, ties):
    rng = np.random.default_rng(P * 2 + ties)
    for trial in range(20):
        levels = np.array([0.0, 0.5, 1.0, 1.5]) if ties else None
        records = _random_records(rng, P, K, levels)
        if sum(i != EMPTY_I for rec in records for _, i in rec) < K:
            continue
        got, n = _merge_threshold_rank(records)
        assert got == _exact(records)


def test_threshold_gathers_few_entries_on_continuous_values():
    """With continuous values and 148 full records the gather stays small."""
    rng = np.random.default_rng(5)
    records = _random_records(rng, 148, K, None)
    records = [sorted([(float(v), i) for v, i in zip(rng.standard_normal(K), rng.permutation(10**6)[:K])],
                      key=lambda e: _key(*e)) for _ in range(148)]
    got, n = _merge_threshold_rank(records)
    assert got == _exact(records)
    assert n <= 64


def _bitonic_merge(a, b):
    """Top-16 of two sorted lists: elementwise better of a[k], b[15-k], then
    half-cleaners with strides 8, 4, 2, 1."""
    c = [b[K - 1 - k] if _better(b[K - 1 - k], a[k]) else a[k] for k in range(K)]
    j = K // 2
    while j >= 1:
        for k in range(K):
            if k & j == 0 and _better(c[k + j], c[k]):
                c[k], c[k + j] = c[k + j], c[k]
        j //= 2
    return c


def _sort16(x):
    """The 16-element bitonic sorting network (descending by the entry order)."""
    c = list(x)
    size = 2
    while size <= K:
        stride = size // 2
        while stride > 0:
            for k in range(K):
                p = k ^ stride
                if p > k:
                    desc = (k & size) == 0
                    if (desc and _better(c[p], c[k])) or (not desc and _better(c[k], c[p])):
                        c[k], c[p] = c[p], c[k]
            stride //= 2
        size *= 2
    return c


@pytest.mark.parametrize("seed", range(30))
def test_bitonic_merge_and_sort_network(seed):
    rng = np.random.default_rng(seed)
    levels = np.array([0.0, 1.0, 2.0]) if seed % 2 else None
    vals = rng.choice(levels, 32) if levels is not None else rng.standard_normal(32)
    ents = [(float(v), int(i)) for v, i in zip(vals, rng.permutation(1000)[:32])]
    a = sorted(ents[:K], key=lambda e: _key(*e))
    b = sorted(ents[K:], key=lambda e: _key(*e))
    assert _bitonic_merge(a, b) == sorted(ents, key=lambda e: _key(*e))[:K]
    assert _sort16(ents[:K]) == a


TAIL = 4   # 16-row units of the narrow last tile of a long range


def _split(n, tail_units):
    """stream_split: (main tiles, units per main tile, tail units)."""
    tail = tail_units if tail_units > 0 and n >= tail_units + 16 else 0
    m = n - tail
    nt = -(-m // 16)
    wu = -(-m // nt) if nt else 0
    return nt, wu, tail


def _stream_tiles(units, G, c, tail_units):
    """Widths (in rows) of CTA c's tiles: its balanced 16-row-unit range cut
    into the fewest equal tiles of at most 256 rows, then the narrow tail."""
    u0, u1 = c * units // G, (c + 1) * units // G
    nt, wu, tail = _split(u1 - u0, tail_units)
    main_end = u1 - tail
    out = []
    for k in range(nt):
        t0 = u0 + k * wu
        if t0 >= main_end:
            break
        out.append((min(t0 + wu, main_end) - t0) * 16)
    if tail:
        out.append(tail * 16)
    return out


def _stream_widths(units, G, tail_units):
    """The widths the host enumerates (one tensor map each, at most four);
    None when more than four would be needed."""
    ws = []
    u_lo = units // G
    for u in (u_lo, u_lo + 1):
        if u < 1:
            continue
        nt, wu, tail = _split(u, tail_units)
        for w in (16 * wu, 16 * (u - tail - (nt - 1) * wu), 16 * tail):
            if w > 0 and w not in ws:
                if len(ws) == 4:
                    return None
                ws.append(w)
    return ws


@pytest.mark.parametrize("V", [16, 17, 100, 4096, 8193, 20000, 129280, 151936, 151937, 256000, 500000])
def test_stream_tile_widths_are_enumerated(V):
    """Every tile a CTA runs has one of the (at most four) enumerated widths,
    the tiles of all CTAs cover the 16-row units exactly once, and none is
    wider than 256 rows."""
    units = -(-V // 16)
    for sms in (148, 132, 8):
        G = min(units, sms)
        tail = TAIL
        ws = _stream_widths(units, G, tail)
        if ws is None:                 # the host drops the tail rather than need a fifth map
            tail = 0
            ws = _stream_widths(units, G, tail)
        assert ws is not None and len(ws) <= 4
        covered = 0
        for c in range(G):
            tiles = _stream_tiles(units, G, c, tail)
            assert all(w in ws and 0 < w <= 256 for w in tiles)
            covered += sum(tiles)
            if tail and (c + 1) * units // G - c * units // G >= tail + 16:
                assert tiles[-1] == 16 * tail  # long ranges end with the narrow tile
        assert covered == units * 16


def test_stream_tail_at_the_weight_streaming_workloads():
    """qwen3-4b-bs1 and 27b-class (V = 151,936 over 148 CTAs) keep the narrow
    64-row last tile on every CTA."""
    units = 151936 // 16
    assert _stream_widths(units, 148, TAIL) is not None
    for c in range(148):
        assert _stream_tiles(units, 148, c, TAIL)[-1] == 64
