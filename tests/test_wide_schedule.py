"""CPU model of the tensor-bound LM head's wide-tile schedule (no GPU): the
host's choice between RUNS and BLOCKS(R) and each CTA pair's walk over wide
steps (two 256-row vocabulary tiles, or one at the end of a job), written
out as in lmhead_topk.cu.  Checked at the workloads' sizes with 74 pair
units (148 SMs):
- every (token tile, vocabulary tile) is computed exactly once;
- a job's steps are consecutive, start with `first`, end with `last`, and
  keep one record slot below P, and no (row, slot) record is written twice;
- BLOCKS keeps the vocabulary window its concurrent jobs read within the
  bound the planner uses, and the busiest unit stays near the average."""
import math

import pytest

TILE_N = 256
RESTART = 0.15
W_WINDOW = 48.0 * 1024 * 1024


def plan(M, V, d, units):
    m_tiles = (M + 255) // 256
    v_tiles = (V + TILE_N - 1) // TILE_N
    best, sched = 1e30, None
    nr = min(units // m_tiles, v_tiles)
    if nr >= 1:
        t_run = (v_tiles + nr - 1) // nr
        best = t_run * (1.0 + RESTART / t_run)
        sched = dict(kind="RUNS", nr=nr, P=nr, used=nr * m_tiles)
    tile_bytes = TILE_N * d * 2.0
    R = 2
    while R <= 64:
        nvb = (v_tiles + R - 1) // R
        jobs = m_tiles * nvb
        u = min(jobs, units)
        window = (u / m_tiles + 1.0) * R * tile_bytes
        if R > 2 and window > W_WINDOW:
            break
        c = ((jobs + u - 1) // u) * R * (1.0 + RESTART / R)
        if c < best:
            best, sched = c, dict(kind="BLOCKS", R=R, nvb=nvb, P=nvb, used=u, window=window)
        R *= 2
    sched.update(m_tiles=m_tiles, v_tiles=v_tiles)
    return sched


def wide_tile(s, u, units, k):
    """(mt, vt, n_sub, slot, first, last) of step k of unit u, or None."""
    if s["kind"] == "RUNS":
        mt, r = u % s["m_tiles"], u // s["m_tiles"]
        lo, hi = r * s["v_tiles"] // s["nr"], (r + 1) * s["v_tiles"] // s["nr"]
        vt = lo + 2 * k
        if vt >= hi:
            return None
        return mt, vt, min(2, hi - vt), r, k == 0, vt + 2 >= hi
    jobs, job, kk = s["m_tiles"] * s["nvb"], u, k
    while True:
        if job >= jobs:
            return None
        vb = job // s["m_tiles"]
        lo = vb * s["R"]
        hi = min(lo + s["R"], s["v_tiles"])
        nsteps = (hi - lo + 1) // 2
        if kk < nsteps:
            vt = lo + 2 * kk
            return job - vb * s["m_tiles"], vt, min(2, hi - vt), vb, kk == 0, kk == nsteps - 1
        kk -= nsteps
        job += units


SHAPES = [("qwen3-4b-batched", 448, 151936, 2560), ("throughput", 4096, 129280, 4096),
          ("M=129", 129, 3000, 128), ("M=300", 300, 517, 64), ("M=448", 448, 4000, 256), ("M=200", 200, 2600, 192)]


@pytest.mark.parametrize("name,M,V,d", SHAPES)
def test_wide_schedule_covers_every_tile_once(name, M, V, d):
    s = plan(M, V, d, 74)
    units = s["used"]
    seen = {}
    records = set()
    busiest = 0
    for u in range(units):
        k, work, cur = 0, 0, None
        while True:
            t = wide_tile(s, u, units, k)
            if t is None:
                break
            mt, vt, n_sub, slot, first, last = t
            assert 0 <= slot < s["P"]
            assert first == (cur is None)
            cur = (mt, slot) if cur is None else cur
            assert cur == (mt, slot)             # one job: one token tile, one slot
            for j in range(n_sub):
                key = (mt, vt + j)
                assert key not in seen, (key, u, seen.get(key))
                seen[key] = u
            work += n_sub
            if last:
                assert (mt, slot) not in records  # one record per (token tile, slot)
                records.add((mt, slot))
                cur = None
            k += 1
        assert cur is None                        # every job ends with `last`
        busiest = max(busiest, work)
    assert len(seen) == s["m_tiles"] * s["v_tiles"]
    avg = s["m_tiles"] * s["v_tiles"] / 74
    assert busiest <= math.ceil(avg) + s.get("R", 2) + 1
    if s["kind"] == "BLOCKS" and s["R"] > 2:
        assert s["window"] <= W_WINDOW


def test_throughput_uses_short_blocks_and_qwen_batched_runs():
    """The planner's choices at the two tensor-bound workloads: the batched
    4B shape (2 token tiles) runs one vocabulary range per pair; the
    throughput shape (16 token tiles) deals jobs of 4 vocabulary tiles, whose
    concurrent W window (about 40 MB at d = 4096) fits in L2."""
    assert plan(448, 151936, 2560, 74)["kind"] == "RUNS"
    s = plan(4096, 129280, 4096, 74)
    assert s["kind"] == "BLOCKS" and s["R"] == 4 and s["window"] <= W_WINDOW
