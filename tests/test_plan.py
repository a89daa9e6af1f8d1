"""Host-side checks of the decode work partition, no GPU needed.

The split-K decode reads every (batch, kv head, query-head group) unit's cache in
chunks and writes one partial (running max, sum, weighted values) per slot; the
combine step merges a unit's slots (the attention of a long sequence split into
independent pieces whose softmax partials are merged, as the decode kernels of
Flash-Decoding do).  The planner picks either a uniform grid (nsplit equal token
ranges per unit) or, for equal-length sequences, a stream-K grid (one CTA per SM,
each an equal share of all chunks laid end to end).  These tests take the plan
through the C ABI's host-only tq_decode_plan and replay the kernel's per-CTA and
per-warp index arithmetic in Python: every chunk is read once, every partial slot
of every unit is written exactly once (a partial or an emptied slot), and the
plan's workspace bound holds.
"""
import itertools

import pytest

from kv_cache_vector_14_b200 import tq

SMS = 148            # B200


def units_of(B, Hq, Hkv):
    G = Hq // Hkv
    return B * Hkv * ((G + 7) // 8)


def warps_of(G):
    return 16 if G <= 4 else 8


def replay_streamk(N, nC, nck, nsplit, NW, T, chunk):
    """The stream-K kernel's index arithmetic for every CTA and warp: returns
    reads[u][x] (times chunk x of unit u is folded into a merge) and
    writes[u][s] (times slot s of unit u is written)."""
    U = N // nck
    reads = [[0] * nck for _ in range(U)]
    writes = [[0] * nsplit for _ in range(U)]

    def first_cta(u):
        return ((u * nck + 1) * nC - 1) // N

    def tok(x, u):
        return min((x - u * nck) * chunk, T)

    for c in range(nC):
        lo, hi = c * N // nC, (c + 1) * N // nC
        S = hi - lo
        assert S > 0
        u0, u1 = lo // nck, (hi - 1) // nck
        assert u1 - u0 <= 1                           # at most two units per CTA
        nxt = (u0 + 1) * nck
        groups = [(u0, c - first_cta(u0), nxt <= hi, tok(lo, u0), tok(min(nxt, hi), u0))]
        cut = None
        if u1 != u0:
            cut = nxt
            groups.append((u1, c - first_cta(u1), hi == (u1 + 1) * nck, tok(nxt, u1), tok(hi, u1)))
        for u, slot, end, s0, s1 in groups:
            assert 0 <= slot < nsplit
            assert 0 <= s0 <= s1 <= T
        # per warp: contiguous runs of the CTA's share; at most one crosses into B
        wlo = [lo + w * S // NW for w in range(NW + 1)]
        assert wlo[0] == lo and wlo[NW] == hi
        crossing = [w for w in range(NW) if cut is not None and wlo[w] < cut < wlo[w + 1]]
        assert len(crossing) <= 1
        aEnd = bBeg = NW
        aX = False
        if cut is not None:
            for w in range(NW):
                if wlo[w] >= cut or cut < wlo[w + 1]:
                    aEnd = bBeg = w
                    aX = wlo[w] < cut
                    break
        # what the merge folds into unit A: warps [0, aEnd) whole, and the crossing
        # warp's chunks before the cut (kept aside by that warp); into unit B:
        # warps [bBeg, NW), each from the cut on
        a_chunks = [x for w in range(aEnd) for x in range(wlo[w], wlo[w + 1])]
        if aX:
            a_chunks += list(range(wlo[bBeg], cut))
        b_chunks = [x for w in range(bBeg, NW) for x in range(max(wlo[w], cut), wlo[w + 1])] if cut else []
        for x in a_chunks:
            assert x // nck == u0
            reads[u0][x - u0 * nck] += 1
        for x in b_chunks:
            assert x // nck == u1
            reads[u1][x - u1 * nck] += 1
        for u, slot, end, _, _ in groups:
            writes[u][slot] += 1
            if end:                                   # the unit's last CTA empties the unused slots
                for sp in range(slot + 1, nsplit):
                    writes[u][sp] += 1
    return reads, writes


def check_streamk(plan, B, Hq, Hkv, T):
    U = units_of(B, Hq, Hkv)
    nck, nC, ns, chunk = plan["streamk_chunks"], plan["streamk_ctas"], plan["nsplit"], plan["chunk_tokens"]
    assert nck == -(-T // chunk)
    assert U <= nC <= SMS
    reads, writes = replay_streamk(U * nck, nC, nck, ns, warps_of(Hq // Hkv), T, chunk)
    assert all(r == 1 for row in reads for r in row)
    assert all(w == 1 for row in writes for w in row)
    # the slot count is the most CTAs any unit spans (no slot goes unused by all units)
    span = max(((u * nck + nck) * nC - 1) // (U * nck) - ((u * nck + 1) * nC - 1) // (U * nck) + 1
               for u in range(U))
    assert ns == span


def check_uniform(plan, T):
    ns, st, chunk = plan["nsplit"], plan["split_tokens"], plan["chunk_tokens"]
    assert plan["streamk_ctas"] == 0 and plan["streamk_chunks"] == 0
    assert 1 <= ns <= 2048
    assert st % chunk == 0
    if T > 0:
        assert ns * st >= T                           # the splits cover the sequence
        assert (ns - 1) * st < T                      # and none of them is empty


# Decisions on the benchmark workloads, each the faster grid as measured on B200
# (CUDA events, same data): stream-K for the long-context and append-and-attend
# shapes, the uniform grid for the single-sequence GQA shape.
@pytest.mark.parametrize("d,B,Hq,Hkv,T,streamk", [
    (128, 4, 16, 8, 102400, True),     # long context, 32 units of 3200 chunks
    (256, 16, 32, 8, 8448, True),      # append-and-attend at its longest step
    (128, 1, 32, 8, 40960, False),     # one sequence, 8 units: 18 splits x 8 fill the SMs
])
def test_plan_decisions(libtq, d, B, Hq, Hkv, T, streamk):
    p = tq.tq_decode_plan(SMS, d, B, Hq, Hkv, T)
    if streamk:
        assert p["streamk_ctas"] == SMS
        check_streamk(p, B, Hq, Hkv, T)
    else:
        check_uniform(p, T)


def test_long_context_plan_exact(libtq):
    p = tq.tq_decode_plan(SMS, 128, 4, 16, 8, 102400)
    assert p == {"nsplit": 6, "split_tokens": 11392, "streamk_ctas": 148, "streamk_chunks": 3200,
                 "chunk_tokens": 32}
    # 102400 chunks over 148 CTAs: a unit of 3200 chunks spans at most 6 CTAs
    assert tq.tq_decode_plan(SMS, 256, 16, 32, 8, 8448)["chunk_tokens"] == 16


SHAPES = list(itertools.product([64, 128, 256], [1, 2, 5, 16], [(8, 8), (16, 8), (32, 8), (32, 4), (64, 4)],
                                [1, 17, 31, 32, 33, 1000, 8448, 40960]))


@pytest.mark.parametrize("d,B,hh,T", SHAPES)
def test_partition_invariants(libtq, d, B, hh, T):
    Hq, Hkv = hh
    p = tq.tq_decode_plan(SMS, d, B, Hq, Hkv, T)
    if p["streamk_ctas"]:
        check_streamk(p, B, Hq, Hkv, T)
    else:
        check_uniform(p, T)
    # ragged lengths never take the stream-K grid, and keep a covering uniform grid
    q = tq.tq_decode_plan(SMS, d, B, Hq, Hkv, T, equal_len=False)
    check_uniform(q, T)


@pytest.mark.parametrize("nC,U,nck", [(148, 32, 3200), (148, 128, 528), (148, 148, 7), (147, 147, 1), (148, 74, 3),
                                      (148, 37, 4), (132, 64, 65), (148, 1, 148), (7, 3, 5)])
@pytest.mark.parametrize("NW", [8, 16])
def test_streamk_replay_any_split(nC, U, nck, NW):
    # the kernel's arithmetic on grids the planner can hand it (every CTA has at
    # least one chunk and touches at most two units), including shares shorter
    # than the warp count and units shorter than a share
    N = U * nck
    ns = max(((u * nck + nck) * nC - 1) // N - ((u * nck + 1) * nC - 1) // N + 1 for u in range(U))
    T = nck * 32 - 5
    reads, writes = replay_streamk(N, nC, nck, ns, NW, T, 32)
    assert all(r == 1 for row in reads for r in row)
    assert all(w == 1 for row in writes for w in row)


def test_degenerate_and_invalid(libtq):
    p = tq.tq_decode_plan(SMS, 128, 0, 16, 8, 1024)       # empty batch
    assert p["streamk_ctas"] == 0 and p["nsplit"] >= 1
    p = tq.tq_decode_plan(SMS, 128, 4, 16, 8, 0)          # empty cache
    assert p["streamk_ctas"] == 0 and p["nsplit"] >= 1
    p = tq.tq_decode_plan(1, 128, 4, 16, 8, 102400)       # one SM: one unit per CTA at most
    assert p["streamk_ctas"] == 0
    check_uniform(p, 102400)
    for bad in [(SMS, 96, 1, 8, 8, 10), (SMS, 128, 1, 12, 8, 10), (SMS, 128, 1, 8, 8, -1), (0, 128, 1, 8, 8, 10),
                (SMS, 128, -1, 8, 8, 10)]:
        with pytest.raises(tq.TQError):
            tq.tq_decode_plan(*bad)
