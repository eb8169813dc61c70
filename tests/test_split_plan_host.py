"""The chunk-range plan of the elu d=64 split forward, checked on the host.

The library cuts the T = B*H*ceil(N/128) chunks, in (head, chunk) order, into
G contiguous ranges (G = min(148, T, 16*B*H)); range k starts at chunk
floor(T*k/G).  The workspace size the library reports encodes T and G, which
ties the plan below to the library's own host code.  The device side of the
plan is mirrored here to check its invariants for many shapes:
  - every snapshot the output launch reads was written by the state launch;
  - every head's final state is written exactly once;
  - the carry of a range that starts inside a head sums exactly the chunks of
    that head before it, from the aggregates the earlier ranges wrote.
"""
import pytest

import causal_kernelized_sequence_b200 as la

C, NSM, MAX_PER_HEAD = 128, 148, 16
TILE, SNAP, AGG = 128 * 64 * 2, 80 // 16 * 64 * 32, 64 * 80


def plan(B, H, N):
    nc = (N + C - 1) // C
    T = B * H * nc
    G = min(T, NSM, B * H * MAX_PER_HEAD)
    return T, G, nc


def begin(T, G, k):
    return (T * k) // G


SHAPES = [(B, H, N) for B, H in [(1, 1), (1, 2), (2, 3), (4, 8), (1, 37), (8, 16), (1, 300), (64, 64)]
          for N in [1, 17, 64, 128, 129, 256, 300, 700, 1000, 4096, 4097]]


@pytest.mark.parametrize("B,H,N", SHAPES)
def test_workspace_encodes_the_plan(B, H, N):
    la.load_library()
    T, G, _ = plan(B, H, N)
    assert la.la_forward_workspace_bytes(B, H, N, 64, 64, la.LA_FMAP_ELU1, la.LA_BF16) == \
        T * (TILE + SNAP) + G * 2 * AGG * 4


@pytest.mark.parametrize("B,H,N", SHAPES)
def test_range_bookkeeping(B, H, N):
    T, G, nc = plan(B, H, N)
    snaps, finals, agg_last, agg_first = set(), {}, {}, {}
    covered_by = {}   # range -> chunks summed into its last-segment aggregate
    for kb in range(G):
        tb, nit = begin(T, G, kb), begin(T, G, kb + 1) - begin(T, G, kb)
        assert nit >= 1
        c0 = tb % nc
        carry_in = c0 != 0
        first_len = min(nit, nc - c0)
        seg_start = tb
        for it in range(nit):
            t = tb + it
            c = t % nc
            if c == 0:
                seg_start = t
            head_end, last = c == nc - 1, it == nit - 1
            if not head_end and not last:
                snaps.add(t + 1)                 # the local state before chunk t+1
            elif head_end and carry_in and it < first_len:
                agg_first[kb] = set(range(tb, t + 1))
            elif head_end:
                finals[t // nc] = finals.get(t // nc, 0) + 1
            else:
                agg_last[kb] = True
                covered_by[kb] = set(range(seg_start, t + 1))
    # the output launch's reads
    for kb in range(G):
        tb, nit = begin(T, G, kb), begin(T, G, kb + 1) - begin(T, G, kb)
        for it in range(nit):
            if it > 0 and (tb + it) % nc != 0:
                assert tb + it in snaps, (kb, it)
        c0 = tb % nc
        if c0:
            head0 = tb - c0
            jlo = kb - 1
            while jlo > 0 and begin(T, G, jlo) > head0:
                jlo -= 1
            got = set()
            for jb in range(jlo, kb):
                assert jb in covered_by, (kb, jb)
                assert not (got & covered_by[jb])
                got |= covered_by[jb]
            assert got == set(range(head0, tb)), (kb, sorted(got))
            # a head that ends inside this range gets its final state from the carry
            first_len = min(begin(T, G, kb + 1) - tb, nc - c0)
            if first_len < begin(T, G, kb + 1) - tb or c0 + first_len == nc:
                finals[tb // nc] = finals.get(tb // nc, 0) + 1
    assert finals == {h: 1 for h in range(B * H)}


# ------------------------------------------------------------------ segments
# The one-launch forward (elu d=128, Taylor) and the tensor-core backward split
# a sequence into P segments of cps chunks so that B*H*P blocks roughly fill
# the 148 SMs; segment s covers chunks [s*cps, min(nc, (s+1)*cps)).

def segments(B, H, N):
    nc = (N + C - 1) // C
    p = max(1, NSM // (B * H))
    p = min(p, nc)
    cps = (nc + p - 1) // p
    return (nc + cps - 1) // cps, cps, nc


SEG_SHAPES = [(B, H, N) for B, H in [(1, 1), (1, 2), (2, 3), (2, 16), (8, 16), (1, 200)]
              for N in [1, 100, 128, 129, 1000, 4097, 16384, 65536]]


@pytest.mark.parametrize("B,H,N", SEG_SHAPES)
def test_segment_plan(B, H, N):
    la.load_library()
    P, cps, nc = segments(B, H, N)
    # every chunk in exactly one segment, none empty
    chunks = [c for s in range(P) for c in range(s * cps, min(nc, (s + 1) * cps))]
    assert chunks == list(range(nc)) and all(s * cps < nc for s in range(P))
    assert B * H * P <= max(NSM, B * H)
    # the workspaces the library asks for hold one increment per (head, segment)
    inc128 = 128 * 144 * 4                   # elu d=128: F x (d_v + 16) fp32
    incT = 160 * 80 * 4                      # Taylor: 160 packed features x (64 + 16)
    assert la.la_forward_workspace_bytes(B, H, N, 128, 128, la.LA_FMAP_ELU1, la.LA_BF16) == \
        (B * H * P * inc128 if P > 1 else 0)
    assert la.la_forward_workspace_bytes(B, H, N, 16, 64, la.LA_FMAP_TAYLOR2, la.LA_BF16) == \
        (B * H * P * incT if P > 1 else 0)
    # backward: den_i, dden_i per token, plus S and R increments when split
    assert la.la_backward_workspace_bytes(B, H, N, 128, 128, la.LA_FMAP_ELU1, la.LA_BF16) == \
        B * H * N * 2 * 4 + (2 * B * H * P * 128 * 144 * 4 if P > 1 else 0)
