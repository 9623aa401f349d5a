"""The feature permutation of the warp-level GEMVs (NVFP4 and bf16 decode),
checked on the CPU.

An m16n8k16 MMA sums its 16 k slots in any order, so the kernels feed the
weights and the activations through one common permutation of each block of
BK features: in k-tile kt, the slot kappa = 8h + 2tq + p (tq = lane % 4;
h, p in {0, 1}) holds feature (BK/4) tq + 4 kt + 2h + p.  The NVFP4 GEMV uses
BK = 128 (or a 64-feature tail); the staged bf16 GEMV uses units of BK = 32,
one 16-byte word of 8 features per thread and row.  The GEMV is correct only
if that map is a bijection of the block (every product summed exactly once),
and it is fast only if thread tq's features form one contiguous run of BK/4
(one 16-byte load of codes or of bf16 weights, contiguous activations).
"""
import pytest


def feature(BK, kt, tq, h, p):
    return (BK // 4) * tq + 4 * kt + 2 * h + p


@pytest.mark.parametrize("BK", [128, 64, 32])
def test_permutation_is_a_bijection_with_contiguous_runs(BK):
    seen = {}
    for kt in range(BK // 16):
        for tq in range(4):
            for h in range(2):
                for p in range(2):
                    f = feature(BK, kt, tq, h, p)
                    kappa = 8 * h + 2 * tq + p
                    assert 0 <= kappa < 16
                    assert f not in seen, (f, seen.get(f))
                    seen[f] = (kt, kappa)
    assert sorted(seen) == list(range(BK))
    for tq in range(4):
        run = sorted(feature(BK, kt, tq, h, p) for kt in range(BK // 16)
                     for h in range(2) for p in range(2))
        assert run == list(range((BK // 4) * tq, (BK // 4) * (tq + 1)))


@pytest.mark.parametrize("BK", [128, 64, 32])
def test_a_and_b_fragments_meet_on_the_same_features(BK):
    """In m16n8k16 a thread holds A[row][2tq + p] and A[row][2tq + 8 + p]
    (h = 0, 1) and B[2tq + p][col], B[2tq + 8 + p][col]: the slot kappa of both
    operands is 8h + 2tq + p, so weights and activations of one slot are the
    same feature exactly when both use the map above.  Each slot of each
    k-tile is owned by one thread (tq) of the quad."""
    for kt in range(BK // 16):
        owners = {}
        for tq in range(4):
            for h in range(2):
                for p in range(2):
                    owners.setdefault(8 * h + 2 * tq + p, set()).add(tq)
        assert sorted(owners) == list(range(16))
        assert all(len(v) == 1 for v in owners.values())


UNIT = 32          # features per unit of the staged bf16 GEMV
WARPS = 8
CH = 11            # units per chunk


def staged_chunks(K):
    """(warp, first unit, units) of every chunk the staged GEMV's warps copy:
    warp w owns units [w U / 8, (w + 1) U / 8) of U = K / 32, in chunks of up
    to CH units."""
    U = K // UNIT
    out = []
    for w in range(WARPS):
        lo, hi = w * U // WARPS, (w + 1) * U // WARPS
        c = 0
        while lo + c * CH < hi:
            ua = lo + c * CH
            out.append((w, ua, min(CH, hi - ua)))
            c += 1
    return out


@pytest.mark.parametrize("K", [32, 64, 224, 1024, 2688, 3712, 4096])
def test_staged_chunks_cover_k_once(K):
    """Every unit of K is copied by exactly one chunk of one warp, and a copy is a
    multiple of 16 bytes that starts on a 16-byte boundary (rows are K * 2 bytes
    apart, K a multiple of 32)."""
    seen = [0] * (K // UNIT)
    for w, ua, n in staged_chunks(K):
        assert 1 <= n <= CH
        assert (ua * UNIT * 2) % 16 == 0 and (n * UNIT * 2) % 16 == 0
        for u in range(ua, ua + n):
            seen[u] += 1
    assert seen == [1] * (K // UNIT)


def test_staged_chunk_counts_of_the_shared_expert():
    """K = 2688 (the up projection) takes one chunk per warp: a single round trip;
    K = 3712 (the down projection) takes two."""
    per_warp = lambda K: max(sum(1 for w2, _, _ in staged_chunks(K) if w2 == w)
                             for w in range(WARPS))
    assert per_warp(2688) == 1
    assert per_warp(3712) == 2
