"""The feature permutation of the warp-level GEMVs (NVFP4 and bf16 decode),
checked on the CPU.

An m16n8k16 MMA sums its 16 k slots in any order, so the kernels feed the
weights and the activations through one common permutation of each block of
BK features (BK = 128, or a 64-feature tail): in k-tile kt, the slot
kappa = 8h + 2tq + p (tq = lane % 4; h, p in {0, 1}) holds feature
(BK/4) tq + 4 kt + 2h + p.  The GEMV is correct only if that map is a
bijection of the block (every product summed exactly once), and it is fast
only if thread tq's features form one contiguous run of BK/4 (one 16-byte
code load, four-bf16 activation loads).
"""
import pytest


def feature(BK, kt, tq, h, p):
    return (BK // 4) * tq + 4 * kt + 2 * h + p


@pytest.mark.parametrize("BK", [128, 64])
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


@pytest.mark.parametrize("BK", [128, 64])
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
