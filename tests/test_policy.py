"""The dense-first schedule (Radial Attention, sec. 6: the first 2 DiT blocks and
the first 12 denoising steps keep dense attention) on the host (CPU)."""
from types import SimpleNamespace

import pytest


@pytest.fixture(scope="module")
def ra():
    import __graft_entry__
    __graft_entry__.build()
    import static_sparse_attention_b200 as ra
    return ra


def test_dense_first_policy_follows_the_rule(ra):
    sparse, dense = SimpleNamespace(n=100), SimpleNamespace(n=100)
    pol = ra.DenseFirstPolicy(sparse, dense)
    T, L = 50, 60
    grid = [[pol.mask(t, l) is dense for l in range(L)] for t in range(T)]
    for t in range(T):
        for l in range(L):
            assert grid[t][l] == (t < 12 or l < 2), (t, l)
    n_dense = sum(map(sum, grid))
    assert n_dense == 12 * 60 + 38 * 2 == pol.dense_calls(T, L)


@pytest.mark.parametrize("steps,blocks,ds,db", [(5, 3, 12, 2), (20, 1, 0, 0), (3, 40, 1, 50), (0, 10, 12, 2)])
def test_dense_call_count(ra, steps, blocks, ds, db):
    pol = ra.DenseFirstPolicy(SimpleNamespace(n=1), SimpleNamespace(n=1), dense_steps=ds, dense_blocks=db)
    assert pol.dense_calls(steps, blocks) == sum(pol.is_dense(t, l) for t in range(steps) for l in range(blocks))


def test_policy_rejects_bad_arguments(ra):
    with pytest.raises(ValueError):
        ra.DenseFirstPolicy(SimpleNamespace(n=1), SimpleNamespace(n=2))
    with pytest.raises(ValueError):
        ra.DenseFirstPolicy(SimpleNamespace(n=1), SimpleNamespace(n=1), dense_steps=-1)
