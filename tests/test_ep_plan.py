"""The expert-parallel exchange plan (ft_ep_plan, host only), against a brute
force that follows each routed pair by name.

Every pair is tagged (source rank, row in the source's permuted order,
expert).  The brute force sends the tags through an explicit all-to-all, then
checks the plan's maps on them: the receiver's FFN must visit its experts'
rows expert by expert (sources in rank order, then the source's own order),
and the return trip must bring every tag back to the row it left from."""
import numpy as np
import pytest

from moe_expert_layer_renorm_b200 import _lib
from moe_expert_layer_renorm_b200.ep import ExchangePlan, owned_experts


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _random_counts(g, G, E, skew):
    if skew == "one_expert":
        c = np.zeros((G, E), np.int64)
        c[:, g.integers(E)] = g.integers(0, 50, size=G)
        return c
    if skew == "empty":
        return np.zeros((G, E), np.int64)
    c = g.integers(0, 7, size=(G, E))
    c[g.random((G, E)) < 0.3] = 0
    return c


def _tags(counts_s, s):
    """(source, row, expert) of every row of source s, in its permuted order."""
    out = []
    for e, n in enumerate(counts_s):
        out += [(s, len(out) + i, e) for i in range(n)]
    return out


@pytest.mark.parametrize("G,E", [(1, 8), (2, 8), (3, 12), (4, 128), (8, 32), (8, 8)])
@pytest.mark.parametrize("skew", ["random", "one_expert", "empty"])
def test_plan_moves_every_row_to_its_owner_and_back(G, E, skew):
    g = np.random.default_rng(G * 1000 + E + len(skew))
    counts = _random_counts(g, G, E, skew)
    all_off = np.stack([_offsets(counts[s]) for s in range(G)])
    tags = [_tags(counts[s], s) for s in range(G)]
    plans = [ExchangePlan(all_off, G, E, r) for r in range(G)]

    # the split sizes agree between every pair of ranks
    for s in range(G):
        for d in range(G):
            assert plans[s].send_rows[d] == plans[d].recv_rows[s]
    assert sum(p.n_recv for p in plans) == counts.sum()

    # all-to-all, by hand: rank s's rows for d are those of d's experts, in order
    def owner(e):
        return next(r for r in range(G) if e in owned_experts(E, G, r))

    arrived = {d: [] for d in range(G)}
    for s in range(G):
        for d in range(G):
            mine = [t for t in tags[s] if owner(t[2]) == d]
            assert len(mine) == plans[s].send_rows[d]
            arrived[d] += mine
    for d in range(G):
        p = plans[d]
        got = arrived[d]
        assert len(got) == p.n_recv
        # the FFN's view: local row r reads arrival row perm_src_local[r]
        visit = [got[i] for i in p.perm_src_local[:p.n_recv]]
        assert visit == sorted(got, key=lambda t: (t[2], t[0], t[1]))
        e0 = owned_experts(E, G, d)[0]
        for j in range(E // G):
            grp = visit[p.local_offsets[j]:p.local_offsets[j + 1]]
            assert all(t[2] == e0 + j for t in grp)
        assert p.local_offsets[0] == 0 and p.local_offsets[-1] == p.n_recv
        # ret_idx is the inverse map
        if p.n_recv:
            assert np.array_equal(p.perm_src_local[p.ret_idx[:p.n_recv]], np.arange(p.n_recv))
        # outputs keyed by tag go back in arrival order
        out_local = visit
        out_send = [out_local[i] for i in p.ret_idx[:p.n_recv]]
        assert out_send == got

    # return trip: rank s gets from d what it sent to d, in the order it sent it
    for s in range(G):
        back = []
        for d in range(G):
            start = sum(plans[d].recv_rows[:s])
            chunk = [arrived[d][i] for i in range(start, start + plans[d].recv_rows[s])]
            back += chunk
        assert back == tags[s]


def test_one_rank_is_the_identity():
    off = _offsets([3, 0, 5, 1])
    p = ExchangePlan(off[None, :], 1, 4, 0)
    assert p.n_recv == 9
    assert np.array_equal(p.perm_src_local, np.arange(9))
    assert np.array_equal(p.ret_idx, np.arange(9))
    assert np.array_equal(p.local_offsets, off)
    assert p.send_rows.tolist() == [9] and p.recv_rows.tolist() == [9]


def test_hand_worked_two_ranks():
    # rank 0 routed 2, 1, 0, 2 rows to experts 0..3; rank 1 routed 0, 1, 3, 0
    off = np.array([[0, 2, 3, 3, 5], [0, 0, 1, 4, 4]], np.int32)
    p0, p1 = ExchangePlan(off, 2, 4, 0), ExchangePlan(off, 2, 4, 1)
    assert p0.send_rows.tolist() == [3, 2] and p0.recv_rows.tolist() == [3, 1]
    assert p1.send_rows.tolist() == [1, 3] and p1.recv_rows.tolist() == [2, 3]
    # rank 0 owns experts 0, 1: arrivals 0,1 (e0 from r0), 2 (e1 from r0), 3 (e1 from r1)
    assert p0.local_offsets.tolist() == [0, 2, 4] and p0.perm_src_local.tolist() == [0, 1, 2, 3]
    # rank 1 owns experts 2, 3: arrivals 0,1 (e3 from r0), 2,3,4 (e2 from r1)
    assert p1.local_offsets.tolist() == [0, 3, 5]
    assert p1.perm_src_local.tolist() == [2, 3, 4, 0, 1]
    assert p1.ret_idx.tolist() == [3, 4, 0, 1, 2]


def _plan(off, G, E, rank, cap, with_maps=True):
    a = lambda n: np.zeros(max(n, 1), np.int32)
    return _lib.ep_plan(np.ascontiguousarray(off, np.int32), G, E, rank, cap, a(G), a(G), a(E // max(G, 1) + 1),
                        a(cap) if with_maps else None, a(cap) if with_maps else None)


def test_rejections():
    off = np.array([[0, 1, 2, 3, 4], [0, 1, 1, 1, 1]], np.int32)
    assert _plan(off, 2, 4, 0, 8) == 3                    # experts 0, 1: 2 rows from rank 0, 1 from rank 1
    assert _plan(off, 2, 4, 1, 0, with_maps=False) == 2   # sizes only
    for args in ((off, 2, 4, 2, 8), (off, 2, 4, -1, 8), (off[:, :4], 2, 3, 0, 8), (off, 0, 4, 0, 8)):
        with pytest.raises(_lib.FtError) as e:
            _plan(*args)
        assert e.value.code == _lib.FT_ERR_INVALID_ARG
    with pytest.raises(_lib.FtError, match="cap"):
        _plan(off, 2, 4, 0, 2)
    bad = off.copy()
    bad[1, 0] = 1
    with pytest.raises(_lib.FtError, match="start"):
        _plan(bad, 2, 4, 0, 8)
    bad = off.copy()
    bad[0, 3] = 1
    with pytest.raises(_lib.FtError, match="decreases"):
        _plan(bad, 2, 4, 0, 8)
    with pytest.raises(ValueError):
        owned_experts(10, 4, 0)
