"""Property-based pin of the oracle's routing: for any expert ids (valid, masked
-1, or out of range) the result is the unique stable grouping -- checked against
a definition written differently (a counting pass per expert)."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import layer as L


@settings(max_examples=200, deadline=None)
@given(st.integers(1, 12), st.integers(1, 40), st.data())
def test_route_is_the_stable_grouping(E, T, data):
    k = data.draw(st.integers(1, E))
    ids = np.array(data.draw(st.lists(st.integers(-3, E + 2), min_size=T * k, max_size=T * k)),
                   dtype=np.int64).reshape(T, k)
    counts, offsets, perm, inv = L.route(ids, E)
    flat = ids.reshape(-1)
    # Definition: expert e's block lists the slots holding e in increasing order,
    # blocks in expert order; slots with an id outside [0, E) are in no block.
    expect = [s for e in range(E) for s in range(flat.size) if flat[s] == e]
    assert list(perm[:len(expect)]) == expect
    assert all(p == -1 for p in perm[len(expect):])
    assert [int(c) for c in counts] == [int((flat == e).sum()) for e in range(E)]
    assert int(offsets[0]) == 0 and list(np.diff(offsets)) == list(counts)
    for pos, s in enumerate(expect):
        assert inv[s] == pos
    for s in range(flat.size):
        if not 0 <= flat[s] < E:
            assert inv[s] == -1
