"""The oracle against the small hand-worked fixtures under tests/golden/.

Each fixture states its citation and its working; the values in it were
worked out by hand, not by running any code."""
import os

import numpy as np
import pytest

from oracle import loopvq_oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                yield line


def test_rates_printed_in_the_abstract():
    rows = [r.split() for r in _rows("rates.txt")]
    assert len(rows) == 2
    for c, g, bits, rate in rows:
        c, g, bits, rate = int(c), int(g), int(bits), float(rate)
        assert O.bits_per_element(c, g, bits) == rate
        # packed bytes of one plane, spread over the g loop steps' elements
        n, d = 1000, 128
        assert O.packed_bytes_per_plane(n, d, c) * 8 / (n * d * g) == rate


def test_rates_match_the_library_layout():
    import sub_bit_vq_b200 as L
    for row in _rows("rates.txt"):
        c, g, _, rate = row.split()
        cfg = L.LoopVQConfig(n_layers=1, n_kv_heads=2, n_q_heads=2, head_dim=96 if c == "8" else 128,
                             n_loops=int(g), loop_group=int(g), chan_group=int(c), n_pages=4,
                             max_batch=1, max_pages_per_seq=4, page_tokens=96 if c == "8" else 64)
        assert L.loopvq_cache_layout(cfg)["bits_per_element"] == float(rate)


def test_pool_offsets_hand_worked():
    rows = [r.split() for r in _rows("pool_offsets.txt")]
    assert len(rows) == 9
    for J, kv, pt, slot, j, off in (map(int, r) for r in rows):
        assert O.plane_offset(slot, j, J, kv, pt) == off, (J, kv, slot, j)
        assert O.plane_offsets(np.array([slot]), J, kv, pt)[0, j] == off


def _encode_fixture():
    x, cw, cases = {}, {}, []
    for r in _rows("encode_hand.txt"):
        head, _, tail = r.partition(":")
        key = head.split()
        vals = [float(v) for v in tail.split()]
        if key[0] == "x":
            x[int(key[1])] = vals
        elif key[0] == "cw":
            cw[(int(key[1]), int(key[2]))] = vals
        elif key[0] == "case":
            cases.append({"w": {} if key[1] == "w" else None, "dist": {}, "idx": {}})
        elif key[0] == "w":
            cases[-1]["w"][int(key[1])] = vals
        elif key[0] == "dist":
            cases[-1]["dist"][int(key[1])] = vals
        elif key[0] == "idx":
            cases[-1]["idx"][int(key[1])] = int(vals[0])
    return x, cw, cases


def test_encode_hand_worked():
    x, cw, cases = _encode_fixture()
    g, c, d, E = 2, 2, 4, 4
    J = d // c
    X = np.zeros((g, 1, 1, d))
    for tau in range(g):
        X[tau, 0, 0] = x[tau]
    cb = np.zeros((1, g, J, E, c))                 # [H][g][J][E][c]
    for (j, e), v in cw.items():
        for tau in range(g):
            cb[0, tau, j, e] = v[tau * c:(tau + 1) * c]
    assert len(cases) == 3
    for case in cases:
        w = None
        if case["w"] is not None:
            w = np.zeros((g, 1, 1, d))
            for j, v in case["w"].items():
                for tau in range(g):
                    w[tau, 0, 0, j * c:(j + 1) * c] = v[tau * c:(tau + 1) * c]
        idx, dist = O.encode_group_ref(X, cb, w)
        for j in range(J):
            np.testing.assert_allclose(dist[0, 0, j], case["dist"][j], rtol=0, atol=1e-12)
            assert idx[0, 0, j] == case["idx"][j]
