"""Pins of the oracle's routing, replay and permute steps.  No GPU.

Top-k per token: "prime-rl 0.6.0 løfter trillion-parameter RL ...",
§Drift og omkostninger i realiteten.  Replay payload [num_layers, top_k,
seq_len]: "RL at 1T scale: prime-rl performance deep dive", §Router Replay.
"""
import json
import os

import numpy as np
import pytest
import scipy.special

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _logits(rng, T, E, ties=False):
    if ties:
        return rng.integers(-3, 3, (T, E)).astype(np.float32)
    return rng.standard_normal((T, E)).astype(np.float32)


@pytest.mark.parametrize("T,E,k,ties", [(300, 8, 2, False), (257, 64, 6, False),
                                        (200, 32, 8, True), (50, 5, 5, True)])
def test_topk_matches_stable_argsort(orc, T, E, k, ties):
    rng = np.random.default_rng(20)
    z = _logits(rng, T, E, ties)
    idx, w = orc.route_topk(z, k)
    ref = np.argsort(-z, axis=1, kind="stable")[:, :k]
    assert np.array_equal(idx, ref)
    # invariant: every chosen logit >= every unchosen one
    chosen = np.zeros_like(z, bool)
    np.put_along_axis(chosen, idx.astype(np.int64), True, axis=1)
    if k < E:
        assert np.all(np.where(chosen, z, np.inf).min(1) >= np.where(chosen, -np.inf, z).max(1))
    # weights: softmax over the chosen logits (library), summing to 1
    zS = np.take_along_axis(z, idx.astype(np.int64), axis=1).astype(np.float64)
    assert np.allclose(w, scipy.special.softmax(zS, axis=1), rtol=1e-6, atol=1e-7)
    assert np.allclose(w.astype(np.float64).sum(1), 1.0, atol=1e-6)


def test_topk_neg_inf_logits(orc):
    z = np.array([[-np.inf, 0.5, -np.inf, 0.25, -np.inf, 1.0]], np.float32)
    idx, w = orc.route_topk(z, 3)
    assert list(idx[0]) == [5, 1, 3]
    idx, w = orc.route_topk(z, 4)
    assert list(idx[0]) == [5, 1, 3, 0] and w[0, 3] == 0.0


def test_replay_of_capture_reproduces_topk(orc):
    rng = np.random.default_rng(21)
    T, E, k, L = 333, 16, 4, 3
    zs = [_logits(rng, T, E) for _ in range(L)]
    routed = [orc.route_topk(z, k) for z in zs]
    payload = np.stack([r[0].T for r in routed])  # [L, k, T]
    for layer in range(L):
        idx, w, st = orc.route_replay(payload, layer, E, z=zs[layer])
        assert st == 0
        assert np.array_equal(idx, routed[layer][0])
        assert np.array_equal(w, routed[layer][1])


def test_replay_arbitrary_payload_and_given_weights(orc):
    rng = np.random.default_rng(22)
    T, E, k, L = 100, 64, 6, 2
    payload = np.stack([np.stack([rng.permutation(E)[:k] for _ in range(T)]).T
                        for _ in range(L)]).astype(np.int32)
    w_in = rng.random((T, k)).astype(np.float32)
    idx, w, st = orc.route_replay(payload, 1, E, w_in=w_in)
    assert st == 0
    assert np.array_equal(idx, payload[1].T)
    assert np.array_equal(w, w_in)


def test_replay_rejects_bad_payloads(orc):
    T, E, k = 4, 8, 2
    P = np.array([[[0, 1, 2, 3], [4, 5, 6, 7]]], np.int32)
    w_in = np.full((T, k), 0.5, np.float32)
    assert orc.route_replay(P, 0, E, w_in=w_in)[2] == 0
    bad = P.copy(); bad[0, 1, 2] = 8
    idx, w, st = orc.route_replay(bad, 0, E, w_in=w_in)
    assert st == 4 and np.all(w[2] == 0) and np.all(w[[0, 1, 3]] == 0.5)
    dup = P.copy(); dup[0, 1, 0] = 0
    assert orc.route_replay(dup, 0, E, w_in=w_in)[2] == 4
    neg = P.copy(); neg[0, 0, 3] = -1
    assert orc.route_replay(neg, 0, E, w_in=w_in)[2] == 4


def test_golden_replay_layout(orc):
    with open(os.path.join(GOLDEN, "replay_payload_layout.json")) as f:
        g = json.load(f)
    P = np.array(g["payload"], np.int32)
    for layer, want in enumerate(g["idx_per_layer"]):
        idx, _, st = orc.route_replay(P, layer, g["E"], w_in=np.ones((P.shape[2], P.shape[1]), np.float32))
        assert st == 0 and idx.tolist() == want


@pytest.mark.parametrize("T,E,k,align", [(300, 8, 2, 128), (300, 8, 2, 1), (1000, 64, 6, 128),
                                         (64, 32, 8, 128), (1, 4, 4, 128), (0, 4, 2, 128)])
def test_permute_against_library_sort(orc, T, E, k, align):
    rng = np.random.default_rng(23)
    p = np.arange(1, E + 1, dtype=np.float64) ** -1.5
    if E - k >= 2:
        p[-2:] = 0  # empty experts
    p /= p.sum()
    idx = np.array([rng.choice(E, k, replace=False, p=p) for _ in range(T)],
                   np.int32).reshape(T, k)
    counts, offsets, pos, src = orc.permute(idx, E, align)
    flat = idx.ravel()
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    padded = (counts + align - 1) // align * align
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(padded)]))
    assert counts.sum() == T * k
    order = np.argsort(flat, kind="stable")  # entries grouped by expert, stable
    rows = np.concatenate([np.arange(offsets[e], offsets[e] + counts[e]) for e in range(E)])
    assert np.array_equal(pos.ravel()[order], rows)
    ok = src >= 0
    assert np.array_equal(np.sort(src[ok]), np.arange(T * k))
    assert np.array_equal(src[pos.ravel()], np.arange(T * k))
    # unpermute(permute(X)) == X for every copy j
    X = rng.standard_normal((T, 5))
    Xp = np.zeros((len(src), 5)); Xp[ok] = X[src[ok] // k]
    for j in range(k):
        assert np.array_equal(Xp[pos[:, j]], X)


def test_permute_drops_invalid_entries(orc):
    idx = np.array([[0, 9], [1, 0]], np.int32)
    counts, offsets, pos, src = orc.permute(idx, 4, 1)
    assert counts.tolist() == [2, 1, 0, 0] and pos.tolist() == [[0, -1], [2, 1]]
