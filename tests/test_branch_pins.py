"""Pins of the oracle's multi-branch layer (branches share the embedding table and the value
projection; each has its own key projection and its own residual-stream row).

Checked against facts that do not restate the composition: the one-branch case equals the
single-branch oracle; identical branches give identical results and permuted branches give
permuted results; a zero key projection gates its branch at exactly 1/2 and no other; with
the conv switched off, Delta_b / g_b is the same vector for every branch (one shared v); and
decode token by token with per-branch state reproduces prefill.
"""
from __future__ import annotations

import numpy as np

import oracle
from helpers import make_inputs, small_workload


def _fwd(wl, inp, **kw):
    return oracle.forward_branches(inp["ids"], inp["remap"], inp["tables"], inp["h"], inp["Wk"], inp["Wv"],
                                   inp["gamma_q"], inp["gamma_k"], inp["gamma_c"], inp["conv_w"],
                                   orders=wl.orders, K=wl.K, primes=wl.primes, seed=wl.hash_seed,
                                   pad_id=wl.pad_id, eps=wl.eps, **kw)


def test_one_branch_is_the_single_branch_layer():
    wl = small_workload(B=2, T=30)
    inp = make_inputs(wl)
    single = oracle.forward(inp["ids"], inp["remap"], inp["tables"], inp["h"], inp["Wk"], inp["Wv"],
                            inp["gamma_q"], inp["gamma_k"], inp["gamma_c"], inp["conv_w"], orders=wl.orders,
                            K=wl.K, primes=wl.primes, seed=wl.hash_seed, pad_id=wl.pad_id, eps=wl.eps)
    inp1 = dict(inp, h=inp["h"][:, None, :])
    multi = _fwd(wl, inp1)
    assert np.array_equal(multi["out"][:, 0], single["out"])
    assert np.array_equal(multi["delta"][:, 0], single["delta"])
    assert np.array_equal(multi["idx"], single["idx"])


def test_identical_and_permuted_branches():
    wl = small_workload(B=2, T=25, branches=3)
    inp = make_inputs(wl)
    d = wl.d_h
    # branch 2 := branch 0 (same hidden row, same key projection)
    h = inp["h"].copy()
    h[:, 2] = h[:, 0]
    wk = inp["Wk"].copy()
    wk[2 * d:3 * d] = wk[0:d]
    r = _fwd(wl, dict(inp, h=h, Wk=wk))
    assert np.array_equal(r["out"][:, 2], r["out"][:, 0])
    assert not np.array_equal(r["out"][:, 1], r["out"][:, 0])
    # permuting the branches (hidden rows and key projections together) permutes the results
    perm = [1, 2, 0]
    hp = inp["h"][:, perm]
    wkp = np.concatenate([inp["Wk"][b * d:(b + 1) * d] for b in perm])
    r0 = _fwd(wl, inp)
    rp = _fwd(wl, dict(inp, h=hp, Wk=wkp))
    assert np.array_equal(rp["out"], r0["out"][:, perm])
    assert np.array_equal(rp["gate"], r0["gate"][:, perm])


def test_zero_key_projection_gates_only_its_branch_at_one_half():
    wl = small_workload(B=1, T=20, branches=2)
    inp = make_inputs(wl)
    wk = inp["Wk"].copy()
    wk[: wl.d_h] = 0            # branch 0: k~ = 0, so q.k = 0 and g = sigmoid(0)
    r = _fwd(wl, dict(inp, Wk=wk))
    assert np.all(r["gate"][:, 0] == 0.5)
    assert np.all(np.abs(r["gate"][:, 1] - 0.5) > 1e-6)


def test_branches_share_one_value_vector():
    """With all conv taps zero, Delta_b = U_b = g_b v: Delta_b / g_b must be the same vector for
    every branch (a per-branch value projection would break this)."""
    wl = small_workload(B=2, T=18, branches=3)
    inp = make_inputs(wl)
    r = _fwd(wl, dict(inp, conv_w=np.zeros_like(inp["conv_w"])))
    v = r["delta"] / r["gate"][:, :, None]
    for b in (1, 2):
        assert np.allclose(v[:, b], v[:, 0], rtol=1e-12, atol=1e-15)
    assert not np.allclose(r["gate"][:, 1], r["gate"][:, 0])


def test_branch_decode_matches_prefill():
    wl = small_workload(B=2, T=12, branches=2)
    inp = make_inputs(wl)
    full = _fwd(wl, inp)
    M = wl.branches
    hist = np.full((wl.B, wl.hist_len), wl.pad_id, dtype=np.int32)
    state = np.zeros((wl.B, M, wl.state_len, wl.d_h), dtype=np.uint16)
    h_all = inp["h"].reshape(wl.B, wl.T, M, wl.d_h)
    deltas = []
    for t in range(wl.T):
        step = dict(inp, ids=inp["ids"][:, t:t + 1], h=h_all[:, t].copy())
        r = _fwd(wl, step, history=hist, conv_state=state, decode_outputs=True)
        hist, state = r["history"], r["state"]
        deltas.append(r["delta"])
    delta = np.stack(deltas, axis=1).reshape(wl.B * wl.T, M, wl.d_h)
    assert np.abs(delta - full["delta"]).max() < 2e-2
    assert np.abs(delta - full["delta"]).mean() < 2e-3
