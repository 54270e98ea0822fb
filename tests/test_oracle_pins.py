"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test names what it pins: a published test vector, a closed form, a library routine
as a special case, a brute-force enumeration, or an invariant the pages fix.  Mistakes
these are chosen to catch: a wrong constant or shift in the hash primitives, a gram
window that is off by one or reversed, a wrong head/column order, a transposed weight, a
dropped term in the gate or the residual, a wrong conv tap order or dilation, rounding twice.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

import oracle
import synth
from helpers import ONE_BF16, bf16, f32, make_inputs, small_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
M64 = (1 << 64) - 1


# ------------------------------------------------------------------------ hash primitives
def test_splitmix64_published_vectors():
    """SplitMix64 first outputs from state 0 (published reference vectors)."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "splitmix64_vectors.txt"))
            if l.strip() and not l.startswith("#")]
    for idx, hexval in rows:
        state = (int(idx) * 0x9E3779B97F4A7C15) & M64
        assert oracle.splitmix64(state) == int(hexval, 16)


def test_fmix64_inverts_with_published_inverse_constants():
    """fmix64 followed by the published inverse returns the input: pins both multipliers
    and all three xor-shifts (a wrong shift or constant breaks invertibility)."""
    g = {k: int(v, 16) for k, v in (l.split() for l in open(os.path.join(GOLDEN, "fmix64_inverse.txt"))
                                     if l.strip() and not l.startswith("#"))}
    assert (g["mult1"] * g["inv1"]) & M64 == 1 and (g["mult2"] * g["inv2"]) & M64 == 1
    rng = np.random.default_rng(3)
    for k in [0, 1, 2, M64, 0x8000000000000000] + [int(x) for x in rng.integers(0, 2**63, 200)]:
        y = oracle.fmix64(k)
        y ^= y >> 33
        y = (y * g["inv2"]) & M64
        y ^= y >> 33
        y = (y * g["inv1"]) & M64
        y ^= y >> 33
        assert y == k
    assert oracle.fmix64(0) == 0


def test_multipliers_odd_and_distinct():
    ms = {oracle.hash_multiplier(0x5EED, o, j, i) for o in (2, 3) for j in range(8) for i in range(o)}
    assert len(ms) == 40 and all(m & 1 for m in ms)


# ------------------------------------------------------------------------ bf16 rounding
def _nearest_bf16_bruteforce(x: float) -> int:
    """Scan the two bf16 neighbours of x (via exact float64 arithmetic), nearest wins,
    ties go to the even pattern."""
    f = np.float32(x)
    b = int(np.array([f], dtype=np.float32).view(np.uint32)[0] >> 16)
    cands = [(b + d) & 0xFFFF for d in (-1, 0, 1, 2)]
    best = None
    for c in cands:
        v = float(synth.bf16_to_float(np.array([c], dtype=np.uint16))[0])
        if not math.isfinite(v) or (c & 0x7F80) == 0x7F80:
            continue
        if math.copysign(1.0, v) != math.copysign(1.0, x) and v != 0.0:
            continue
        err = abs(v - x)
        key = (err, c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_double_to_bf16_single_rounding_ties_and_bruteforce():
    # exact tie between 1 and 1+2^-7 -> even (1.0)
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    # just above the tie: must round up.  Rounding through binary32 first loses the 2^-40
    # and ties down -- the double-rounding mistake this pins.
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle.double_to_bf16(-(1.0 + 2.0 ** -8 + 2.0 ** -40)) == 0xBF81
    # odd mantissa tie rounds up to even
    assert oracle.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    rng = np.random.default_rng(11)
    xs = np.concatenate([rng.normal(0, 1, 3000), rng.normal(0, 1e-3, 500), rng.normal(0, 300, 500)])
    for x in xs:
        assert oracle.double_to_bf16(float(x)) == _nearest_bf16_bruteforce(float(x))


def test_double_to_bf16_matches_torch_on_binary32_inputs():
    """For binary32-representable inputs one rounding = torch's float->bf16 (RNE)."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(12)
    xs = rng.normal(0, 2, 5000).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.double_to_bf16(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(ref, got)


# ------------------------------------------------------------------------ remap
def test_remap_is_table_lookup_and_rejects_out_of_vocab():
    wl = small_workload()
    table = wl.remap()
    ids = wl.ids()
    assert np.array_equal(oracle.remap(ids, table), table[ids])   # numpy fancy indexing
    ident = np.arange(wl.vocab_in, dtype=np.int32)
    assert np.array_equal(oracle.remap(ids, ident), ids)
    with pytest.raises(ValueError):
        oracle.remap(np.array([[wl.vocab_in]], dtype=np.int32), table)
    with pytest.raises(ValueError):
        oracle.remap(np.array([[-1]], dtype=np.int32), table)


def test_synthetic_remap_is_many_to_one_and_onto():
    t = synth.remap_table(1000, 770, 123)
    assert t.min() == 0 and t.max() == 769 and np.unique(t).size == 770
    # the pages' compression: 128k ids down by 23%
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    assert round(128_000 * (1 - facts["compression_fraction"]["value"])) == 98_560


# ------------------------------------------------------------------------ hash windows
@pytest.mark.parametrize("V", [8, 31])
def test_hash_brute_force_every_gram(V):
    """Every bigram and trigram of a V-id vocabulary, placed in sequences of length 3, gets
    at every position exactly the row ids of its own gram evaluated in isolation (with the
    pad id before the sequence start): pins the window (which ids, in which order), the
    column layout (order-major, head-minor) and the padding."""
    orders, K = (2, 3), 2
    primes = (1009, 1013, 1019, 1021)
    seed, pad = 77, V
    a, b, c = np.meshgrid(np.arange(V), np.arange(V), np.arange(V), indexing="ij")
    xr = np.stack([a.ravel(), b.ravel(), c.ravel()], axis=1).astype(np.int32)   # [V^3, 3]
    idx = oracle.hash_ids(xr, orders, K, primes, seed, pad).reshape(V ** 3, 3, 4)
    H = {}
    def ref(gram, o, j):
        key = (tuple(gram), o, j)
        if key not in H:
            H[key] = oracle.hash_gram(gram, o, j, seed, primes[(o - 2) * K + j])
        return H[key]
    for s in range(0, V ** 3, max(1, V ** 3 // 400)):
        x0, x1, x2 = (int(v) for v in xr[s])
        windows = {0: {2: [x0, pad], 3: [x0, pad, pad]},
                   1: {2: [x1, x0], 3: [x1, x0, pad]},
                   2: {2: [x2, x1], 3: [x2, x1, x0]}}
        for t in range(3):
            for o in (2, 3):
                for j in range(K):
                    assert idx[s, t, (o - 2) * K + j] == ref(windows[t][o], o, j)
    # exhaustive over the bigram table at position 2: same gram -> same row, any sequence
    bi = idx[:, 2, :K]
    for j in range(K):
        byg = {}
        for s in range(V ** 3):
            g = (int(xr[s, 2]), int(xr[s, 1]))
            assert byg.setdefault(g, bi[s, j]) == bi[s, j]


def test_hash_order_sensitive_and_history_equivalent():
    orders, K, primes, seed, pad = (2, 3), 1, (999983, 999979), 5, 1000
    assert oracle.hash_gram([1, 2], 2, 0, seed, primes[0]) != oracle.hash_gram([2, 1], 2, 0, seed, primes[0])
    rng = np.random.default_rng(0)
    x = rng.integers(0, 1000, (3, 50)).astype(np.int32)
    full = oracle.hash_ids(x, orders, K, primes, seed, pad).reshape(3, 50, 2)
    # splitting a sequence and carrying the last (max order - 1) ids as history is exact
    first = oracle.hash_ids(x[:, :20], orders, K, primes, seed, pad).reshape(3, 20, 2)
    hist = oracle.advance_history(x[:, :20], None, 2, pad)
    assert np.array_equal(hist, x[:, 18:20])
    second = oracle.hash_ids(x[:, 20:], orders, K, primes, seed, pad, history=hist).reshape(3, 30, 2)
    assert np.array_equal(np.concatenate([first, second], axis=1), full)
    # a one-token step with a one-token-long prior call still carries the pad correctly
    h1 = oracle.advance_history(x[:, :1], None, 2, pad)
    assert np.array_equal(h1[:, 0], np.full(3, pad)) and np.array_equal(h1[:, 1], x[:, 0])


def _chi2_p(counts: np.ndarray) -> float:
    from scipy.stats import chisquare
    return float(chisquare(counts).pvalue)


def test_hash_occupancy_uniform_and_heads_independent():
    """Row ids spread uniformly over each prime table (chi-square vs uniform) and two heads
    of one order collide on a pair of grams about as often as independent hashes (1/P)."""
    primes = (10007, 10009, 10037, 10039)
    seed, pad = 0x5EED, 770
    V = 770
    a, b = np.meshgrid(np.arange(V), np.arange(V), indexing="ij")
    xr = np.stack([b.ravel(), a.ravel()], axis=1).astype(np.int32)   # every bigram (a, b)
    idx = oracle.hash_ids(xr, (2, 3), 2, primes, seed, pad).reshape(V * V, 2, 4)
    big = idx[:, 1, :2]                                              # 2-gram heads at t=1
    for j in range(2):
        assert big[:, j].max() < primes[j]
        counts = np.bincount(big[:, j], minlength=primes[j])
        assert _chi2_p(counts) > 1e-3
    # trigram heads on 10^6 sampled trigrams
    rng = np.random.default_rng(9)
    tri = rng.integers(0, V, (1_000_000, 3)).astype(np.int32)
    tidx = oracle.hash_ids(tri, (2, 3), 2, primes, seed, pad).reshape(-1, 3, 4)[:, 2, 2:]
    for j in range(2):
        assert _chi2_p(np.bincount(tidx[:, j], minlength=primes[2 + j])) > 1e-3
    # pair collisions: for random gram pairs, P(h0 equal) * P(h1 equal) ~ joint rate
    n = big.shape[0]
    i1, i2 = rng.integers(0, n, 2_000_000), rng.integers(0, n, 2_000_000)
    keep = i1 != i2
    c0 = big[i1[keep], 0] == big[i2[keep], 0]
    c1 = big[i1[keep], 1] == big[i2[keep], 1]
    assert abs(c0.mean() - 1 / primes[0]) < 4 * math.sqrt(1 / primes[0] / keep.sum())
    assert (c0 & c1).sum() <= 3      # expected ~2e-2 joint collisions if independent


# ------------------------------------------------------------------------ gather layout
def test_gather_layout_two_passes():
    """Tables filled with exactly representable codes: pass 1 encodes (table, column),
    pass 2 encodes the row, so every position of m is checked against the concatenation
    order (head h occupies columns h*d_e .. h*d_e + d_e - 1)."""
    wl = small_workload(K=3, d_e=24)
    H, d_e = wl.H, wl.d_e
    xr = wl.remap()[wl.ids()]
    idx = oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    t1 = [bf16(np.tile(((h * d_e + np.arange(d_e)) % 256).astype(np.float32), (P, 1))) for h, P in enumerate(wl.primes)]
    m1 = f32(oracle.gather(idx, t1)).reshape(-1, H, d_e)
    for h in range(H):
        assert np.array_equal(m1[:, h, :], np.tile((h * d_e + np.arange(d_e)) % 256, (m1.shape[0], 1)))
    t2 = [bf16(np.tile((np.arange(P) % 256).astype(np.float32)[:, None], (1, d_e))) for P in wl.primes]
    m2 = f32(oracle.gather(idx, t2)).reshape(-1, H, d_e)
    for h in range(H):
        assert np.array_equal(m2[:, h, :], np.tile((idx[:, h] % 256)[:, None], (1, d_e)))


# ------------------------------------------------------------------------ gate closed forms
def _unit_gammas(d):
    return [np.full(d, ONE_BF16, dtype=np.uint16)] * 3


def test_gate_closed_form_aligned_and_opposed():
    """W_k = W_v = I, h = +m gives q.k/sqrt(d) = sqrt(d) (up to eps) so g = sigmoid(sqrt d);
    h = -m gives sigmoid(-sqrt d) ~ 0: the pages' suppression of contradicting memory."""
    d, T = 64, 12
    rng = np.random.default_rng(1)
    m = bf16(rng.normal(0, 1, (T, d)))
    eye = bf16(np.eye(d))
    zero_w = np.zeros((d, 4), dtype=np.uint16)
    gq, gk, gc = _unit_gammas(d)
    for sign in (+1, -1):
        h = bf16(sign * f32(m))
        r = oracle.gate_conv(h, m, eye, eye, gq, gk, gc, zero_w, 1, T)
        expect = 1 / (1 + math.exp(-sign * math.sqrt(d)))
        assert np.allclose(r["gate"], expect, rtol=1e-5, atol=1e-9)
        # conv weights zero -> Delta = U = g * v exactly (no conv term, no dropped U)
        assert np.allclose(r["delta"], r["gate"][:, None] * f32(m), rtol=1e-12, atol=1e-15)
    assert r["gate"].max() < 1e-3


def test_projection_orientation_non_square():
    """W_k = 0 makes k = 0 and g = sigmoid(0) = 1/2 exactly, so Delta = v/2 with conv off:
    v must equal W_v @ m (numpy matmul) on a non-square [d_h, d_m] weight, which catches a
    transposed operand; a permutation-shaped W_k aligned with h pins the k side."""
    d_m, d_h, T = 48, 32, 10
    rng = np.random.default_rng(2)
    m = bf16(rng.normal(0, 1, (T, d_m)))
    Wv = bf16(rng.normal(0, 0.1, (d_h, d_m)))
    Wk0 = np.zeros((d_h, d_m), dtype=np.uint16)
    h = bf16(rng.normal(0, 1, (T, d_h)))
    gq, gk, gc = _unit_gammas(d_h)
    zw = np.zeros((d_h, 4), dtype=np.uint16)
    r = oracle.gate_conv(h, m, Wk0, Wv, gq, gk, gc, zw, 1, T)
    assert np.all(r["gate"] == 0.5)
    v = f32(m).astype(np.float64) @ f32(Wv).astype(np.float64).T
    assert np.allclose(2 * r["delta"], v, rtol=1e-12, atol=1e-12)
    # W_k selects columns perm[r] of m; h = m[:, perm] makes k~ = h, so g = sigmoid(sqrt d_h)
    perm = rng.permutation(d_m)[:d_h]
    Wk = np.zeros((d_h, d_m), dtype=np.float32)
    Wk[np.arange(d_h), perm] = 1.0
    h2 = m[:, perm]
    r2 = oracle.gate_conv(h2, m, bf16(Wk), Wv, gq, gk, gc, zw, 1, T)
    assert np.allclose(r2["gate"], 1 / (1 + math.exp(-math.sqrt(d_h))), rtol=1e-5)
    # the transposed reading (W_k as [d_m, d_h]) cannot even form k~ = h here
    assert not np.allclose(f32(m).astype(np.float64)[:, :d_h] @ Wk[:, :d_h], f32(h2))


def test_gate_in_open_unit_interval_and_gamma_scaling():
    wl = small_workload(T=30)
    inp = make_inputs(wl)
    xr = wl.remap()[inp["ids"]]
    idx = oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    m = oracle.gather(idx, inp["tables"])
    r = oracle.gate_conv(inp["h"], m, inp["Wk"], inp["Wv"], inp["gamma_q"], inp["gamma_k"],
                         inp["gamma_c"], inp["conv_w"], wl.B, wl.T)
    assert np.all(r["gate"] > 0) and np.all(r["gate"] < 1)
    # gamma_q = gamma_k = 2 scales q.k by 4 -- the logit is 4x larger
    two = np.full(wl.d_h, 0x4000, dtype=np.uint16)
    r2 = oracle.gate_conv(inp["h"], m, inp["Wk"], inp["Wv"], two, two, inp["gamma_c"],
                          inp["conv_w"], wl.B, wl.T)
    logit = lambda g: np.log(g / (1 - g))
    assert np.allclose(logit(r2["gate"]), 4 * logit(r["gate"]), rtol=1e-9, atol=1e-9)


# ------------------------------------------------------------------------ conv
def test_conv_impulse_response_taps_and_dilation():
    """Memory is zero except a one-hot at token s, channel ch.  With W_k = W_v = I the conv
    input u is zero except u_s[ch] = g/sqrt(g^2/d + eps) (RMSNorm of a one-hot), so
    Delta[t, ch] = [t==s] g + c sigmoid(c) with c = w[ch][i] u_s exactly at t = s + 3i, and
    Delta = 0 everywhere else: pins tap order (tap 0 = current), dilation 3, kernel 4,
    causality and the SiLU form."""
    d, T, s, ch = 32, 24, 5, 7
    eps = 1e-6
    m = np.zeros((T, d), dtype=np.float32)
    m[s, ch] = 1.0
    m = bf16(m)
    rng = np.random.default_rng(4)
    h = bf16(rng.normal(0, 1, (T, d)))
    eye = bf16(np.eye(d))
    w = bf16(rng.normal(0, 0.5, (d, 4)))
    gq, gk, gc = _unit_gammas(d)
    r = oracle.gate_conv(h, m, eye, eye, gq, gk, gc, w, 1, T, eps=eps)
    g = r["gate"][s]
    us = g / math.sqrt(g * g / d + eps)
    wf = f32(w).astype(np.float64)
    expect = np.zeros((T, d))
    expect[s, ch] = g
    for i in range(4):
        c = wf[ch, i] * us
        expect[s + 3 * i, ch] += c / (1 + math.exp(-c))
    assert np.allclose(r["delta"], expect, rtol=1e-12, atol=1e-14)
    # out is the bf16 RNE of h + Delta
    want = np.array([oracle.double_to_bf16(float(x)) for x in (f32(h) + expect).ravel()], dtype=np.uint16)
    assert np.array_equal(r["out"].ravel(), want)


def _forward(wl, inp, **kw):
    return oracle.forward(inp["ids"], inp["remap"], inp["tables"], inp["h"], inp["Wk"], inp["Wv"],
                          inp["gamma_q"], inp["gamma_k"], inp["gamma_c"], inp["conv_w"],
                          orders=wl.orders, K=wl.K, primes=wl.primes, seed=wl.hash_seed,
                          pad_id=wl.pad_id, eps=wl.eps, **kw)


def test_causality_and_receptive_field():
    """Changing the token at s (and h at s) leaves every output before s bit-identical and
    changes Delta only at s+{0,1,2}+{0,3,6,9}: grams reach 2 back, the conv 9 back."""
    wl = small_workload(B=1, T=40)
    inp = make_inputs(wl)
    base = _forward(wl, inp)
    s = 17
    inp2 = dict(inp)
    ids2 = inp["ids"].copy()
    ids2[0, s] = (ids2[0, s] + 1) % wl.vocab_in
    while wl.remap()[ids2[0, s]] == wl.remap()[inp["ids"][0, s]]:
        ids2[0, s] = (ids2[0, s] + 1) % wl.vocab_in
    inp2["ids"] = ids2
    pert = _forward(wl, inp2)
    assert np.array_equal(pert["out"][:s], base["out"][:s])
    reach = sorted({s + a + b for a in (0, 1, 2) for b in (0, 3, 6, 9)})
    changed = np.nonzero(np.any(pert["delta"] != base["delta"], axis=1))[0]
    assert set(changed.tolist()) <= set(reach)
    assert s in changed
    # perturbing h at s: only positions s, s+3, s+6, s+9 (gate at s, then the conv)
    inp3 = dict(inp)
    h3 = inp["h"].copy()
    h3[s] = bf16(-f32(h3[s]))
    inp3["h"] = h3
    pert3 = _forward(wl, inp3)
    changed3 = set(np.nonzero(np.any(pert3["delta"] != base["delta"], axis=1))[0].tolist())
    assert changed3 <= {s, s + 3, s + 6, s + 9} and s in changed3


def test_forward_equals_composed_steps():
    wl = small_workload(B=2, T=25)
    inp = make_inputs(wl)
    r = _forward(wl, inp)
    xr = oracle.remap(inp["ids"], inp["remap"])
    idx = oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    assert np.array_equal(idx, r["idx"])
    m = oracle.gather(idx, inp["tables"])
    g = oracle.gate_conv(inp["h"], m, inp["Wk"], inp["Wv"], inp["gamma_q"], inp["gamma_k"],
                         inp["gamma_c"], inp["conv_w"], wl.B, wl.T)
    assert np.array_equal(g["out"], r["out"]) and np.array_equal(g["delta"], r["delta"])


def test_decode_steps_match_prefill():
    """Running a sequence token by token with the hash history and the conv state carried
    between calls reproduces one-shot prefill: indices exactly, outputs within the bf16
    rounding of the stored conv state."""
    wl = small_workload(B=3, T=14)
    inp = make_inputs(wl)
    full = _forward(wl, inp)
    hist = np.full((wl.B, wl.hist_len), wl.pad_id, dtype=np.int32)
    state = np.zeros((wl.B, wl.state_len, wl.d_h), dtype=np.uint16)
    outs, deltas, idxs = [], [], []
    h_all = inp["h"].reshape(wl.B, wl.T, wl.d_h)
    for t in range(wl.T):
        step = dict(inp)
        step["ids"] = inp["ids"][:, t:t + 1]
        step["h"] = h_all[:, t, :].copy()
        r = _forward(wl, step, history=hist, conv_state=state, decode_outputs=True)
        hist, state = r["history"], r["state"]
        outs.append(r["out"]); deltas.append(r["delta"]); idxs.append(r["idx"])
    idx = np.stack(idxs, axis=1).reshape(wl.B * wl.T, -1)
    assert np.array_equal(idx, full["idx"])
    delta = np.stack(deltas, axis=1).reshape(wl.B * wl.T, -1)
    assert np.abs(delta - full["delta"]).max() < 2e-2
    assert np.abs(delta - full["delta"]).mean() < 2e-3
    # the state after the last step holds bf16(u) of the last 9 positions
    ref_state = oracle.gate_conv(inp["h"], oracle.gather(full["idx"], inp["tables"]), inp["Wk"],
                                 inp["Wv"], inp["gamma_q"], inp["gamma_k"], inp["gamma_c"],
                                 inp["conv_w"], wl.B, wl.T, want_state=True)["state"]
    diff = np.abs(f32(state).astype(np.float64) - f32(ref_state))
    assert diff.max() < 0.05


# ------------------------------------------------------------------------ geometry facts
def test_workload_geometry_matches_pages():
    facts = {k: v["value"] for k, v in json.load(open(os.path.join(GOLDEN, "pages_facts.json"))).items()
             if not k.startswith("_")}
    wl = synth.get_workload("decode20m")
    params = sum(wl.primes) * wl.d_e
    assert round(params / 1e9, 1) == facts["ngram_params_billion"]
    assert round(wl.table_bytes / 2 ** 30, 1) == facts["ngram_bf16_gib"]
    assert abs(sum(wl.primes) - facts["ngram_entries"]) < 100
    assert wl.d_h == facts["hidden_dim"] and wl.vocab_in == facts["vocab"]
    assert wl.conv_kernel == facts["conv_kernel"] and wl.conv_dilation == max(facts["orders"])
    assert facts["heads_2gram"] + facts["heads_3gram"] == facts["row_ids_per_token"]
    assert facts["row_ids_per_token"] * facts["values_per_row"] == facts["memory_vector_dim"]
    l2 = synth.get_workload("layer2560")
    assert l2.H == facts["row_ids_per_token"] and l2.d_e == facts["values_per_row"]
    assert l2.d_m == facts["memory_vector_dim"]
    assert all(synth.workloads.is_prime(p) for w in synth.WORKLOADS.values() for p in w.primes)
