"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: remapped ids, row ids, gathered memory vectors, the GPU input generator.
Tolerance (stated in gpu_helpers): Delta max-abs 1e-2 / mean-abs 1e-3; out within
max(1e-2, one bf16 ulp) and mean-abs 1e-3.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hashed_gram_embedding_remap_b200 as E
import oracle
import synth
from gpu_helpers import (DeviceInputs, assert_bf16_within_ulp, assert_delta_close, assert_out_close, host_tables,
                         table_scales, to_dev, to_host_u16)
from helpers import small_workload
from synth import fill_gpu

pytestmark = pytest.mark.gpu


def _idx_oracle(wl, ids_np, history=None):
    xr = wl.remap()[ids_np]
    return oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id, history=history)


# ------------------------------------------------------------------ generator
def test_gpu_fill_matches_cpu_bits():
    spec = synth.FillSpec(2024, 3, 0.02)
    t = fill_gpu.filled((1003, 40), spec)
    assert np.array_equal(to_host_u16(t), synth.fill_bf16(spec, (1003, 40)))
    # rows regenerated on demand from a large tensor
    big = fill_gpu.filled((200_003, 160), spec)
    rows = np.array([0, 1, 77777, 200_002])
    assert np.array_equal(to_host_u16(big[torch.from_numpy(rows).cuda()]), synth.fill_rows_bf16(spec, 160, rows))


# ------------------------------------------------------------------ steps 1-2
@pytest.mark.parametrize("name", ["tiny", "layer2560", "prefill20m"])
def test_remap_and_hash_bit_exact_full_size(name):
    wl = synth.get_workload(name)
    plan = E.Plan.from_workload(wl)
    ids = wl.ids()
    d_ids, d_remap = to_dev(ids), to_dev(wl.remap())
    xr = torch.empty_like(d_ids)
    E.engram_remap(plan, d_ids, d_remap, xr)
    xr_ref = oracle.remap(ids, wl.remap())
    assert np.array_equal(xr.cpu().numpy(), xr_ref)
    idx = torch.empty((wl.n_tok, wl.H), dtype=torch.int32, device="cuda")
    E.engram_hash(plan, xr, idx)
    ref = oracle.hash_ids(xr_ref, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    assert np.array_equal(idx.cpu().numpy().view(np.uint32), ref)


def test_hash_with_history_and_advance():
    wl = synth.get_workload("decode20m")
    plan = E.Plan.from_workload(wl)
    hist_np = wl.history()
    for T in (1, 2, 5):
        ids = synth.zipf_ids(wl.vocab_in, 1.1, (wl.B, T), 99 + T)
        d_ids, hist = to_dev(ids), to_dev(hist_np)
        idx = torch.empty((wl.B * T, wl.H), dtype=torch.int32, device="cuda")
        E.engram_hash(plan, d_ids, idx, history=hist)
        ref = oracle.hash_ids(ids, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id, history=hist_np)
        assert np.array_equal(idx.cpu().numpy().view(np.uint32), ref)
        E.engram_advance_history(plan, d_ids, hist)
        assert np.array_equal(hist.cpu().numpy(), oracle.advance_history(ids, hist_np, 2, wl.pad_id))


def test_hash_brute_force_small_vocab():
    V = 31
    wl = small_workload(vocab_in=V, vocab_out=V, B=V * V, T=3)
    plan = E.Plan.from_workload(wl)
    a, b, c = np.meshgrid(np.arange(V), np.arange(V), np.arange(V), indexing="ij")
    xr = np.stack([a.ravel(), b.ravel(), c.ravel()], axis=1).astype(np.int32)
    idx = torch.empty((xr.size, wl.H), dtype=torch.int32, device="cuda")
    E.engram_hash(plan, to_dev(xr), idx)
    ref = oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    assert np.array_equal(idx.cpu().numpy().view(np.uint32), ref)


# ------------------------------------------------------------------ step 3
@pytest.mark.parametrize("bulk", [False, True])
@pytest.mark.parametrize("K,d_e,B,T", [(2, 32, 3, 97), (3, 40, 3, 97), (8, 160, 3, 97), (1, 1024, 3, 97),
                                       (1, 2560, 3, 97), (1, 2560, 8, 1000)])
def test_gather_bit_exact(K, d_e, B, T, bulk):
    """The register gather and the bulk-copy gather (ENGRAM_FLAG_BULK_GATHER: a 32-row ring per
    one-warp CTA for rows under 2 KB, an 8-row ring for 1,024 and 2,560 columns, the second
    the 20M-row geometry) against the oracle; 16,000 rows of 2,560 columns take 22 rows per
    CTA, so the ring wraps."""
    wl = small_workload(K=K, d_e=d_e, B=B, T=T)
    plan = E.Plan.from_workload(wl, flags=E.ENGRAM_FLAG_BULK_GATHER if bulk else 0)
    if bulk:
        assert E.engram_forward_path(plan, B, T) & E.ENGRAM_PATH_BULK_GATHER or B * T * wl.H <= 16384
    tables_np = [synth.fill_bf16(wl.table_spec(h), (wl.primes[h], d_e)) for h in range(wl.H)]
    tables = [to_dev(t) for t in tables_np]
    idx_np = _idx_oracle(wl, wl.ids())
    m = torch.empty((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
    E.engram_gather(plan, to_dev(idx_np.view(np.int32)), tables, m)
    assert np.array_equal(to_host_u16(m), oracle.gather(idx_np, tables_np))


def test_gather_full_size_layer2560_sampled_rows():
    wl = synth.get_workload("layer2560")
    di = DeviceInputs(wl)
    idx_np = _idx_oracle(wl, di.ids_np)
    m = torch.empty((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
    E.engram_gather(di.plan, to_dev(idx_np.view(np.int32)), di.tables, m)
    rng = np.random.default_rng(5)
    sample = np.concatenate([[0, 1, wl.n_tok - 1], rng.integers(0, wl.n_tok, 200)])
    got = to_host_u16(m[torch.from_numpy(sample).cuda()]).reshape(len(sample), wl.H, wl.d_e)
    for h in range(wl.H):
        ref = synth.fill_rows_bf16(wl.table_spec(h), wl.d_e, idx_np[sample, h])
        assert np.array_equal(got[:, h, :], ref)


def test_bad_ids_and_rows_raise_status_not_faults():
    wl = small_workload(B=1, T=16)
    plan = E.Plan.from_workload(wl)
    E.engram_device_status(clear=True)
    ids = torch.tensor([[0, 5, wl.vocab_in + 3, -1] * 4], dtype=torch.int32, device="cuda")
    out = torch.empty_like(ids)
    E.engram_remap(plan, ids, to_dev(wl.remap()), out)
    assert E.engram_device_status(clear=True) & E.ENGRAM_STATUS_BAD_TOKEN
    assert (out.cpu().numpy()[0, 2::4] == wl.pad_id).all()
    tables = [to_dev(synth.fill_bf16(wl.table_spec(h), (wl.primes[h], wl.d_e))) for h in range(wl.H)]
    idx = torch.zeros((4, wl.H), dtype=torch.int32, device="cuda")
    idx[1, 2] = wl.primes[2]          # one past the end
    m = torch.empty((4, wl.d_m), dtype=torch.bfloat16, device="cuda")
    E.engram_gather(plan, idx, tables, m)
    assert E.engram_device_status(clear=True) & E.ENGRAM_STATUS_BAD_ROW
    mh = to_host_u16(m).reshape(4, wl.H, wl.d_e)
    assert (mh[1, 2] == 0).all() and not (mh[0, 2] == 0).all()
    assert E.engram_device_status(clear=True) == 0
    # the bulk-copy gather (ENGRAM_FLAG_BULK_GATHER, 2,560-column rows): a row beyond the table
    # is written as zeros and flagged, the other rows land
    wb = small_workload(B=1, T=16, K=1, d_e=2560)
    pb = E.Plan.from_workload(wb, flags=E.ENGRAM_FLAG_BULK_GATHER)
    tb = [to_dev(synth.fill_bf16(wb.table_spec(h), (wb.primes[h], wb.d_e))) for h in range(wb.H)]
    ib = torch.zeros((5, wb.H), dtype=torch.int32, device="cuda")
    ib[3, 1] = wb.primes[1] + 7
    ib[2, 0] = 5
    mb = torch.full((5, wb.d_m), 3.0, dtype=torch.bfloat16, device="cuda")
    E.engram_gather(pb, ib, tb, mb)
    assert E.engram_device_status(clear=True) & E.ENGRAM_STATUS_BAD_ROW
    mbh = to_host_u16(mb).reshape(5, wb.H, wb.d_e)
    assert (mbh[3, 1] == 0).all()
    assert np.array_equal(mbh[2, 0], synth.fill_rows_bf16(wb.table_spec(0), wb.d_e, np.array([5]))[0])
    assert np.array_equal(mbh[4, 1], synth.fill_rows_bf16(wb.table_spec(1), wb.d_e, np.array([0]))[0])
    assert E.engram_device_status(clear=True) == 0


# ------------------------------------------------------------------ steps 1-6
def _oracle_full(wl, di):
    w = di.host_weights()
    tables = host_tables(wl)
    h = synth.fill_bf16(wl.h_spec(0), (wl.n_tok, wl.d_h))
    kw = dict(table_scales=table_scales(wl))
    if wl.decode:
        kw.update(history=wl.history(), conv_state=to_host_u16(di.conv_state), decode_outputs=True)
    return oracle.forward(di.ids_np, di.remap_np, tables, h, w["Wk"], w["Wv"], w["gamma_q"],
                          w["gamma_k"], w["gamma_c"], w["conv_w"], orders=wl.orders, K=wl.K,
                          primes=wl.primes, seed=wl.hash_seed, pad_id=wl.pad_id, eps=wl.eps, **kw)


PARITY_CASES = {
    # name: workload (n_tok spans several 128-token tiles with a ragged tail where noted)
    "tiny": synth.get_workload("tiny"),
    "ragged_k_bn64": small_workload("ragged_k", B=3, T=333, K=3, d_e=40, d_h=384),     # d_m=240
    "bn128": small_workload("bn128", B=2, T=4777, K=2, d_e=24, d_h=384),               # 9554 tok
    # BN = 256 tiles; d_e = 24: most 64-column k-blocks straddle two or three tables
    "bn256": small_workload("bn256", B=5, T=1901, K=2, d_e=24, d_h=512),               # 9505 tok
    "seq_edges": small_workload("fseq", B=40, T=200, K=2, d_e=16, d_h=256),            # starts inside tiles
    "short_seqs": small_workload("fshort", B=800, T=10, K=2, d_e=16, d_h=256),         # T < conv halo + 1
    "bn256_d2560": small_workload("bn256u", B=4, T=500, K=2, d_e=32, d_h=2560),        # 2000 tok
    "seq_shorter_than_halo": small_workload("short", B=40, T=7, K=2, d_e=16, d_h=128),
    # gate kernel over several channel slices, two sequences with ragged 48-token chunks
    "gate_3_slices": small_workload("g3s", B=2, T=301, K=2, d_e=24, d_h=1536),
    # streaming gate kernel with 72-token CTAs (the longer walks serve the bench workloads;
    # 36- and 9-token CTAs serve the small cases above); 6000 = 83 x 72 + 24: ragged last CTA
    "gate_walk72": small_workload("gw72", B=4, T=6000, K=2, d_e=16, d_h=256),
    # decode-sized batches: the projection splits K across CTAs (partial accumulators + reduce)
    "splitk_64tok": small_workload("splitk64", B=64, T=1, K=1, d_e=512, d_h=512),          # 4 splits
    "splitk_ragged_k": small_workload("splitk200", B=100, T=2, K=1, d_e=360, d_h=512),     # d_m=720, 3 splits
    # the 20M-row layer's widths (d_e = 2560, d_m = 5120, d_h = 2560) on 210 tokens: split-K
    # over two 128-token tiles, the second ragged
    "splitk_d2560": small_workload("splitk2560", B=3, T=70, K=1, d_e=2560, d_h=2560),
}


@pytest.mark.parametrize("case", list(PARITY_CASES))
def test_forward_matches_oracle(case):
    wl = PARITY_CASES[case]
    di = DeviceInputs(wl).forward()
    torch.cuda.synchronize()
    ref = _oracle_full(wl, di)
    assert_delta_close(di.delta.cpu().numpy(), ref["delta"])
    assert_out_close(to_host_u16(di.out), ref["out"])
    assert E.engram_device_status(clear=True) == 0


PAIR_CASES = {
    "bn256": PARITY_CASES["bn256"],                  # d_h 512: 4 channel slices, 38 x 4 units
    "gate_walk72": PARITY_CASES["gate_walk72"],      # d_h 256, 24,000 tokens
    # the 20M-row layer's widths: d_e = 2560 (40 k-blocks per table), d_m = 5120, d_h = 2560;
    # 9,003 tokens: the last tile's odd CTA holds no token
    "d2560": small_workload("pair_2560", B=3, T=3001, K=1, d_e=2560, d_h=2560),
    "bn256_d64": small_workload("pair_256", B=48, T=211, K=2, d_e=64, d_h=512),
    # three branches: key slices of three W_k, then the value slices
    "branches3": small_workload("pair_b3", B=3, T=3001, K=1, d_e=64, d_h=512, branches=3),
    "d2560_b2": small_workload("pair_2560b", B=2, T=4500, K=1, d_e=2560, d_h=2560, branches=2),
}


@pytest.mark.parametrize("packed", [False, True])
@pytest.mark.parametrize("case", list(PAIR_CASES))
def test_pair_mma_bit_identical_to_single_cta(case, packed):
    """The projection on CTA pairs (cta_group::2 MMAs, 256 x 256 units) computes exactly what
    the single-CTA kernel computes: Delta, out (and so v and the gate partial sums) bit for
    bit, with row-major weights and with the packed weight tiles (each CTA loading its 128-row
    half)."""
    wl = PAIR_CASES[case]
    a = DeviceInputs(wl, random_gammas=True)
    assert E.engram_forward_path(a.plan, wl.B, wl.T) & E.ENGRAM_PATH_PAIR_MMA
    b = DeviceInputs(wl, tables=a.tables, flags=E.ENGRAM_FLAG_SINGLE_CTA_MMA, random_gammas=True)
    assert not E.engram_forward_path(b.plan, wl.B, wl.T) & E.ENGRAM_PATH_PAIR_MMA
    if packed:
        for d in (a, b):
            d.weights = E.Weights(d.w_k, d.w_v, d.gamma_q, d.gamma_k, d.gamma_c, d.conv_w,
                                  packed=E.pack_weights(d.plan, d.w_k, d.w_v))
    a.forward()
    b.forward()
    torch.cuda.synchronize()
    assert torch.equal(a.delta, b.delta)
    assert torch.equal(a.out.view(torch.int16), b.out.view(torch.int16))
    assert E.engram_device_status(clear=True) == 0


ROW_ORDER_CASES = {
    # 24,000 tokens x 4 tables of ~1,000 rows: most rows repeat many times
    "walk72": PARITY_CASES["gate_walk72"],
    # the 16-table layer's widths (d_e = 160: 20 chunks per row), ~100,000-row tables: 3,126
    # buckets per table; 4,200 tokens = 67,200 rows, just above the row-order threshold
    "h16_d160": small_workload("ro16", B=2, T=2100, K=8, d_e=160, d_h=256,
                               primes=tuple(synth.largest_prime_below(100003 + 40 * h) for h in range(16))),
    # e4m3 tables with their per-table scales
    "fp8": small_workload("ro8", B=2, T=9000, K=2, d_e=32, d_h=256, table_dtype="fp8"),
    # the 20M-row layer's row width (d_e = 2560, 320 chunks per row), two tables
    "d2560": small_workload("ro2560", B=2, T=16500, K=1, d_e=2560, d_h=256, primes=(100003, 100019)),
}


@pytest.mark.parametrize("case", list(ROW_ORDER_CASES))
def test_row_order_gather_bit_identical_to_token_order(case):
    """In-batch dedup of the HBM reads: the gather walking the batch's rows grouped by row id
    (ENGRAM_PATH_ROW_ORDER) gives the same m as the gather in token order, hence the same
    Delta and out bit for bit."""
    wl = ROW_ORDER_CASES[case]
    a = DeviceInputs(wl, flags=E.ENGRAM_FLAG_ROW_ORDER_GATHER, random_gammas=True)
    assert E.engram_forward_path(a.plan, wl.B, wl.T) & E.ENGRAM_PATH_ROW_ORDER
    b = DeviceInputs(wl, tables=a.tables, random_gammas=True)
    assert not E.engram_forward_path(b.plan, wl.B, wl.T) & E.ENGRAM_PATH_ROW_ORDER
    for _ in range(2):   # the list is rebuilt on every call
        a.forward()
        b.forward()
        torch.cuda.synchronize()
        assert torch.equal(a.delta, b.delta)
        assert torch.equal(a.out.view(torch.int16), b.out.view(torch.int16))
    assert E.engram_device_status(clear=True) == 0


@pytest.mark.parametrize("B,d_h", [(256, 2560), (96, 512)])
def test_pair_split_k_decode_bit_identical_to_single_cta(B, d_h):
    """One-token decode steps whose projection splits K: on CTA pairs (256-token units, each
    weight tile read by one pair) the partial accumulators, and so Delta, out, the conv state
    and the hash history, equal the single-CTA kernel's bit for bit when both split K the same
    number of ways."""
    wl = small_workload("pair_dec", B=B, T=1, K=1, d_e=d_h, d_h=d_h, decode=True)
    a = DeviceInputs(wl, random_gammas=True)
    b = DeviceInputs(wl, tables=a.tables, flags=E.ENGRAM_FLAG_SINGLE_CTA_MMA, random_gammas=True)
    pa, pb = E.engram_forward_path(a.plan, wl.B, 1), E.engram_forward_path(b.plan, wl.B, 1)
    assert pa & E.ENGRAM_PATH_PAIR_MMA and pa & E.ENGRAM_PATH_SPLIT_K
    assert not pb & E.ENGRAM_PATH_PAIR_MMA and pb & E.ENGRAM_PATH_SPLIT_K
    for step in range(3):
        ids = to_dev(synth.zipf_ids(wl.vocab_in, 1.1, (wl.B, 1), 700 + step))
        a.ids = b.ids = ids
        a.forward()
        b.forward()
        torch.cuda.synchronize()
        assert torch.equal(a.delta, b.delta)
        assert torch.equal(a.out.view(torch.int16), b.out.view(torch.int16))
        assert torch.equal(a.conv_state.view(torch.int16), b.conv_state.view(torch.int16))
        assert torch.equal(a.history, b.history)
    assert E.engram_device_status(clear=True) == 0


def test_kernel_launch_count_per_call():
    """The library's launch counter (bench.py's gpu_launches): a prefill call launches remap +
    hash, gather, projection, gate scalars and the streaming gate kernel (5); a one-token
    split-K decode step with hash history and conv state launches the lookup, the projection
    and the fused reduce + gate + conv + history kernel (3); the same call twice counts the
    same; a call rejected on the host counts nothing."""
    wl = PARITY_CASES["bn128"]                  # 9,554 tokens x 4 tables: the separate hash and gather
    di = DeviceInputs(wl).forward()
    torch.cuda.synchronize()
    n0 = E.kernel_launches()
    di.forward()
    n1 = E.kernel_launches()
    di.forward()
    n2 = E.kernel_launches()
    assert n1 - n0 == 5 and n2 - n1 == 5
    with pytest.raises(E.EngramError):
        E.engram_forward(di.plan, di.weights, di.tables, di.ids, di.h, di.out, di.ws[:16])   # workspace too small
    assert E.kernel_launches() == n2
    dec = small_workload("dec_split", B=32, T=1, K=1, d_e=512, d_h=512, decode=True)
    dd = DeviceInputs(dec)
    assert E.engram_forward_path(dd.plan, dec.B, 1) & (E.ENGRAM_PATH_FUSED_LOOKUP | E.ENGRAM_PATH_SPLIT_K) == (
        E.ENGRAM_PATH_FUSED_LOOKUP | E.ENGRAM_PATH_SPLIT_K)
    dd.forward()
    torch.cuda.synchronize()
    n0 = E.kernel_launches()
    dd.forward()
    dd.forward()
    assert E.kernel_launches() - n0 == 6


@pytest.mark.parametrize("case", ["ragged_k_bn64", "bn256_d2560", "splitk_64tok", "seq_edges"])
def test_forward_with_non_unit_gains(case):
    wl = PARITY_CASES[case]
    di = DeviceInputs(wl, random_gammas=True).forward()
    torch.cuda.synchronize()
    ref = _oracle_full(wl, di)
    assert_delta_close(di.delta.cpu().numpy(), ref["delta"])
    assert_out_close(to_host_u16(di.out), ref["out"])


def test_gate_conv_entry_matches_forward():
    wl = PARITY_CASES["ragged_k_bn64"]
    di = DeviceInputs(wl).forward()
    out_fwd = di.out.clone()
    idx_np = _idx_oracle(wl, di.ids_np)
    m = torch.empty((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
    E.engram_gather(di.plan, to_dev(idx_np.view(np.int32)), di.tables, m)
    out2 = torch.empty_like(di.out)
    E.engram_gate_conv(di.plan, di.weights, di.h, m, wl.B, wl.T, out2, di.ws)
    assert torch.equal(out_fwd.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("geom", ["small", "splitk", "splitk_256seq", "splitk_d2560", "splitk_d384", "chunk4"])
def test_decode_steps_match_oracle_and_update_state(geom):
    """Consecutive calls carrying the hash history and conv state: one token per call
    (one-token decode kernels, with and without split-K, over one and two 128-token tiles,
    also at the 20M-row layer's widths) and four tokens per call (the chain kernel reading
    and rewriting the carried state)."""
    if geom == "small":
        wl = small_workload("dec", B=6, T=1, K=2, d_e=32, d_h=256, decode=True)
    elif geom == "splitk":
        wl = small_workload("dec_split", B=32, T=1, K=1, d_e=512, d_h=512, decode=True)
    elif geom == "splitk_256seq":
        wl = small_workload("dec_256", B=256, T=1, K=1, d_e=512, d_h=512, decode=True)
    elif geom == "splitk_d384":   # split K, d_h not a multiple of 256: split reduce + decode gate kernels
        wl = small_workload("dec_384", B=64, T=1, K=1, d_e=512, d_h=384, decode=True)
    elif geom == "splitk_d2560":
        wl = small_workload("dec_2560", B=200, T=1, K=1, d_e=2560, d_h=2560, decode=True)
    else:
        wl = small_workload("dec_chunk", B=5, T=4, K=2, d_e=32, d_h=256, decode=True)
    di = DeviceInputs(wl, random_gammas=geom != "small")
    w = di.host_weights()
    tables = [synth.fill_bf16(wl.table_spec(h), (wl.primes[h], wl.d_e)) for h in range(wl.H)]
    hist = wl.history()
    state = to_host_u16(di.conv_state)
    for step in range(3 if geom == "splitk_d2560" else 12):
        ids_np = synth.zipf_ids(wl.vocab_in, 1.1, (wl.B, wl.T), 500 + step)
        h_np = synth.fill_bf16(wl.h_spec(step), (wl.B * wl.T, wl.d_h))
        di.ids = to_dev(ids_np)
        di.h = to_dev(h_np)
        di.forward()
        ref = oracle.forward(ids_np, di.remap_np, tables, h_np, w["Wk"], w["Wv"], w["gamma_q"], w["gamma_k"],
                             w["gamma_c"], w["conv_w"], orders=wl.orders, K=wl.K, primes=wl.primes,
                             seed=wl.hash_seed, pad_id=wl.pad_id, eps=wl.eps, history=hist,
                             conv_state=state, decode_outputs=True)
        torch.cuda.synchronize()
        assert_delta_close(di.delta.cpu().numpy(), ref["delta"])
        assert_out_close(to_host_u16(di.out), ref["out"])
        assert np.array_equal(di.history.cpu().numpy(), ref["history"])
        # the new slot is bf16(u) on both sides: each value within one bf16 ulp of the oracle's
        assert_bf16_within_ulp(to_host_u16(di.conv_state), ref["state"])
        hist, state = ref["history"], to_host_u16(di.conv_state)


@pytest.mark.parametrize("geom", ["fused_d2560", "decode_kernel_d384"])
def test_gate_conv_decode_steps_queued_back_to_back(geom):
    """engram_gate_conv decode steps queued on one stream with nothing between them, the conv
    state carried from call to call: every step's output and the final state equal those of
    the same steps run one at a time.  (The decode kernels read and shift the carried state
    before they wait for the projection, so a call's first kernel must not overlap the
    previous call's last one.)"""
    if geom == "fused_d2560":   # split-K projection + decode_fused_kernel
        wl = small_workload("dec_q2560", B=200, T=1, K=1, d_e=2560, d_h=2560, decode=True)
    else:                       # split-K reduce + gate_conv_decode_kernel
        wl = small_workload("dec_q384", B=64, T=1, K=1, d_e=512, d_h=384, decode=True)
    di = DeviceInputs(wl, random_gammas=True)
    steps = 6
    ms, hs = [], []
    for step in range(steps):
        ids_np = synth.zipf_ids(wl.vocab_in, 1.1, (wl.B, wl.T), 900 + step)
        idx = _idx_oracle(wl, ids_np)
        m = torch.empty((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
        E.engram_gather(di.plan, to_dev(idx.view(np.int32)), di.tables, m)
        ms.append(m)
        hs.append(to_dev(synth.fill_bf16(wl.h_spec(step), (wl.B * wl.T, wl.d_h))))
    state0 = di.conv_state.clone()
    torch.cuda.synchronize()

    def run(sync_each):
        state = state0.clone()
        outs = [torch.empty_like(di.out) for _ in range(steps)]
        torch.cuda.synchronize()
        for k in range(steps):
            E.engram_gate_conv(di.plan, di.weights, hs[k], ms[k], wl.B, wl.T, outs[k], di.ws, conv_state=state)
            if sync_each:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return outs, state

    outs_a, state_a = run(True)
    outs_b, state_b = run(False)
    for k in range(steps):
        assert torch.equal(outs_a[k].view(torch.int16), outs_b[k].view(torch.int16)), k
    assert torch.equal(state_a.view(torch.int16), state_b.view(torch.int16))
    assert E.engram_device_status(clear=True) == 0


def _window_oracle(wl, di, w, b, t):
    """Oracle for token (b, t) on a window of at most 1 + state_len tokens, with the rows it
    needs regenerated from the seeded generator (the tables are never materialised)."""
    S = wl.state_len
    w0 = max(0, t - S)
    ids = di.ids_np[b:b + 1, w0:t + 1]
    remap = di.remap_np
    xr_full = remap[di.ids_np[b]]
    hist = np.array([[xr_full[p] if p >= 0 else wl.pad_id for p in (w0 - 2, w0 - 1)]], dtype=np.int32)
    xr = remap[ids]
    idx = oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id, history=hist)
    W = idx.shape[0]
    tables = [synth.fill_rows_bf16(wl.table_spec(h), wl.d_e, idx[:, h]) for h in range(wl.H)]
    m = oracle.gather(np.tile(np.arange(W, dtype=np.uint32)[:, None], (1, wl.H)), tables)
    rows = np.arange(b * wl.T + w0, b * wl.T + t + 1)
    h = synth.fill_rows_bf16(wl.h_spec(0), wl.d_h, rows)
    r = oracle.gate_conv(h, m, w["Wk"], w["Wv"], w["gamma_q"], w["gamma_k"], w["gamma_c"], w["conv_w"],
                         1, W, dil=wl.conv_dilation, eps=wl.eps)
    return r["delta"][-1], r["out"][-1]


@pytest.mark.slow
def test_forward_full_size_layer2560_sampled():
    """The full 8x4096 workload in the benchmark's launch configuration, checked on sampled
    tokens (sequence starts, tile edges, random) that the oracle computes one by one."""
    wl = synth.get_workload("layer2560")
    di = DeviceInputs(wl).forward()
    torch.cuda.synchronize()
    w = {k: v for k, v in di.host_weights().items()}
    rng = np.random.default_rng(8)
    picks = [(0, 0), (0, 1), (0, 2), (0, 9), (1, 0), (7, wl.T - 1), (3, 127), (3, 128), (5, 4095)]
    picks += [(int(rng.integers(0, wl.B)), int(rng.integers(0, wl.T))) for _ in range(15)]
    got_d = di.delta.cpu().numpy()
    got_o = to_host_u16(di.out)
    ds, rs, os_, ros = [], [], [], []
    for b, t in picks:
        d_ref, o_ref = _window_oracle(wl, di, w, b, t)
        n = b * wl.T + t
        ds.append(got_d[n]); rs.append(d_ref); os_.append(got_o[n]); ros.append(o_ref)
    assert_delta_close(np.stack(ds), np.stack(rs))
    assert_out_close(np.stack(os_), np.stack(ros))


def test_forward_replays_identically_in_a_cuda_graph():
    """After one eager call on the device, engram_forward can be captured in a CUDA graph;
    replays give the eager result bit for bit."""
    wl = PARITY_CASES["ragged_k_bn64"]
    di = DeviceInputs(wl).forward(delta=False)
    torch.cuda.synchronize()
    eager = di.out.clone()
    di.out.zero_()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
        E.engram_forward(di.plan, di.weights, di.tables, di.ids, di.h, di.out, di.ws, remap=di.remap,
                         stream=torch.cuda.current_stream())
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(2):
        di.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(di.out.view(torch.int16), eager.view(torch.int16))


def _free_device():
    import gc
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_decode_step_on_full_95gib_tables_sampled():
    """One decode step of 256 sequences on the full 2 x 9,999,991 x 2560 tables (row byte
    offsets far above 2^32), checked on sampled sequences with their rows regenerated."""
    wl = synth.get_workload("decode20m")
    free, _ = torch.cuda.mem_get_info()
    if free < wl.table_bytes + (4 << 30):
        pytest.skip("not enough device memory for the 95.4 GiB tables")
    try:
        di = DeviceInputs(wl)
        state_before = to_host_u16(di.conv_state)
        hist_before = di.history.cpu().numpy()
        di.forward()
        torch.cuda.synchronize()
        w = di.host_weights()
        rng = np.random.default_rng(21)
        seqs = np.sort(rng.choice(wl.B, 12, replace=False))
        ids = di.ids_np[seqs]
        idx = oracle.hash_ids(ids, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id, history=hist_before[seqs])
        assert idx.max() > (1 << 32) // (wl.d_e * 2)          # rows past the 4 GiB offset boundary
        tables = [synth.fill_rows_bf16(wl.table_spec(h), wl.d_e, idx[:, h]) for h in range(wl.H)]
        m = oracle.gather(np.tile(np.arange(len(seqs), dtype=np.uint32)[:, None], (1, wl.H)), tables)
        h_rows = synth.fill_rows_bf16(wl.h_spec(0), wl.d_h, seqs)
        ref = oracle.gate_conv(h_rows, m, w["Wk"], w["Wv"], w["gamma_q"], w["gamma_k"], w["gamma_c"],
                               w["conv_w"], len(seqs), 1, dil=wl.conv_dilation, eps=wl.eps,
                               conv_state=state_before[seqs], want_state=True)
        assert_delta_close(di.delta.cpu().numpy()[seqs], ref["delta"])
        assert_out_close(to_host_u16(di.out)[seqs], ref["out"])
    finally:
        di = None
        _free_device()


@pytest.mark.slow
def test_forward_on_16x20m_tables_sampled_rows():
    """The pages' own geometry (16 tables x 19,999,999 rows x 160, ~102 GB): the gathered
    memory vectors on sampled tokens equal the regenerated rows bit for bit."""
    wl = synth.get_workload("ngram16x20m")
    free, _ = torch.cuda.mem_get_info()
    if free < wl.table_bytes + (4 << 30):
        pytest.skip("not enough device memory for the 102 GB tables")
    try:
        plan = E.Plan.from_workload(wl)
        tables = [fill_gpu.filled((wl.primes[h], wl.d_e), wl.table_spec(h)) for h in range(wl.H)]
        ids = wl.ids()
        idx_np = _idx_oracle(wl, ids)
        m = torch.empty((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
        E.engram_gather(plan, to_dev(idx_np.view(np.int32)), tables, m)
        rng = np.random.default_rng(6)
        sample = np.concatenate([[0, wl.n_tok - 1], rng.integers(0, wl.n_tok, 120)])
        got = to_host_u16(m[torch.from_numpy(sample).cuda()]).reshape(len(sample), wl.H, wl.d_e)
        for h in range(wl.H):
            assert np.array_equal(got[:, h, :], synth.fill_rows_bf16(wl.table_spec(h), wl.d_e, idx_np[sample, h]))
    finally:
        tables = m = None
        _free_device()


@pytest.mark.slow
def test_prefill_on_full_95gib_tables_sampled():
    """32 x 8192 tokens (30% copied phrases) on the full 2 x 9,999,991 x 2560 tables, in the
    benchmark's launch configuration, checked on sampled tokens (sequence starts, the edges of
    128-token tiles and 144-token gate chunks, random) that the oracle computes one by one."""
    wl = synth.get_workload("prefill20m")
    free, _ = torch.cuda.mem_get_info()
    if free < wl.table_bytes + (12 << 30):
        pytest.skip("not enough device memory for the 95.4 GiB tables and the 262,144-token batch")
    di = None
    try:
        di = DeviceInputs(wl).forward()
        torch.cuda.synchronize()
        w = di.host_weights()
        rng = np.random.default_rng(31)
        picks = [(0, 0), (0, 1), (0, 8), (0, 9), (5, 127), (5, 128), (9, 143), (9, 144), (31, wl.T - 1)]
        picks += [(int(rng.integers(0, wl.B)), int(rng.integers(0, wl.T))) for _ in range(12)]
        got_d, got_o = [], []
        ref_d, ref_o = [], []
        for b, t in picks:
            n = b * wl.T + t
            d_ref, o_ref = _window_oracle(wl, di, w, b, t)
            got_d.append(di.delta[n].cpu().numpy())
            got_o.append(to_host_u16(di.out[n]))
            ref_d.append(d_ref)
            ref_o.append(o_ref)
        assert_delta_close(np.stack(got_d), np.stack(ref_d))
        assert_out_close(np.stack(got_o), np.stack(ref_o))
        assert E.engram_device_status(clear=True) == 0
    finally:
        di = None
        _free_device()


@pytest.mark.slow
def test_decode_step_on_full_host_pinned_tables_sampled():
    """One decode step of 64 sequences with the full 102 GB tables in pinned, mapped host
    memory (distinct rows staged through HBM), checked on sampled sequences against the
    oracle with the rows regenerated."""
    import psutil
    wl = synth.get_workload("hostpinned20m")
    if psutil.virtual_memory().available < wl.table_bytes + (16 << 30):
        pytest.skip("not enough host memory for 102 GB of pinned tables")
    bufs = []
    try:
        for h in range(wl.H):
            hm = fill_gpu.HostMapped(wl.primes[h], wl.d_e)
            fill_gpu.fill_(hm.tensor, wl.table_spec(h))
            bufs.append(hm)
        torch.cuda.synchronize()
        di = DeviceInputs(wl, tables=[b.tensor for b in bufs])
        di.plan = E.Plan.from_workload(wl, host_tables=True)
        di.ws = E.alloc_workspace(di.plan, wl.n_tok)
        state_before = to_host_u16(di.conv_state)
        hist_before = di.history.cpu().numpy()
        di.forward()
        torch.cuda.synchronize()
        w = di.host_weights()
        seqs = np.sort(np.random.default_rng(41).choice(wl.B, 10, replace=False))
        ids = di.ids_np[seqs]
        idx = oracle.hash_ids(ids, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id, history=hist_before[seqs])
        tables = [synth.fill_rows_bf16(wl.table_spec(h), wl.d_e, idx[:, h]) for h in range(wl.H)]
        m = oracle.gather(np.tile(np.arange(len(seqs), dtype=np.uint32)[:, None], (1, wl.H)), tables)
        h_rows = synth.fill_rows_bf16(wl.h_spec(0), wl.d_h, seqs)
        ref = oracle.gate_conv(h_rows, m, w["Wk"], w["Wv"], w["gamma_q"], w["gamma_k"], w["gamma_c"],
                               w["conv_w"], len(seqs), 1, dil=wl.conv_dilation, eps=wl.eps,
                               conv_state=state_before[seqs], want_state=True)
        assert_delta_close(di.delta.cpu().numpy()[seqs], ref["delta"])
        assert_out_close(to_host_u16(di.out)[seqs], ref["out"])
        assert E.engram_device_status(clear=True) == 0
    finally:
        di = None
        for b in bufs:
            b.close()
        _free_device()
