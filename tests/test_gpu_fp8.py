"""FP8 (e4m3) tables on the GPU, against the oracle.

Bit-exact: the GPU e4m3 generator, and every gathered value (the bf16 nearest to
decode(code) * scale_h, one rounding of the exact product) on every path that reads a table:
the wide gather, the fused remap+hash+gather kernel of decode-sized batches, and host-mapped
tables staged through HBM.  The layer output keeps the tolerances of the bf16 tables.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hashed_gram_embedding_remap_b200 as E
import oracle
import synth
from gpu_helpers import (DeviceInputs, assert_delta_close, assert_out_close, host_rows, host_tables, table_scales,
                         to_dev, to_host_u16)
from helpers import small_workload
from synth import fill_gpu

pytestmark = pytest.mark.gpu


def _u8_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def _idx_oracle(wl, ids_np, history=None):
    xr = wl.remap()[ids_np]
    return oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id, history=history)


def _same_bits_or_both_nan(got: np.ndarray, ref: np.ndarray):
    gn = np.isnan(synth.bf16_to_float(got))
    rn = np.isnan(synth.bf16_to_float(ref))
    assert np.array_equal(gn, rn)
    assert np.array_equal(got[~rn], ref[~rn])


def test_gpu_fp8_fill_matches_cpu_codes():
    spec = synth.FillSpec(77, 9, 1.0)
    n = 123457                                 # not a multiple of 16: the tail path too
    got = fill_gpu.filled_fp8((n,), spec).cpu().numpy()
    assert np.array_equal(got, synth.fill_fp8(spec, (n,)))


def _midpoint_scales(count: int, seed: int = 5):
    """Scales for which some code's binary32 product -- rounded to nearest, or truncated --
    lands exactly on a bf16 midpoint while the exact product does not: the cases where a
    plain fp32 multiply then round, or a truncation without its sticky bit, is one ulp off."""
    rng = np.random.default_rng(seed)
    v = np.array([oracle.e4m3_to_double(c) for c in range(1, 0x7F)])
    out = []
    while len(out) < count:
        s = rng.uniform(0.001, 0.05, 20000).astype(np.float32)
        prod = v[:, None] * s.astype(np.float64)[None, :]        # exact
        rn = prod.astype(np.float32)
        rz = np.where(np.abs(rn.astype(np.float64)) > np.abs(prod), np.nextafter(rn, np.float32(0)), rn)
        inexact = rn.astype(np.float64) != prod
        hit = inexact & (((rn.view(np.uint32) & 0xFFFF) == 0x8000) | ((rz.view(np.uint32) & 0xFFFF) == 0x8000))
        cols = np.unique(np.nonzero(hit)[1])
        out.extend(float(s[c]) for c in cols[: count - len(out)])
    return out


@pytest.mark.parametrize("K,d_e", [(4, 32), (1, 2560)])
def test_gather_every_code_and_midpoint_scales_bit_exact(K, d_e):
    """Tables whose first rows hold all 256 codes (NaN codes included) with per-table scales
    that hit the double-rounding case; gathered rows equal the oracle's bit for bit (NaN codes:
    both NaN)."""
    base = small_workload("fp8g", B=3, T=200, K=K, d_e=d_e, d_h=256, table_dtype="fp8")
    scales = _midpoint_scales(base.H)
    plan = E.Plan(orders=base.orders, heads_per_order=K, table_rows=base.primes, row_dim=d_e,
                  hidden_dim=base.d_h, vocab_in=base.vocab_in, vocab_out=base.vocab_out,
                  hash_seed=base.hash_seed, table_dtype=E.ENGRAM_TABLE_FP8_E4M3, table_scale=scales)
    rng = np.random.default_rng(8)
    tabs = []
    for h in range(base.H):
        t = rng.integers(0, 256, size=(base.primes[h], d_e), dtype=np.uint8)
        t.reshape(-1)[:256] = np.arange(256, dtype=np.uint8)
        tabs.append(t)
    idx_np = _idx_oracle(base, base.ids())
    idx_np[: (256 + d_e - 1) // d_e] = np.arange((256 + d_e - 1) // d_e, dtype=np.uint32)[:, None]
    m = torch.empty((base.n_tok, base.d_m), dtype=torch.bfloat16, device="cuda")
    E.engram_gather(plan, to_dev(idx_np.view(np.int32)), [_u8_dev(t) for t in tabs], m)
    torch.cuda.synchronize()
    _same_bits_or_both_nan(to_host_u16(m), oracle.gather(idx_np, tabs, [np.float32(s) for s in scales]))
    assert E.engram_device_status(clear=True) == 0


FP8_CASES = {
    # 512 tokens x 4 tables: remap + hash + gather fused (one warp per row)
    "lookup_tiny": synth.get_workload("tiny").with_(table_dtype="fp8"),
    # 5,000 tokens x 4 tables: hash kernel, then the wide gather
    "gather_wide": small_workload("fp8w", B=2, T=2500, K=2, d_e=32, d_h=384, table_dtype="fp8"),
    # 2,560-wide rows, split-K projection
    "wide_rows": small_workload("fp8r", B=48, T=1, K=1, d_e=2560, d_h=512, table_dtype="fp8"),
}


@pytest.mark.parametrize("case", list(FP8_CASES))
def test_forward_fp8_tables_matches_oracle(case):
    wl = FP8_CASES[case]
    di = DeviceInputs(wl).forward()
    torch.cuda.synchronize()
    w = di.host_weights()
    ref = oracle.forward(di.ids_np, di.remap_np, host_tables(wl), synth.fill_bf16(wl.h_spec(0), (wl.n_tok, wl.d_h)),
                         w["Wk"], w["Wv"], w["gamma_q"], w["gamma_k"], w["gamma_c"], w["conv_w"],
                         orders=wl.orders, K=wl.K, primes=wl.primes, seed=wl.hash_seed, pad_id=wl.pad_id,
                         eps=wl.eps, table_scales=table_scales(wl))
    assert_delta_close(di.delta.cpu().numpy(), ref["delta"])
    assert_out_close(to_host_u16(di.out), ref["out"])
    assert E.engram_device_status(clear=True) == 0


def test_fp8_decode_steps_carry_state():
    wl = small_workload("fp8dec", B=6, T=1, K=2, d_e=32, d_h=256, decode=True, table_dtype="fp8")
    di = DeviceInputs(wl)
    w = di.host_weights()
    tables = host_tables(wl)
    hist, state = wl.history(), to_host_u16(di.conv_state)
    for step in range(6):
        ids_np = synth.zipf_ids(wl.vocab_in, 1.1, (wl.B, wl.T), 700 + step)
        h_np = synth.fill_bf16(wl.h_spec(step), (wl.B * wl.T, wl.d_h))
        di.ids, di.h = to_dev(ids_np), to_dev(h_np)
        di.forward()
        ref = oracle.forward(ids_np, di.remap_np, tables, h_np, w["Wk"], w["Wv"], w["gamma_q"], w["gamma_k"],
                             w["gamma_c"], w["conv_w"], orders=wl.orders, K=wl.K, primes=wl.primes,
                             seed=wl.hash_seed, pad_id=wl.pad_id, eps=wl.eps, history=hist, conv_state=state,
                             decode_outputs=True, table_scales=table_scales(wl))
        torch.cuda.synchronize()
        assert_delta_close(di.delta.cpu().numpy(), ref["delta"])
        assert_out_close(to_host_u16(di.out), ref["out"])
        assert np.array_equal(di.history.cpu().numpy(), ref["history"])
        hist, state = ref["history"], to_host_u16(di.conv_state)


@pytest.mark.parametrize("B,T", [(64, 1), (3, 3000)])   # staged (<= 8192 tokens) and direct zero-copy
def test_fp8_host_tables_bit_identical_to_device_tables(B, T):
    wl = small_workload("fp8pin", B=B, T=T, K=1, d_e=256, d_h=256, primes=(100003, 100019), table_dtype="fp8")
    dev = DeviceInputs(wl).forward(delta=False)
    torch.cuda.synchronize()
    bufs = []
    for h in range(wl.H):
        hm = fill_gpu.HostMapped(wl.primes[h], wl.d_e, elem_bytes=1)
        fill_gpu.fill_fp8_(hm.tensor, wl.table_spec(h))
        bufs.append(hm)
    torch.cuda.synchronize()
    plan_h = E.Plan.from_workload(wl, host_tables=True)
    out_h = torch.empty_like(dev.out)
    ws = E.alloc_workspace(plan_h, wl.n_tok)
    E.engram_forward(plan_h, dev.weights, [b.tensor for b in bufs], dev.ids, dev.h, out_h, ws, remap=dev.remap)
    torch.cuda.synchronize()
    assert torch.equal(out_h.view(torch.int16), dev.out.view(torch.int16))
    assert E.engram_device_status(clear=True) == 0
    for b in bufs:
        b.close()


def test_fp8_stage_rows_copies_codes_unchanged():
    wl = small_workload("fp8stage", B=4, T=300, K=3, d_e=48, d_h=128, ids_kind="zipf", zipf_s=1.3,
                        table_dtype="fp8")
    plan = E.Plan.from_workload(wl)
    tabs = [fill_gpu.filled_fp8((wl.primes[h], wl.d_e), wl.table_spec(h)) for h in range(wl.H)]
    idx_np = _idx_oracle(wl, wl.ids())
    n = idx_np.shape[0]
    staging = [torch.empty((n, wl.d_e), dtype=torch.uint8, device="cuda") for _ in range(wl.H)]
    sidx = torch.empty((n, wl.H), dtype=torch.int32, device="cuda")
    uniq = torch.empty((wl.H, n), dtype=torch.int32, device="cuda")
    nu = torch.empty((wl.H,), dtype=torch.int32, device="cuda")
    E.engram_stage_rows(plan, to_dev(idx_np.view(np.int32)), tabs, staging, sidx, uniq, nu)
    m = torch.empty((n, wl.d_m), dtype=torch.bfloat16, device="cuda")
    E.engram_gather(plan, sidx, staging, m, rows_bound=n)
    torch.cuda.synchronize()
    nu_h = nu.cpu().numpy()
    for h in range(wl.H):
        ref = np.unique(idx_np[:, h])
        assert nu_h[h] == ref.size
        assert np.array_equal(staging[h][: nu_h[h]].cpu().numpy(), synth.fill_rows_fp8(wl.table_spec(h), wl.d_e, ref))
    assert np.array_equal(to_host_u16(m), oracle.gather(idx_np, host_tables(wl), table_scales(wl)))


def test_binding_rejects_bf16_tensors_for_fp8_plan():
    wl = synth.get_workload("tiny").with_(table_dtype="fp8")
    plan = E.Plan.from_workload(wl)
    tabs = [torch.empty((wl.primes[h], wl.d_e), dtype=torch.bfloat16, device="cuda") for h in range(wl.H)]
    idx = torch.zeros((4, wl.H), dtype=torch.int32, device="cuda")
    m = torch.empty((4, wl.d_m), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        E.engram_gather(plan, idx, tabs, m)


@pytest.mark.slow
def test_fp8_16x20m_tables_sampled_rows():
    """The pages' geometry (16 tables x 19,999,999 rows x 160) as e4m3 (51 GB): gathered rows
    on sampled tokens equal the oracle's dequantisation of the regenerated codes."""
    wl = synth.get_workload("ngram16x20m").with_(table_dtype="fp8")
    free, _ = torch.cuda.mem_get_info()
    if free < wl.table_bytes + (4 << 30):
        pytest.skip("not enough device memory for the 51 GB tables")
    tables = m = None
    try:
        plan = E.Plan.from_workload(wl)
        tables = [fill_gpu.filled_fp8((wl.primes[h], wl.d_e), wl.table_spec(h)) for h in range(wl.H)]
        idx_np = _idx_oracle(wl, wl.ids())
        m = torch.empty((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
        E.engram_gather(plan, to_dev(idx_np.view(np.int32)), tables, m)
        rng = np.random.default_rng(9)
        sample = np.concatenate([[0, wl.n_tok - 1], rng.integers(0, wl.n_tok, 120)])
        got = to_host_u16(m[torch.from_numpy(sample).cuda()]).reshape(len(sample), wl.H, wl.d_e)
        for h in range(wl.H):
            assert np.array_equal(got[:, h, :], host_rows(wl, h, idx_np[sample, h]))
    finally:
        tables = m = None
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
