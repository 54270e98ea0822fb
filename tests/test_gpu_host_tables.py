"""Host-resident tables (pinned, mapped host memory): distinct rows are staged into HBM once
per batch and the results are bit-identical to HBM-resident tables (the pages report
bit-identical tokens and logprobs after moving the n-gram table to pinned host memory)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hashed_gram_embedding_remap_b200 as E
import oracle
import synth
from gpu_helpers import DeviceInputs, to_dev, to_host_u16
from helpers import small_workload
from synth import fill_gpu

pytestmark = pytest.mark.gpu


def _host_tables(wl):
    bufs = []
    for h in range(wl.H):
        hm = fill_gpu.HostMapped(wl.primes[h], wl.d_e)
        fill_gpu.fill_(hm.tensor, wl.table_spec(h))
        bufs.append(hm)
    torch.cuda.synchronize()
    return bufs


def test_stage_rows_dedups_and_copies_exactly():
    wl = small_workload("stage", B=4, T=300, K=3, d_e=40, d_h=128, ids_kind="zipf", zipf_s=1.3)
    plan = E.Plan.from_workload(wl)
    bufs = _host_tables(wl)
    xr = wl.remap()[wl.ids()]
    idx_np = oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    n = idx_np.shape[0]
    staging = [torch.empty((n, wl.d_e), dtype=torch.bfloat16, device="cuda") for _ in range(wl.H)]
    sidx = torch.empty((n, wl.H), dtype=torch.int32, device="cuda")
    uniq = torch.empty((wl.H, n), dtype=torch.int32, device="cuda")
    nu = torch.empty((wl.H,), dtype=torch.int32, device="cuda")
    E.engram_stage_rows(plan, to_dev(idx_np.view(np.int32)), [b.tensor for b in bufs], staging, sidx, uniq, nu)
    torch.cuda.synchronize()
    sidx_h, uniq_h, nu_h = sidx.cpu().numpy(), uniq.cpu().numpy().view(np.uint32), nu.cpu().numpy()
    for h in range(wl.H):
        ref = np.unique(idx_np[:, h])
        assert nu_h[h] == ref.size < n          # Zipf(1.3) grams repeat inside the batch
        assert np.array_equal(uniq_h[h, :nu_h[h]], ref)
        assert np.array_equal(uniq_h[h, sidx_h[:, h]], idx_np[:, h])
        rows = synth.fill_rows_bf16(wl.table_spec(h), wl.d_e, ref)
        assert np.array_equal(to_host_u16(staging[h][:nu_h[h]]), rows)
    for b in bufs:
        b.close()


@pytest.mark.parametrize("B,T", [(64, 1), (3, 3000)])   # staged (<= 8192 tokens) and direct zero-copy
def test_host_tables_bit_identical_to_device_tables(B, T):
    wl = small_workload("hostpin", B=B, T=T, K=1, d_e=256, d_h=256, primes=(100003, 100019))
    dev = DeviceInputs(wl).forward(delta=False)
    torch.cuda.synchronize()
    bufs = _host_tables(wl)
    plan_h = E.Plan.from_workload(wl, host_tables=True)
    out_h = torch.empty_like(dev.out)
    ws = E.alloc_workspace(plan_h, wl.n_tok)
    E.engram_forward(plan_h, dev.weights, [b.tensor for b in bufs], dev.ids, dev.h, out_h, ws, remap=dev.remap)
    torch.cuda.synchronize()
    assert torch.equal(out_h.view(torch.int16), dev.out.view(torch.int16))
    assert E.engram_device_status(clear=True) == 0
    for b in bufs:
        b.close()


@pytest.mark.parametrize("B,T,history", [(64, 1, True), (1, 200, False), (40, 8, True)])
def test_stage_rows_from_ids_matches_hash_then_stage(B, T, history):
    """engram_stage_rows_from_ids (one kernel up to 256 (token, table) rows: 64 x 1 with a hash
    history and 1 x 200; the hash kernel + staging kernels above it: 40 x 8) stages exactly
    what engram_hash followed by engram_stage_rows stages: row ids, slots, distinct-row lists,
    counts and the staged bytes."""
    wl = small_workload("stage_ids", B=B, T=T, K=1, d_e=64, d_h=128, primes=(1009, 1013), ids_kind="zipf",
                        zipf_s=1.3, decode=history)
    plan = E.Plan.from_workload(wl, host_tables=True)
    bufs = _host_tables(wl)
    tables = [b.tensor for b in bufs]
    ids = to_dev(wl.ids())
    remap = to_dev(wl.remap())
    hist = to_dev(wl.history()) if history else None
    n = wl.n_tok

    def buffers():
        return ([torch.full((n, wl.d_e), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(wl.H)],
                torch.full((n, wl.H), -1, dtype=torch.int32, device="cuda"),
                torch.full((n, wl.H), -1, dtype=torch.int32, device="cuda"),
                torch.full((wl.H, n), -1, dtype=torch.int32, device="cuda"),
                torch.full((wl.H,), -1, dtype=torch.int32, device="cuda"))

    st_a, idx_a, sidx_a, uq_a, nu_a = buffers()
    E.engram_stage_rows_from_ids(plan, ids, tables, st_a, idx_a, sidx_a, uq_a, nu_a, remap=remap, history=hist)
    st_b, idx_b, sidx_b, uq_b, nu_b = buffers()
    xr = torch.empty_like(ids)
    E.engram_remap(plan, ids, remap, xr)
    E.engram_hash(plan, xr, idx_b, history=hist)
    E.engram_stage_rows(plan, idx_b, tables, st_b, sidx_b, uq_b, nu_b)
    torch.cuda.synchronize()
    assert torch.equal(idx_a, idx_b) and torch.equal(sidx_a, sidx_b) and torch.equal(nu_a, nu_b)
    for h in range(wl.H):
        k = int(nu_a[h])
        assert torch.equal(uq_a[h, :k], uq_b[h, :k])
        assert torch.equal(st_a[h][:k].view(torch.int16), st_b[h][:k].view(torch.int16))
    # and the row ids are the oracle's
    ref = oracle.hash_ids(wl.remap()[wl.ids()], wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id,
                          history=wl.history() if history else None)
    assert np.array_equal(idx_a.cpu().numpy().view(np.uint32), ref)
    assert E.engram_device_status(clear=True) == 0
    for b in bufs:
        b.close()
