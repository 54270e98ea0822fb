"""HBM row cache in front of host-resident tables: staged rows are exact whatever the cache
holds; hits, replacements and tags follow the documented direct-mapped policy (checked
against a host model of it); every cached slot holds exactly the row its tag names; the
layer computed from cached staging is bit-identical to HBM-resident tables."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hashed_gram_embedding_remap_b200 as E
import oracle
import synth
from cache_model import CacheModel
from gpu_helpers import DeviceInputs, host_rows, to_dev, to_host_u16
from helpers import small_workload
from synth import fill_gpu

pytestmark = pytest.mark.gpu


def _host_tables(wl):
    eb = wl.table_elem_bytes
    bufs = []
    for h in range(wl.H):
        hm = fill_gpu.HostMapped(wl.primes[h], wl.d_e, elem_bytes=eb)
        (fill_gpu.fill_fp8_ if eb == 1 else fill_gpu.fill_)(hm.tensor, wl.table_spec(h))
        bufs.append(hm)
    torch.cuda.synchronize()
    return bufs


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy() if t.dtype == torch.uint8 else to_host_u16(t)


def _stored_rows(wl, h, rows):
    """Table rows as stored (bf16 patterns or e4m3 codes)."""
    if wl.table_dtype == "fp8":
        return synth.fill_rows_fp8(wl.table_spec(h), wl.d_e, rows)
    return synth.fill_rows_bf16(wl.table_spec(h), wl.d_e, rows)


@pytest.mark.parametrize("dtype,slots", [("bf16", 64), ("bf16", 4096), ("fp8", 256)])
def test_cached_staging_exact_and_policy_matches_model(dtype, slots):
    wl = small_workload("rc", B=48, T=1, K=2, d_e=64, d_h=128, primes=(1009, 1013, 1019, 1021),
                        vocab_in=60, vocab_out=60, identity_remap=True, table_dtype=dtype)
    plan = E.Plan.from_workload(wl, host_tables=True)
    bufs = _host_tables(wl)
    tables = [b.tensor for b in bufs]
    cache = E.RowCache(plan, slots)
    model = CacheModel(wl.H, slots, wl.primes)
    n = wl.n_tok
    tdt = torch.uint8 if dtype == "fp8" else torch.bfloat16
    staging = [torch.empty((n, wl.d_e), dtype=tdt, device="cuda") for _ in range(wl.H)]
    sidx = torch.empty((n, wl.H), dtype=torch.int32, device="cuda")
    uniq = torch.empty((wl.H, n), dtype=torch.int32, device="cuda")
    nu = torch.empty((wl.H,), dtype=torch.int32, device="cuda")
    flags = torch.empty((wl.H, n), dtype=torch.int32, device="cuda")
    n_hits = torch.zeros((wl.H,), dtype=torch.int32, device="cuda")
    total_hits = 0
    for step in range(12):
        ids = synth.zipf_ids(wl.vocab_in, 1.2, (wl.B, 3), 300 + step).astype(np.int32)   # identity remap
        idx_np = oracle.hash_ids(ids[:, 2:], wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id,
                                 history=np.ascontiguousarray(ids[:, :2]))
        n_hits.zero_()
        E.engram_stage_rows_cached(plan, to_dev(idx_np.view(np.int32)), tables, cache, staging, sidx, uniq, nu,
                                   flags, n_hits)
        torch.cuda.synchronize()
        want_hits = model.step(idx_np)
        assert n_hits.cpu().tolist() == want_hits, step
        total_hits += sum(want_hits)
        sidx_h, uniq_h, nu_h = sidx.cpu().numpy(), uniq.cpu().numpy().view(np.uint32), nu.cpu().numpy()
        for h in range(wl.H):
            ref = np.unique(idx_np[:, h])
            assert nu_h[h] == ref.size and np.array_equal(uniq_h[h, : nu_h[h]], ref)
            assert np.array_equal(uniq_h[h, sidx_h[:, h]], idx_np[:, h])
            assert np.array_equal(_bits(staging[h][: nu_h[h]]), _stored_rows(wl, h, ref))
            tags = cache.tags[h].cpu().numpy().view(np.uint32).astype(np.int64)
            assert np.array_equal(tags, model.tags[h])
            held = np.nonzero(tags)[0]
            if held.size:
                assert np.array_equal(_bits(cache.data[h][torch.from_numpy(held).cuda()]),
                                      _stored_rows(wl, h, tags[held] - 1))
            assert (cache.claim[h].cpu().numpy().view(np.uint32) == 0xFFFFFFFF).all()
    assert total_hits > 0
    assert E.engram_device_status(clear=True) == 0
    for b in bufs:
        b.close()


def test_layer_from_cached_staging_is_bit_identical():
    wl = small_workload("rcl", B=64, T=1, K=1, d_e=256, d_h=256, primes=(100003, 100019), zipf_s=1.3)
    dev = DeviceInputs(wl).forward(delta=False)
    torch.cuda.synchronize()
    plan_h = E.Plan.from_workload(wl, host_tables=True)
    bufs = _host_tables(wl)
    cache = E.RowCache(plan_h, 1 << 10)
    n = wl.n_tok
    xr = torch.empty_like(dev.ids)
    E.engram_remap(plan_h, dev.ids, dev.remap, xr)
    idx = torch.empty((n, wl.H), dtype=torch.int32, device="cuda")
    E.engram_hash(plan_h, xr, idx)
    staging = [torch.empty((n, wl.d_e), dtype=torch.bfloat16, device="cuda") for _ in range(wl.H)]
    sidx = torch.empty((n, wl.H), dtype=torch.int32, device="cuda")
    uniq = torch.empty((wl.H, n), dtype=torch.int32, device="cuda")
    nu = torch.empty((wl.H,), dtype=torch.int32, device="cuda")
    flags = torch.empty((wl.H, n), dtype=torch.int32, device="cuda")
    n_hits = torch.zeros((wl.H,), dtype=torch.int32, device="cuda")
    m = torch.empty((n, wl.d_m), dtype=torch.bfloat16, device="cuda")
    ws = E.alloc_workspace(plan_h, n)
    for rep in range(2):   # second pass: every row served from the cache
        n_hits.zero_()
        E.engram_stage_rows_cached(plan_h, idx, [b.tensor for b in bufs], cache, staging, sidx, uniq, nu, flags, n_hits)
        E.engram_gather(plan_h, sidx, staging, m, rows_bound=n)
        out = torch.empty_like(dev.out)
        E.engram_gate_conv(plan_h, dev.weights, dev.h, m, wl.B, wl.T, out, ws)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), dev.out.view(torch.int16))
    assert int(n_hits.sum()) > 0
    for b in bufs:
        b.close()
