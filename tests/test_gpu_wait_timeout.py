"""The failure path of the bounded device-side waits.

Every pipeline wait inside the projection kernel gives up after a bound; the kernel then
raises ENGRAM_STATUS_WAIT_TIMEOUT, releases its other roles, frees its tensor memory and
returns, so the device stays usable.  engram_selftest_wait_timeout runs that kernel with its
producer stalled (no tile is ever loaded) and a short bound, so that the first wait of every
CTA runs out: nothing faults or hangs, the GPU only idles for the bound.
"""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import hashed_gram_embedding_remap_b200 as E
from gpu_helpers import DeviceInputs, assert_delta_close, assert_out_close, to_host_u16
from helpers import small_workload
from test_gpu_parity import _oracle_full

pytestmark = pytest.mark.gpu


def test_stalled_projection_times_out_unwinds_and_leaves_the_device_usable():
    wl = small_workload("stall", B=2, T=300, K=2, d_e=32, d_h=256)
    di = DeviceInputs(wl)
    torch.cuda.synchronize()
    E.engram_device_status(clear=True)
    E.engram_synchronize()                       # nothing pending: OK
    m = torch.zeros((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
    t0 = time.perf_counter()
    E.engram_selftest_wait_timeout(di.plan, di.weights, di.h, m, di.ws, wait_limit_ns=200_000)   # 0.2 ms
    with pytest.raises(E.EngramError) as ei:
        E.engram_synchronize()
    elapsed = time.perf_counter() - t0
    assert ei.value.code == E.ENGRAM_ERR_TIMEOUT
    assert elapsed < 10.0, f"the stalled kernel took {elapsed:.1f} s to unwind"
    assert E.engram_device_status(clear=True) & E.ENGRAM_STATUS_WAIT_TIMEOUT
    E.engram_synchronize()                       # cleared: OK again
    # the context survived: a normal forward still matches the oracle
    di.forward()
    E.engram_synchronize()
    ref = _oracle_full(wl, di)
    assert_delta_close(di.delta.cpu().numpy(), ref["delta"])
    assert_out_close(to_host_u16(di.out), ref["out"])
    assert E.engram_device_status(clear=True) == 0
