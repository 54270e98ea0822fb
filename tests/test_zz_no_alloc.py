"""The workspace-free gate/conv entry point (engram_gate_conv_noalloc).

Some hosts cannot allocate device memory for an operator: plugin and custom-op interfaces
of inference servers pass an op only its inputs and outputs and own every allocation, and
some runtimes run under a fixed memory budget or cannot afford the device-wide
synchronisation of cudaMalloc/cudaFree.  For them the library keeps the scratch of the
projection + gate/conv step in a fixed per-GPU array inside its own device data.  This
test calls that entry point through the C ABI twice in a row and checks each result
against the workspace entry point and against the CPU oracle, within the tolerance the
parity tests use.  It lives in its own file so that pytest collects it last.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import pytest
import torch

import hashed_gram_embedding_remap_b200 as E
import oracle
from gpu_helpers import (DeviceInputs, assert_bf16_within_ulp, assert_delta_close, assert_out_close, to_dev,
                         to_host_u16)
from helpers import small_workload

pytestmark = pytest.mark.gpu


def _memory_vectors(wl, di):
    xr = wl.remap()[di.ids_np]
    idx = oracle.hash_ids(xr, wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    m = torch.empty((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
    E.engram_gather(di.plan, to_dev(idx.view(np.int32)), di.tables, m)
    return m


def _oracle(wl, di, m, state0):
    """The oracle's steps 4-6 on the same memory vectors, hidden states and conv state."""
    w = di.host_weights()
    return oracle.gate_conv(to_host_u16(di.h), to_host_u16(m), w["Wk"], w["Wv"], w["gamma_q"], w["gamma_k"],
                            w["gamma_c"], w["conv_w"], wl.B, wl.T, dil=wl.conv_dilation, eps=wl.eps,
                            conv_state=None if state0 is None else to_host_u16(state0),
                            want_state=state0 is not None)


@pytest.mark.parametrize("case", ["prefill", "decode"])
def test_noalloc_matches_workspace_entry_two_calls(case):
    if case == "prefill":
        wl = small_workload("noalloc_prefill", B=3, T=333, K=3, d_e=40, d_h=384)
    else:
        wl = small_workload("noalloc_decode", B=64, T=1, K=2, d_e=32, d_h=512, decode=True)
    di = DeviceInputs(wl)
    m = _memory_vectors(wl, di)
    state0 = di.conv_state.clone() if di.conv_state is not None else None

    ref_out = torch.empty_like(di.out)
    ref_delta = torch.empty_like(di.delta)
    ref_state = state0.clone() if state0 is not None else None
    E.engram_gate_conv(di.plan, di.weights, di.h, m, wl.B, wl.T, ref_out, di.ws, conv_state=ref_state,
                       delta_dbg=ref_delta)
    torch.cuda.synchronize()
    ref_o, ref_d = to_host_u16(ref_out), ref_delta.cpu().numpy()
    orc = _oracle(wl, di, m, state0)

    for call in range(2):
        out = torch.full_like(di.out, 7.0)
        delta = torch.full_like(di.delta, float("nan"))
        state = state0.clone() if state0 is not None else None
        E.engram_gate_conv_noalloc(di.plan, di.weights, di.h, m, wl.B, wl.T, out, conv_state=state,
                                   delta_dbg=delta)
        torch.cuda.synchronize()
        assert_delta_close(delta.cpu().numpy(), ref_d)
        assert_out_close(to_host_u16(out), ref_o)
        assert_delta_close(delta.cpu().numpy(), orc["delta"])
        assert_out_close(to_host_u16(out), orc["out"])
        if state is not None:
            assert_bf16_within_ulp(to_host_u16(state), to_host_u16(ref_state))
            assert_bf16_within_ulp(to_host_u16(state), orc["state"])
    assert E.engram_device_status(clear=True) == 0


def test_noalloc_rejects_requests_beyond_its_scratch():
    wl = small_workload("noalloc_big", B=1, T=8, K=2, d_e=32, d_h=2560)
    plan = E.Plan.from_workload(wl)
    # the fp16 value projections alone (2 bytes per channel and token) exceed the array here
    T = E.ENGRAM_NOALLOC_SCRATCH_BYTES // (2 * wl.d_h) + 1
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    w = E.Weights(dummy, dummy, dummy, dummy, dummy, dummy)
    # straight through the C ABI (the binding would refuse the undersized tensors first): the
    # size check runs on the host before anything is launched, so nothing reads the dummies
    p = C.c_void_p(dummy.data_ptr())
    rc = E.lib.engram_gate_conv_noalloc(plan, w, p, p, 1, T, None, p, None, None)
    assert rc == E.ENGRAM_ERR_UNSUPPORTED and "scratch" in E.last_error()
