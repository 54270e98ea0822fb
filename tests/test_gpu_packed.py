"""Packed projection weights: the packed copy has exactly the documented layout (checked
against a host construction of it), and every path that streams it gives results identical
to the row-major weights (prefill, split-K decode, branches, ragged K)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hashed_gram_embedding_remap_b200 as E
import synth
from gpu_helpers import DeviceInputs, to_dev
from helpers import small_workload

pytestmark = pytest.mark.gpu


def _host_packed(wk: np.ndarray, wv: np.ndarray) -> np.ndarray:
    """The documented layout, built on the host: tile (t, b) of [W_k ; W_v] (256 rows x 64
    columns, zero past d_m) at (t * k_blocks + b) * 32 KB, row r at r * 128 bytes, 16-byte
    chunk j at position j ^ (r % 8)."""
    w = np.concatenate([wk, wv], axis=0)
    rows, d_m = w.shape
    kb = (d_m + 63) // 64
    wp = np.zeros((rows, kb * 64), dtype=np.uint16)
    wp[:, :d_m] = w
    tiles = wp.reshape(rows // 256, 256, kb, 8, 8)            # [t, r, b, chunk, 8 values]
    out = np.empty((rows // 256, kb, 256, 8, 8), dtype=np.uint16)
    for r in range(256):
        for j in range(8):
            out[:, :, r, j ^ (r % 8), :] = tiles[:, r, :, j, :]
    return out.reshape(-1)


def test_packed_layout_matches_host_construction():
    wl = small_workload("pk", B=1, T=8, K=3, d_e=40, d_h=512, branches=2)      # d_m = 240 (ragged)
    plan = E.Plan.from_workload(wl)
    wk = synth.fill_bf16(wl.wk_spec(), (2 * wl.d_h, wl.d_m))
    wv = synth.fill_bf16(wl.wv_spec(), (wl.d_h, wl.d_m))
    packed = E.pack_weights(plan, to_dev(wk), to_dev(wv))
    torch.cuda.synchronize()
    got = packed.cpu().numpy().view(np.uint16)
    assert got.size * 2 == E.engram_packed_weights_size(plan)
    assert np.array_equal(got, _host_packed(wk, wv))


@pytest.mark.parametrize("case", ["prefill", "decode_splitk", "branches", "ragged_k"])
def test_packed_weights_give_identical_results(case):
    if case == "prefill":
        wl = small_workload("pkp", B=4, T=2000, K=2, d_e=64, d_h=512)
    elif case == "decode_splitk":
        wl = small_workload("pkd", B=256, T=1, K=1, d_e=512, d_h=512, decode=True)
    elif case == "branches":
        wl = small_workload("pkb", B=2, T=1500, K=2, d_e=64, d_h=512, branches=3)
    else:
        wl = small_workload("pkr", B=3, T=777, K=3, d_e=40, d_h=256)
    di = DeviceInputs(wl, random_gammas=True)
    state0 = di.conv_state.clone() if di.conv_state is not None else None
    hist0 = di.history.clone() if di.history is not None else None
    di.forward()
    torch.cuda.synchronize()
    out_ref, delta_ref = di.out.clone(), di.delta.clone()
    di.weights = E.Weights(di.w_k, di.w_v, di.gamma_q, di.gamma_k, di.gamma_c, di.conv_w,
                           packed=E.pack_weights(di.plan, di.w_k, di.w_v))
    if state0 is not None:
        di.conv_state.copy_(state0)
        di.history.copy_(hist0)
    di.forward()
    torch.cuda.synchronize()
    assert torch.equal(di.out.view(torch.int16), out_ref.view(torch.int16))
    assert torch.equal(di.delta, delta_ref)
    assert E.engram_device_status(clear=True) == 0
