"""Multi-branch layer on the GPU (shared tables, memory vector and value projection; one key
projection and one residual-stream row per branch), against the oracle's branch composition.
Tolerances as for the single-branch layer, per branch."""
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

pytestmark = pytest.mark.gpu


def _ref(wl, di, step=0, ids=None, h=None, history=None, conv_state=None, decode=False):
    w = di.host_weights()
    M = wl.branches
    if h is None:
        h = synth.fill_bf16(wl.h_spec(step), (wl.h_rows, wl.d_h))
    return oracle.forward_branches(di.ids_np if ids is None else ids, di.remap_np, host_tables(wl),
                                   h.reshape(-1, M, wl.d_h), w["Wk"], w["Wv"], w["gamma_q"], w["gamma_k"],
                                   w["gamma_c"], w["conv_w"], orders=wl.orders, K=wl.K, primes=wl.primes,
                                   seed=wl.hash_seed, pad_id=wl.pad_id, eps=wl.eps, history=history,
                                   conv_state=conv_state, decode_outputs=decode, table_scales=table_scales(wl))


BRANCH_CASES = {
    # k=4 / dilation-3 prefill: per-(token, branch) scalars + the 4-channel gate kernel
    "m4_prefill": small_workload("b4", B=2, T=300, K=2, d_e=32, d_h=256, branches=4),
    # 128-wide projection tiles, ragged K (d_m = 240)
    "m2_bn128": small_workload("b2", B=3, T=400, K=3, d_e=40, d_h=384, branches=2),
    # orders {2}: dilation 2, the generic gate kernel
    "m3_generic": small_workload("b3g", B=2, T=150, orders=(2,), K=2, d_e=32, d_h=256, branches=3),
    # decode-sized prefill batch: split-K projection and its reduction
    "m2_splitk": small_workload("b2s", B=40, T=1, K=1, d_e=512, d_h=512, branches=2),
    # FP8 tables under four branches
    "m4_fp8": small_workload("b4f", B=2, T=200, K=2, d_e=32, d_h=256, branches=4, table_dtype="fp8"),
}


@pytest.mark.parametrize("case", list(BRANCH_CASES))
def test_forward_branches_match_oracle(case):
    wl = BRANCH_CASES[case]
    di = DeviceInputs(wl, random_gammas=True).forward()
    torch.cuda.synchronize()
    ref = _ref(wl, di)
    M = wl.branches
    assert_delta_close(di.delta.cpu().numpy().reshape(-1, M, wl.d_h), ref["delta"])
    assert_out_close(to_host_u16(di.out).reshape(-1, M, wl.d_h), ref["out"])
    assert E.engram_device_status(clear=True) == 0


@pytest.mark.parametrize("geom", ["small", "splitk"])
def test_branch_decode_steps_carry_per_branch_state(geom):
    if geom == "small":
        wl = small_workload("bdec", B=8, T=1, K=2, d_e=64, d_h=256, decode=True, branches=3)
    else:   # one-token steps whose projection splits K across CTAs
        wl = small_workload("bdecs", B=16, T=1, K=1, d_e=512, d_h=512, decode=True, branches=2)
    di = DeviceInputs(wl, random_gammas=True)
    M = wl.branches
    hist = wl.history()
    state = to_host_u16(di.conv_state)
    for step in range(8):
        ids_np = synth.zipf_ids(wl.vocab_in, 1.1, (wl.B, wl.T), 900 + step)
        h_np = synth.fill_bf16(wl.h_spec(step), (wl.h_rows, wl.d_h))
        di.ids, di.h = to_dev(ids_np), to_dev(h_np)
        di.forward()
        ref = _ref(wl, di, ids=ids_np, h=h_np, history=hist, conv_state=state, decode=True)
        torch.cuda.synchronize()
        assert_delta_close(di.delta.cpu().numpy().reshape(-1, M, wl.d_h), ref["delta"])
        assert_out_close(to_host_u16(di.out).reshape(-1, M, wl.d_h), ref["out"])
        assert np.array_equal(di.history.cpu().numpy(), ref["history"])
        assert_bf16_within_ulp(to_host_u16(di.conv_state), ref["state"])
        hist, state = ref["history"], to_host_u16(di.conv_state)


def test_branch_noalloc_and_gate_conv_entry_points():
    wl = small_workload("bna", B=2, T=120, K=2, d_e=32, d_h=256, branches=2)
    di = DeviceInputs(wl).forward()
    torch.cuda.synchronize()
    ref = _ref(wl, di)
    idx_np = oracle.hash_ids(wl.remap()[di.ids_np], wl.orders, wl.K, wl.primes, wl.hash_seed, wl.pad_id)
    m = torch.empty((wl.n_tok, wl.d_m), dtype=torch.bfloat16, device="cuda")
    E.engram_gather(di.plan, to_dev(idx_np.view(np.int32)), di.tables, m)
    out2 = torch.empty_like(di.out)
    E.engram_gate_conv(di.plan, di.weights, di.h, m, wl.B, wl.T, out2, di.ws)
    assert torch.equal(out2.view(torch.int16), di.out.view(torch.int16))
    out3, d3 = torch.empty_like(di.out), torch.empty_like(di.delta)
    E.engram_gate_conv_noalloc(di.plan, di.weights, di.h, m, wl.B, wl.T, out3, delta_dbg=d3)
    torch.cuda.synchronize()
    assert_delta_close(d3.cpu().numpy().reshape(-1, 2, wl.d_h), ref["delta"])
    assert_out_close(to_host_u16(out3).reshape(-1, 2, wl.d_h), ref["out"])
    with pytest.raises(ValueError):
        E.engram_gate_conv(di.plan, di.weights, di.h[: wl.n_tok], m, wl.B, wl.T, out2, di.ws)


@pytest.mark.slow
def test_layer2560x4_sampled_tokens():
    """The 4-branch layer at full size in the benchmark's launch configuration, checked on
    sampled tokens that the oracle computes on a window with regenerated table rows."""
    wl = synth.get_workload("layer2560x4")
    di = DeviceInputs(wl).forward()
    torch.cuda.synchronize()
    w = di.host_weights()
    M, S = wl.branches, wl.state_len
    rng = np.random.default_rng(13)
    picks = [(0, 0), (0, 47), (0, 48), (3, 4095), (7, 1000)] + [(int(b), int(t)) for b, t in
                                                               zip(rng.integers(0, wl.B, 5), rng.integers(0, wl.T, 5))]
    remap = di.remap_np
    got_out = to_host_u16(di.out).reshape(wl.n_tok, M, wl.d_h)
    got_delta = di.delta.cpu().numpy().reshape(wl.n_tok, M, wl.d_h)
    for b, t in picks:
        w0 = max(0, t - S)
        xr_full = remap[di.ids_np[b]]
        hist = np.array([[xr_full[p] if p >= 0 else wl.pad_id for p in (w0 - 2, w0 - 1)]], dtype=np.int32)
        idx = oracle.hash_ids(remap[di.ids_np[b:b + 1, w0:t + 1]], wl.orders, wl.K, wl.primes, wl.hash_seed,
                              wl.pad_id, history=hist)
        W = idx.shape[0]
        tabs = [synth.fill_rows_bf16(wl.table_spec(hh), wl.d_e, idx[:, hh]) for hh in range(wl.H)]
        m = oracle.gather(np.tile(np.arange(W, dtype=np.uint32)[:, None], (1, wl.H)), tabs)
        rows = np.arange(b * wl.T + w0, b * wl.T + t + 1)
        hrows = (rows[:, None] * M + np.arange(M)[None, :]).reshape(-1)
        h = synth.fill_rows_bf16(wl.h_spec(0), wl.d_h, hrows).reshape(W, M, wl.d_h)
        for br in range(M):
            r = oracle.gate_conv(h[:, br], m, w["Wk"][br * wl.d_h:(br + 1) * wl.d_h], w["Wv"], w["gamma_q"],
                                 w["gamma_k"], w["gamma_c"], w["conv_w"], 1, W, dil=wl.conv_dilation, eps=wl.eps)
            n = b * wl.T + t
            assert_delta_close(got_delta[n, br][None], r["delta"][-1][None])
            assert_out_close(got_out[n, br][None], r["out"][-1][None])
