"""Shared test helpers: host-side input construction from the seeded generators."""
from __future__ import annotations

import numpy as np

import synth
from synth import Workload, fill_bf16

ONE_BF16 = np.uint16(0x3F80)


def small_workload(name="small", *, B=2, T=40, orders=(2, 3), K=2, primes=None, d_e=16,
                   d_h=64, vocab_in=300, vocab_out=200, **kw) -> Workload:
    H = len(orders) * K
    if primes is None:
        base = [1009, 1013, 1019, 1021, 1031, 1033, 1039, 1049, 1051, 1061, 1063, 1069,
                1087, 1091, 1093, 1097, 1103, 1109, 1117, 1123, 1129, 1151, 1153, 1163,
                1171, 1181, 1187, 1193, 1201, 1213, 1217, 1223]
        primes = tuple(base[:H])
    return Workload(name=name, description="test case", vocab_in=vocab_in, vocab_out=vocab_out,
                    B=B, T=T, orders=tuple(orders), K=K, primes=tuple(primes), d_e=d_e, d_h=d_h,
                    index=kw.pop("index", 17), **kw)


def make_inputs(wl: Workload, step: int = 0, tables=True):
    """Host arrays for one call; bf16 tensors are uint16 bit patterns.  With M = wl.branches
    > 1, h is [n_tok, M, d_h], Wk [M*d_h, d_m] and the conv state [B, M, S, d_h]."""
    M = wl.branches
    h = fill_bf16(wl.h_spec(step), (wl.h_rows, wl.d_h))
    d = dict(
        ids=wl.ids(step),
        remap=wl.remap(),
        h=h.reshape(wl.n_tok, M, wl.d_h) if M > 1 else h,
        Wk=fill_bf16(wl.wk_spec(), (M * wl.d_h, wl.d_m)),
        Wv=fill_bf16(wl.wv_spec(), (wl.d_h, wl.d_m)),
        gamma_q=np.full(wl.d_h, ONE_BF16, dtype=np.uint16),
        gamma_k=np.full(wl.d_h, ONE_BF16, dtype=np.uint16),
        gamma_c=np.full(wl.d_h, ONE_BF16, dtype=np.uint16),
        conv_w=fill_bf16(wl.conv_spec(), (wl.d_h, wl.conv_kernel)),
        history=wl.history(),
        conv_state=(fill_bf16(wl.state_spec(), (wl.B * M, wl.state_len, wl.d_h)).reshape(
            (wl.B, M, wl.state_len, wl.d_h) if M > 1 else (wl.B, wl.state_len, wl.d_h)) if wl.decode else None),
    )
    if tables:
        d["tables"] = [fill_bf16(wl.table_spec(h), (wl.primes[h], wl.d_e)) for h in range(wl.H)]
    return d


def bf16(x) -> np.ndarray:
    return synth.float_to_bf16_rne(np.asarray(x, dtype=np.float32))


def f32(b) -> np.ndarray:
    return synth.bf16_to_float(b)


def bf16_ulp(x_bits: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at each value (the ulp of the value's binade)."""
    v = np.abs(f32(x_bits).astype(np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return 2.0 ** (e - 7)
