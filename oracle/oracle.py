"""ctypes wrapper around the C oracle (test infrastructure only; see ``engram_oracle.c``)."""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "engram_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with the host C compiler (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_LIB)
        u64, i32, i64, dbl = C.c_uint64, C.c_int32, C.c_int64, C.c_double
        P = C.c_void_p
        L.oracle_splitmix64.restype = u64
        L.oracle_splitmix64.argtypes = [u64]
        L.oracle_fmix64.restype = u64
        L.oracle_fmix64.argtypes = [u64]
        L.oracle_hash_multiplier.restype = u64
        L.oracle_hash_multiplier.argtypes = [u64, C.c_int, C.c_int, C.c_int]
        L.oracle_hash_gram.restype = C.c_uint32
        L.oracle_hash_gram.argtypes = [P, C.c_int, C.c_int, u64, u64]
        L.oracle_bf16_to_double.restype = dbl
        L.oracle_bf16_to_double.argtypes = [C.c_uint16]
        L.oracle_double_to_bf16.restype = C.c_uint16
        L.oracle_double_to_bf16.argtypes = [dbl]
        L.oracle_e4m3_to_double.restype = dbl
        L.oracle_e4m3_to_double.argtypes = [C.c_uint8]
        L.oracle_dequant_e4m3.restype = C.c_uint16
        L.oracle_dequant_e4m3.argtypes = [C.c_uint8, C.c_float]
        L.oracle_dequant_table.restype = None
        L.oracle_dequant_table.argtypes = [P, i64, C.c_float, P]
        L.oracle_gather_e4m3.restype = None
        L.oracle_gather_e4m3.argtypes = [P, i64, i32, P, P, i32, P]
        L.oracle_remap.restype = C.c_int
        L.oracle_remap.argtypes = [P, i64, P, i32, P]
        L.oracle_hash.restype = None
        L.oracle_hash.argtypes = [P, i32, i32, P, i32, i32, i32, P, i32, P, u64, P]
        L.oracle_advance_history.restype = None
        L.oracle_advance_history.argtypes = [P, i32, i32, P, i32, i32, P]
        L.oracle_gather.restype = None
        L.oracle_gather.argtypes = [P, i64, i32, P, i32, P]
        L.oracle_gate_conv.restype = C.c_int
        L.oracle_gate_conv.argtypes = [P, P, i32, i32, P, P, P, P, P, P, i32, i32, i32, i32, dbl,
                                       P, P, P, P, P]
        L.oracle_forward.restype = C.c_int
        L.oracle_forward.argtypes = [P, i32, i32, P, i32, P, i32, i32, i32, P, i32, P, u64,
                                     P, i32, P, i32, P, P, P, P, P, P, i32, i32, dbl,
                                     P, P, P, P, P, P, P]
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype)


# ---- scalar primitives ------------------------------------------------------------------
def splitmix64(state: int) -> int:
    return int(lib().oracle_splitmix64(state & 0xFFFFFFFFFFFFFFFF))


def fmix64(k: int) -> int:
    return int(lib().oracle_fmix64(k & 0xFFFFFFFFFFFFFFFF))


def hash_multiplier(seed: int, order: int, head: int, pos: int) -> int:
    return int(lib().oracle_hash_multiplier(seed, order, head, pos))


def hash_gram(gram: Sequence[int], order: int, head: int, seed: int, prime: int) -> int:
    """gram[0] is the current token, gram[i] the token i positions back."""
    g = _c(list(gram), np.int32)
    return int(lib().oracle_hash_gram(_p(g), order, head, seed, prime))


def bf16_to_double(bits: int) -> float:
    return float(lib().oracle_bf16_to_double(bits))


def double_to_bf16(x: float) -> int:
    return int(lib().oracle_double_to_bf16(float(x)))


def e4m3_to_double(code: int) -> float:
    return float(lib().oracle_e4m3_to_double(code & 0xFF))


def dequant_e4m3(code: int, scale) -> int:
    return int(lib().oracle_dequant_e4m3(code & 0xFF, float(np.float32(scale))))


def dequant_table(codes: np.ndarray, scale) -> np.ndarray:
    """e4m3 codes (any shape, uint8) -> bf16 patterns of the same shape."""
    codes = _c(codes, np.uint8)
    out = np.empty(codes.shape, dtype=np.uint16)
    lib().oracle_dequant_table(_p(codes), codes.size, float(np.float32(scale)), _p(out))
    return out


# ---- steps -------------------------------------------------------------------------------
def remap(ids: np.ndarray, table: np.ndarray) -> np.ndarray:
    ids = _c(ids, np.int32)
    table = _c(table, np.int32)
    out = np.empty_like(ids)
    rc = lib().oracle_remap(_p(ids), ids.size, _p(table), table.size, _p(out))
    if rc != 0:
        raise ValueError("token id out of range")
    return out


def hash_ids(xr: np.ndarray, orders, K: int, primes, seed: int, pad_id: int,
             history: Optional[np.ndarray] = None) -> np.ndarray:
    """xr: [B, T] remapped ids.  Returns idx [B*T, H] uint32."""
    xr = _c(xr, np.int32)
    B, T = xr.shape
    orders = _c(list(orders), np.int32)
    primes = _c(list(primes), np.uint64)
    H = len(orders) * K
    assert primes.size == H
    hist_len = int(max(orders)) - 1
    if history is not None:
        history = _c(history, np.int32)
        assert history.shape == (B, hist_len)
    idx = np.empty((B * T, H), dtype=np.uint32)
    lib().oracle_hash(_p(xr), B, T, _p(history), hist_len, pad_id, orders.size, _p(orders), K,
                      _p(primes), seed, _p(idx))
    return idx


def advance_history(xr: np.ndarray, history: Optional[np.ndarray], hist_len: int, pad_id: int):
    xr = _c(xr, np.int32)
    B, T = xr.shape
    history = _c(history, np.int32)
    out = np.empty((B, hist_len), dtype=np.int32)
    lib().oracle_advance_history(_p(xr), B, T, _p(history), hist_len, pad_id, _p(out))
    return out


def _table_ptrs(tables):
    arrs = [_c(t, np.uint16) for t in tables]
    ptrs = (C.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
    return arrs, ptrs


def gather(idx: np.ndarray, tables, scales=None) -> np.ndarray:
    """bf16 tables (uint16 patterns); or e4m3 tables (uint8 codes) with one scale per table."""
    idx = _c(idx, np.uint32)
    n_tok, H = idx.shape
    if scales is None:
        arrs, ptrs = _table_ptrs(tables)
        d_e = arrs[0].shape[1]
        m = np.empty((n_tok, H * d_e), dtype=np.uint16)
        lib().oracle_gather(_p(idx), n_tok, H, ptrs, d_e, _p(m))
        return m
    arrs = [_c(t, np.uint8) for t in tables]
    ptrs = (C.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
    sc = _c([float(x) for x in scales], np.float32)
    d_e = arrs[0].shape[1]
    m = np.empty((n_tok, H * d_e), dtype=np.uint16)
    lib().oracle_gather_e4m3(_p(idx), n_tok, H, ptrs, _p(sc), d_e, _p(m))
    return m


def gate_conv(h, m, Wk, Wv, gamma_q, gamma_k, gamma_c, conv_w, B: int, T: int,
              dil: int = 3, eps: float = 1e-6, conv_state=None, want_state: bool = False):
    """Returns dict(out=bf16 [B*T, d_h], delta=f64, gate=f64 [B*T], state=bf16 or None)."""
    h = _c(h, np.uint16)
    m = _c(m, np.uint16)
    Wk, Wv = _c(Wk, np.uint16), _c(Wv, np.uint16)
    gq, gk, gc = _c(gamma_q, np.uint16), _c(gamma_k, np.uint16), _c(gamma_c, np.uint16)
    conv_w = _c(conv_w, np.uint16)
    d_h, d_m = Wk.shape
    ksize = conv_w.shape[1]
    S = (ksize - 1) * dil
    n = B * T
    out = np.empty((n, d_h), dtype=np.uint16)
    delta = np.empty((n, d_h), dtype=np.float64)
    gate = np.empty((n,), dtype=np.float64)
    cs = _c(conv_state, np.uint16)
    st = np.empty((B, S, d_h), dtype=np.uint16) if want_state else None
    rc = lib().oracle_gate_conv(_p(h), _p(m), d_m, d_h, _p(Wk), _p(Wv), _p(gq), _p(gk), _p(gc),
                                _p(conv_w), ksize, dil, B, T, eps, _p(cs), _p(st), _p(out),
                                _p(delta), _p(gate))
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return dict(out=out, delta=delta, gate=gate, state=st)


def forward(ids, remap_table, tables, h, Wk, Wv, gamma_q, gamma_k, gamma_c, conv_w, *,
            orders, K: int, primes, seed: int, pad_id: int, eps: float = 1e-6,
            history=None, conv_state=None, decode_outputs: bool = False, table_scales=None):
    """All six steps.  Returns dict(out, delta, gate, idx[, state, history]).
    table_scales: None for bf16 tables, else one dequantisation scale per e4m3 table (the
    tables are then uint8 codes, dequantised to bf16 before the lookup)."""
    if table_scales is not None:
        tables = [dequant_table(t, s) for t, s in zip(tables, table_scales)]
    ids = _c(ids, np.int32)
    B, T = ids.shape
    remap_table = _c(remap_table, np.int32)
    orders_a = _c(list(orders), np.int32)
    primes_a = _c(list(primes), np.uint64)
    H = orders_a.size * K
    hist_len = int(max(orders)) - 1
    dil = int(max(orders))
    arrs, ptrs = _table_ptrs(tables)
    d_e = arrs[0].shape[1]
    h = _c(h, np.uint16)
    Wk, Wv = _c(Wk, np.uint16), _c(Wv, np.uint16)
    gq, gk, gc = _c(gamma_q, np.uint16), _c(gamma_k, np.uint16), _c(gamma_c, np.uint16)
    conv_w = _c(conv_w, np.uint16)
    d_h = Wk.shape[0]
    ksize = conv_w.shape[1]
    S = (ksize - 1) * dil
    n = B * T
    out = np.empty((n, d_h), dtype=np.uint16)
    delta = np.empty((n, d_h), dtype=np.float64)
    gate = np.empty((n,), dtype=np.float64)
    idx = np.empty((n, H), dtype=np.uint32)
    history = _c(history, np.int32)
    cs = _c(conv_state, np.uint16)
    st = np.empty((B, S, d_h), dtype=np.uint16) if decode_outputs else None
    hist_out = np.empty((B, hist_len), dtype=np.int32) if decode_outputs else None
    rc = lib().oracle_forward(_p(ids), B, T, _p(remap_table), remap_table.size, _p(history),
                              hist_len, pad_id, orders_a.size, _p(orders_a), K, _p(primes_a),
                              seed, ptrs, d_e, _p(h), d_h, _p(Wk), _p(Wv), _p(gq), _p(gk),
                              _p(gc), _p(conv_w), ksize, dil, eps, _p(cs), _p(st),
                              _p(hist_out), _p(out), _p(delta), _p(gate), _p(idx))
    if rc == -1:
        raise ValueError("token id out of range")
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    res = dict(out=out, delta=delta, gate=gate, idx=idx)
    if decode_outputs:
        res["state"] = st
        res["history"] = hist_out
    return res


def forward_branches(ids, remap_table, tables, h, Wk, Wv, gamma_q, gamma_k, gamma_c, conv_w, *,
                     orders, K: int, primes, seed: int, pad_id: int, eps: float = 1e-6,
                     history=None, conv_state=None, decode_outputs: bool = False, table_scales=None):
    """The multi-branch layer [yktysq, component 4: the branches share the embedding table and
    the value projection, and each has its own key projection, so that each branch gates the
    memory in its own way].  Every branch b is the single-branch layer on its own hidden state
    h[:, b] and key projection Wk[b*d_h:(b+1)*d_h], with the same memory vector m, W_v, gains
    and conv weights; its conv state (decode) is conv_state[:, b].

    h: [B*T, M, d_h]; Wk: [M*d_h, d_m]; conv_state: None or [B, M, S, d_h].
    Returns dict(out [B*T, M, d_h], delta, gate [B*T, M], idx[, state [B, M, S, d_h], history]).
    """
    ids = _c(ids, np.int32)
    B, T = ids.shape
    h = _c(h, np.uint16)
    n, M, d_h = h.shape
    Wk = _c(Wk, np.uint16)
    assert Wk.shape[0] == M * d_h
    dil = int(max(orders))
    hist_len = dil - 1
    xr = remap(ids, remap_table)
    idx = hash_ids(xr, orders, K, primes, seed, pad_id, history=history)
    m = gather(idx, tables, table_scales)
    outs, deltas, gates, states = [], [], [], []
    for b in range(M):
        cs = None if conv_state is None else _c(conv_state, np.uint16)[:, b]
        r = gate_conv(h[:, b], m, Wk[b * d_h:(b + 1) * d_h], Wv, gamma_q, gamma_k, gamma_c, conv_w, B, T,
                      dil=dil, eps=eps, conv_state=cs, want_state=decode_outputs)
        outs.append(r["out"])
        deltas.append(r["delta"])
        gates.append(r["gate"])
        states.append(r["state"])
    res = dict(out=np.stack(outs, axis=1), delta=np.stack(deltas, axis=1), gate=np.stack(gates, axis=1), idx=idx)
    if decode_outputs:
        res["state"] = np.stack(states, axis=1)
        res["history"] = advance_history(xr, history, hist_len, pad_id)
    return res
