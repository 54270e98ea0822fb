"""The C-ABI library loads on the host and exports every entry point include/engram.h declares;
host-side validation works without a GPU (invalid arguments are rejected before any launch)."""
from __future__ import annotations

import ctypes as C
import os
import re

import pytest

import hashed_gram_embedding_remap_b200 as E
import synth
from hashed_gram_embedding_remap_b200 import _native

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "engram.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(engram_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert {"engram_remap", "engram_hash", "engram_gather", "engram_gate_conv", "engram_forward"} <= set(names)
    lib = C.CDLL(E.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in engram.h but not exported"


def test_binding_constants_match_header():
    """Every ENGRAM_* value the binding defines is the header's (status codes, flags, path
    bits, limits): parsed from the #define lines, evaluated as plain integers."""
    src = open(HEADER).read()
    defs = {}
    for name, val in re.findall(r"^#define (ENGRAM_[A-Z0-9_]+) +([^/\n]+)", src, flags=re.M):
        v = val.strip().replace("u", "")
        if re.fullmatch(r"[-+()0-9xa-fA-F <]+", v):
            defs[name] = eval(v)   # integer literals, shifts and parentheses only
    assert len(defs) >= 20
    checked = 0
    for name, v in defs.items():
        if hasattr(_native, name):
            assert getattr(_native, name) == v, name
            checked += 1
    assert checked >= 20
    for name in ("ENGRAM_FLAG_ROW_ORDER_GATHER", "ENGRAM_FLAG_BULK_GATHER", "ENGRAM_PATH_ROW_ORDER",
                 "ENGRAM_PATH_BULK_GATHER", "ENGRAM_PATH_PAIR_MMA"):
        assert name in defs and hasattr(_native, name), name


def test_struct_layouts_match_header():
    for name, cls in (("engram_config", _native.engram_config), ("engram_plan", _native.engram_plan),
                      ("engram_weights", _native.engram_weights), ("engram_row_cache", _native.engram_row_cache)):
        assert E.lib.engram_sizeof(name.encode()) == C.sizeof(cls)
    assert E.lib.engram_sizeof(b"nope") == 0


def _plan(**kw):
    base = dict(orders=(2, 3), heads_per_order=2, table_rows=(10007, 10009, 10037, 10039), row_dim=32,
                hidden_dim=256, vocab_in=1000, vocab_out=770, hash_seed=7)
    base.update(kw)
    return E.Plan(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(table_rows=(10007, 10009, 10037, 10040)), E.ENGRAM_ERR_INVALID_ARG),   # not prime
    (dict(table_rows=(10007, 10009, 10037)), E.ENGRAM_ERR_INVALID_ARG),          # 0 rows for table 3
    (dict(orders=(3, 2)), E.ENGRAM_ERR_INVALID_ARG),                             # not increasing
    (dict(orders=(2, 5)), E.ENGRAM_ERR_UNSUPPORTED),
    (dict(row_dim=30), E.ENGRAM_ERR_UNSUPPORTED),
    (dict(hidden_dim=200), E.ENGRAM_ERR_UNSUPPORTED),
    (dict(eps=0.0), E.ENGRAM_ERR_INVALID_ARG),
    (dict(conv_kernel=9), E.ENGRAM_ERR_UNSUPPORTED),
    (dict(heads_per_order=17), E.ENGRAM_ERR_UNSUPPORTED),
    (dict(flags=0x1), E.ENGRAM_ERR_INVALID_ARG),                                # retired flag bits
    (dict(flags=0x2), E.ENGRAM_ERR_INVALID_ARG),
    (dict(flags=0x20), E.ENGRAM_ERR_INVALID_ARG),                               # unknown flag bit
    (dict(table_dtype=2), E.ENGRAM_ERR_INVALID_ARG),                            # unknown table dtype
    (dict(table_dtype=1, table_scale=(0.1, 0.1, 0.1, 0.0)), E.ENGRAM_ERR_INVALID_ARG),   # zero scale
    (dict(table_dtype=1, table_scale=(0.1, float("inf"), 0.1, 0.1)), E.ENGRAM_ERR_INVALID_ARG),
    (dict(table_dtype=1, table_scale=(0.1, 0.1, 0.1, -0.1)), E.ENGRAM_ERR_INVALID_ARG),
    (dict(table_dtype=1, table_scale=(0.1,) * 5), E.ENGRAM_ERR_INVALID_ARG),   # scale beyond H
    (dict(table_dtype=1, table_scale=(0.1, 2.0 ** -101, 0.1, 0.1)), E.ENGRAM_ERR_INVALID_ARG),  # products
    (dict(table_dtype=1, table_scale=(0.1, 2.0 ** 101, 0.1, 0.1)), E.ENGRAM_ERR_INVALID_ARG),   # leave fp32
    (dict(table_dtype=0, table_scale=(0.1,)), E.ENGRAM_ERR_INVALID_ARG),       # scale on bf16
    (dict(table_dtype=1, table_scale=(0.1,) * 4, row_dim=24), E.ENGRAM_ERR_UNSUPPORTED),
    (dict(num_branches=9), E.ENGRAM_ERR_UNSUPPORTED),
    (dict(num_branches=-1), E.ENGRAM_ERR_UNSUPPORTED),
])
def test_init_rejects_bad_configs(kw, code):
    with pytest.raises(E.EngramError) as ei:
        _plan(**kw)
    assert ei.value.code == code


def test_init_accepts_every_workload_and_derives_constants():
    for name, wl in synth.WORKLOADS.items():
        p = E.Plan.from_workload(wl)
        assert p.num_tables == wl.H and p.mem_dim == wl.d_m
        assert p.hist_len == max(wl.orders) - 1 and p.state_len == 3 * max(wl.orders)
        assert E.engram_workspace_size(p, wl.n_tok) > 0
        pf = E.Plan.from_workload(wl.with_(table_dtype="fp8"))
        assert pf.cfg.table_dtype == E.ENGRAM_TABLE_FP8_E4M3
        assert [pf.plan.cfg.table_scale[h] for h in range(wl.H)] == [float(wl.table_scale(h)) for h in range(wl.H)]
        # host-mapped FP8 tables stage half the bytes of bf16 ones
        hb = E.engram_workspace_size(E.Plan.from_workload(wl, host_tables=True), min(wl.n_tok, 4096))
        hf = E.engram_workspace_size(E.Plan.from_workload(wl.with_(table_dtype="fp8"), host_tables=True),
                                     min(wl.n_tok, 4096))
        assert hf < hb
    p = _plan()
    assert E.engram_workspace_size(p, 1000) < E.engram_workspace_size(p, 2000)
    assert E.engram_workspace_size(p, 0) >= 0


def test_hash_multipliers_are_odd_and_seeded():
    p1, p2 = _plan(hash_seed=1), _plan(hash_seed=2)
    m1 = [p1.plan.mult[h][i] for h in range(4) for i in range(2)]
    m2 = [p2.plan.mult[h][i] for h in range(4) for i in range(2)]
    assert all(x & 1 for x in m1) and m1 != m2


def test_invalid_calls_fail_on_host_without_launching():
    lib = E.lib
    p = _plan()
    launches0 = E.kernel_launches()
    # uninitialised plan
    bad = _native.engram_plan()
    assert lib.engram_hash(C.byref(bad), None, 1, 1, None, None, None) == E.ENGRAM_ERR_INVALID_ARG
    assert "engram_init" in E.last_error()
    # NULL outputs / negative sizes
    assert lib.engram_hash(p, None, 1, 4, None, None, None) == E.ENGRAM_ERR_INVALID_ARG
    assert lib.engram_hash(p, None, -1, 4, None, None, None) == E.ENGRAM_ERR_INVALID_ARG
    assert lib.engram_gather(p, None, None, -5, None, None) == E.ENGRAM_ERR_INVALID_ARG
    # misaligned table pointer
    tabs = (C.c_void_p * 4)(16, 32, 48, 65)
    assert lib.engram_gather(p, C.c_void_p(16), tabs, 3, C.c_void_p(16), None) == E.ENGRAM_ERR_INVALID_ARG
    assert "aligned" in E.last_error()
    # missing weights
    w = _native.engram_weights()
    assert lib.engram_gate_conv(p, C.byref(w), None, None, 1, 1, None, None, None, None, 0, None) \
        == E.ENGRAM_ERR_INVALID_ARG
    # empty calls are no-ops and succeed without a device
    assert lib.engram_hash(p, None, 0, 5, None, None, None) == E.ENGRAM_OK
    assert lib.engram_gather(p, None, None, 0, None, None) == E.ENGRAM_OK
    assert lib.engram_remap(p, None, 0, None, None, None) == E.ENGRAM_OK
    # nothing above reached a kernel launch: the library's own launch count is unchanged
    assert E.kernel_launches() == launches0


def test_workspace_too_small_is_rejected():
    p = _plan()
    ws = E.engram_workspace_size(p, 512)
    w = _native.engram_weights(*[C.c_void_p(256 * (i + 1)) for i in range(6)])
    rc = E.lib.engram_gate_conv(p, C.byref(w), C.c_void_p(256), C.c_void_p(512), 1, 512, None,
                                C.c_void_p(768), None, C.c_void_p(1024), ws - 1, None)
    assert rc == E.ENGRAM_ERR_INVALID_ARG and "workspace" in E.last_error()


def test_product_has_no_oracle_dependency():
    """The CUDA path never imports or links the oracle (the oracle is test infrastructure)."""
    pkg = os.path.dirname(E.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text and "liboracle" not in text


def test_branches_default_and_workspace_growth():
    assert _plan(num_branches=0).num_branches == 1      # a zeroed field reads as one branch
    assert _plan().num_branches == 1
    p1, p4 = _plan(num_branches=1), _plan(num_branches=4)
    assert p4.num_branches == 4 and p4.mem_dim == p1.mem_dim
    # more key tiles (partial sums) and per-branch gate scalars
    assert E.engram_workspace_size(p4, 4096) > E.engram_workspace_size(p1, 4096)
    wl = synth.get_workload("layer2560x4")
    assert E.Plan.from_workload(wl).num_branches == 4 and wl.h_rows == 4 * wl.n_tok


def test_row_cache_arguments_rejected_on_host():
    p = _plan()
    c = _native.engram_row_cache()
    for h in range(4):
        c.data[h] = c.tags[h] = c.claim[h] = 256 * (h + 1)
    for bad in (0, 3, 6, (1 << 32) + 1):
        c.slots = bad
        assert E.lib.engram_row_cache_reset(p, C.byref(c), None) == E.ENGRAM_ERR_INVALID_ARG
        assert "power of two" in E.last_error()
    c.slots = 64
    c.tags[2] = 0
    assert E.lib.engram_row_cache_reset(p, C.byref(c), None) == E.ENGRAM_ERR_INVALID_ARG
    assert E.lib.engram_row_cache_reset(p, None, None) == E.ENGRAM_ERR_INVALID_ARG
    # an empty batch is a no-op even without a device
    assert E.lib.engram_stage_rows_cached(p, None, 0, None, None, None, 1, None, None, None, None, None,
                                          None) == E.ENGRAM_OK


def test_cache_model_policy():
    """The host model used by the GPU cache tests: hits pin slots; the smallest row wins a
    free slot; rows outside the table never enter."""
    from cache_model import CacheModel
    import numpy as np
    m = CacheModel(1, 4, [100])
    assert m.step(np.array([[1], [5], [9], [2]])) == [0]      # 1, 5, 9 share slot 1: 1 wins
    assert m.tags[0].tolist() == [0, 2, 3, 0]
    # 1 hits and pins slot 1 (5 may not replace it); 6 replaces 2 in slot 2; 101 is outside
    assert m.step(np.array([[5], [1], [6], [101]])) == [1]
    assert m.tags[0].tolist() == [0, 2, 7, 0]


def test_packed_weights_size_and_validation():
    p = _plan()                                   # d_h 256, d_m 128: 2 row tiles x 2 k-blocks
    assert E.engram_packed_weights_size(p) == 2 * 2 * 32768
    assert E.engram_packed_weights_size(_plan(hidden_dim=384)) == 0
    assert E.engram_packed_weights_size(_plan(num_branches=3)) == 4 * 2 * 32768
    w = _native.engram_weights(*[C.c_void_p(256 * (i + 1)) for i in range(6)])
    w.w_packed = 4096 + 8                         # misaligned
    rc = E.lib.engram_gate_conv(p, C.byref(w), C.c_void_p(256), C.c_void_p(512), 1, 4, None,
                                C.c_void_p(768), None, C.c_void_p(1024), 1 << 20, None)
    assert rc == E.ENGRAM_ERR_INVALID_ARG and "w_packed" in E.last_error()
    p384 = _plan(hidden_dim=384)
    w.w_packed = 4096
    rc = E.lib.engram_gate_conv(p384, C.byref(w), C.c_void_p(256), C.c_void_p(512), 1, 4, None,
                                C.c_void_p(768), None, C.c_void_p(1024), 1 << 20, None)
    assert rc == E.ENGRAM_ERR_INVALID_ARG and "packed" in E.last_error()
    assert E.lib.engram_pack_weights(p384, C.c_void_p(256), C.c_void_p(512), C.c_void_p(768), 1 << 20,
                                     None) == E.ENGRAM_ERR_UNSUPPORTED



def test_forward_path_selection():
    """engram_forward_path (host only): which kernels a forward call runs."""
    P = E.engram_forward_path
    PAIR = E.ENGRAM_PATH_PAIR_MMA
    ROW = E.ENGRAM_PATH_ROW_ORDER
    RO = E.ENGRAM_FLAG_ROW_ORDER_GATHER
    for name in ("prefill20m", "layer2560"):
        wl = synth.get_workload(name)
        # prefill: hash kernel, gather kernel (token order), projection on CTA pairs
        # (d_h % 256 == 0, enough tiles)
        assert P(E.Plan.from_workload(wl), wl.B, wl.T) == PAIR
        assert P(E.Plan.from_workload(wl, flags=E.ENGRAM_FLAG_SINGLE_CTA_MMA), wl.B, wl.T) == 0
        assert P(E.Plan.from_workload(wl, flags=RO), wl.B, wl.T) == PAIR | ROW   # 524,288 rows
        assert P(E.Plan.from_workload(wl.with_(table_dtype="fp8")), wl.B, wl.T) == PAIR
    p16 = _plan(heads_per_order=8, table_rows=[10007] * 16, row_dim=64, hidden_dim=2560)
    assert P(p16, 1, 1100) == 0            # 5 x 20 tiles: too few for the pairs
    p16r = _plan(heads_per_order=8, table_rows=[10007] * 16, row_dim=64, hidden_dim=2560, flags=RO)
    assert P(p16r, 1, 4096) == PAIR | ROW   # 65,536 rows: row order from here when asked for
    assert P(p16r, 1, 4095) == PAIR
    # the bulk-copy gather, when asked for, on the hash + gather path only (not with row order,
    # not with the fused decode lookup, not for FP8 rows)
    BG = E.ENGRAM_FLAG_BULK_GATHER
    pf = synth.get_workload("prefill20m")
    assert P(E.Plan.from_workload(pf, flags=BG), pf.B, pf.T) == PAIR | E.ENGRAM_PATH_BULK_GATHER
    assert P(E.Plan.from_workload(pf, flags=BG | RO), pf.B, pf.T) == PAIR | ROW
    assert not P(E.Plan.from_workload(pf.with_(table_dtype="fp8"), flags=BG), pf.B, pf.T) & E.ENGRAM_PATH_BULK_GATHER
    dec = synth.get_workload("decode20m")
    assert not P(E.Plan.from_workload(dec, flags=BG), dec.B, 1) & E.ENGRAM_PATH_BULK_GATHER
    assert not P(_plan(hidden_dim=384), 8, 4096) & PAIR
    # decode-sized batches: one lookup kernel, split-K projection
    dec = synth.get_workload("decode20m")
    assert P(E.Plan.from_workload(dec), dec.B, 1) == E.ENGRAM_PATH_FUSED_LOOKUP | E.ENGRAM_PATH_SPLIT_K | PAIR
    assert (P(E.Plan.from_workload(dec, flags=E.ENGRAM_FLAG_SINGLE_CTA_MMA), dec.B, 1)
            == E.ENGRAM_PATH_FUSED_LOOKUP | E.ENGRAM_PATH_SPLIT_K)
    # host-mapped tables: distinct rows staged into HBM first
    hp = synth.get_workload("hostpinned20m")
    assert P(E.Plan.from_workload(hp, host_tables=True), hp.B, 1) & E.ENGRAM_PATH_STAGED_ROWS
    # host tables never take the row-ordered HBM gather (their rows are staged and deduplicated)
    assert P(E.Plan.from_workload(hp, host_tables=True, flags=RO), 64, 128) & (E.ENGRAM_PATH_STAGED_ROWS | ROW) == (
        E.ENGRAM_PATH_STAGED_ROWS)
    assert not P(E.Plan.from_workload(hp, host_tables=True, flags=RO), 64, 8192) & ROW
    with pytest.raises(E.EngramError):
        P(p16, -1, 4)


def test_selftest_and_synchronize_validate_on_host():
    p = _plan()
    w = _native.engram_weights(*[C.c_void_p(256 * (i + 1)) for i in range(6)])
    ws = E.engram_workspace_size(p, 512)
    launches0 = E.kernel_launches()
    for lim in (0, 999, 10 ** 9 + 1):
        rc = E.lib.engram_selftest_wait_timeout(p, C.byref(w), C.c_void_p(256), C.c_void_p(512), 512,
                                                C.c_void_p(1024), ws, lim, None)
        assert rc == E.ENGRAM_ERR_INVALID_ARG and "wait_limit_ns" in E.last_error()
    rc = E.lib.engram_selftest_wait_timeout(p, C.byref(w), C.c_void_p(256), C.c_void_p(512), 512,
                                            C.c_void_p(1024), ws - 1, 10 ** 6, None)
    assert rc == E.ENGRAM_ERR_INVALID_ARG and "workspace" in E.last_error()
    assert E.kernel_launches() == launches0
