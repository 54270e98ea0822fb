"""ctypes binding of the C ABI in include/engram.h (argument marshalling only).

Every function here forwards to the same-named entry point of ``libengram.so``; all the
computation runs in the library's CUDA kernels.  There is no fallback: if the shared
library is missing or cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libengram.so")

ENGRAM_OK = 0
ENGRAM_ERR_INVALID_ARG = -1
ENGRAM_ERR_UNSUPPORTED = -2
ENGRAM_ERR_CUDA = -3
ENGRAM_ERR_TIMEOUT = -5
ENGRAM_STATUS_BAD_TOKEN = 0x1
ENGRAM_STATUS_BAD_ROW = 0x2
ENGRAM_STATUS_WAIT_TIMEOUT = 0x4
ENGRAM_MAX_ORDERS = 4
ENGRAM_MAX_TABLES = 32
ENGRAM_MAX_BRANCHES = 8
ENGRAM_FORWARD_STAGES = 4
ENGRAM_TABLES_DEVICE = 0
ENGRAM_TABLES_HOST_MAPPED = 1
ENGRAM_NOALLOC_SCRATCH_BYTES = 32 << 20
ENGRAM_FLAG_SINGLE_CTA_MMA = 0x4
ENGRAM_FLAG_ROW_ORDER_GATHER = 0x8
ENGRAM_FLAG_BULK_GATHER = 0x10
ENGRAM_PATH_FUSED_LOOKUP = 0x1
ENGRAM_PATH_STAGED_ROWS = 0x2
ENGRAM_PATH_SPLIT_K = 0x8
ENGRAM_PATH_PAIR_MMA = 0x10
ENGRAM_PATH_ROW_ORDER = 0x20
ENGRAM_PATH_BULK_GATHER = 0x40
ENGRAM_TABLE_BF16 = 0
ENGRAM_TABLE_FP8_E4M3 = 1

_ERRNAMES = {-1: "ENGRAM_ERR_INVALID_ARG", -2: "ENGRAM_ERR_UNSUPPORTED", -3: "ENGRAM_ERR_CUDA",
             -5: "ENGRAM_ERR_TIMEOUT"}


class EngramError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_ERRNAMES.get(code, code)}: {msg}")
        self.code = code


class engram_config(C.Structure):
    _fields_ = [
        ("num_orders", C.c_int32),
        ("orders", C.c_int32 * ENGRAM_MAX_ORDERS),
        ("heads_per_order", C.c_int32),
        ("table_rows", C.c_int64 * ENGRAM_MAX_TABLES),
        ("row_dim", C.c_int32),
        ("hidden_dim", C.c_int32),
        ("vocab_in", C.c_int32),
        ("vocab_out", C.c_int32),
        ("pad_id", C.c_int32),
        ("conv_kernel", C.c_int32),
        ("conv_dilation", C.c_int32),
        ("table_location", C.c_int32),
        ("hash_seed", C.c_uint64),
        ("eps", C.c_float),
        ("flags", C.c_int32),
        ("table_dtype", C.c_int32),
        ("table_scale", C.c_float * ENGRAM_MAX_TABLES),
        ("num_branches", C.c_int32),
        ("reserved", C.c_int32 * 4),
    ]


class engram_plan(C.Structure):
    _fields_ = [
        ("cfg", engram_config),
        ("mult", (C.c_uint64 * ENGRAM_MAX_ORDERS) * ENGRAM_MAX_TABLES),
        ("num_tables", C.c_int32),
        ("mem_dim", C.c_int32),
        ("hist_len", C.c_int32),
        ("state_len", C.c_int32),
        ("magic", C.c_uint32),
        ("num_branches", C.c_int32),
        ("reserved", C.c_int32 * 2),
    ]


class engram_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w_k", "w_v", "gamma_q", "gamma_k", "gamma_c", "conv_w", "w_packed")]


class engram_row_cache(C.Structure):
    _fields_ = [
        ("data", C.c_void_p * ENGRAM_MAX_TABLES),
        ("tags", C.c_void_p * ENGRAM_MAX_TABLES),
        ("claim", C.c_void_p * ENGRAM_MAX_TABLES),
        ("slots", C.c_int64),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                          "(run __graft_entry__.build() or python -m hashed_gram_embedding_remap_b200.build)")
    L = C.CDLL(LIB_PATH)
    P, i32, i64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    sig = {
        "engram_init": (C.c_int, [P, P]),
        "engram_workspace_size": (sz, [P, i64]),
        "engram_remap": (C.c_int, [P, P, i64, P, P, P]),
        "engram_hash": (C.c_int, [P, P, i32, i32, P, P, P]),
        "engram_advance_history": (C.c_int, [P, P, i32, i32, P, P]),
        "engram_gather": (C.c_int, [P, P, P, i64, P, P]),
        "engram_stage_rows": (C.c_int, [P, P, i64, P, P, i32, P, P, P, P]),
        "engram_stage_rows_from_ids": (C.c_int, [P, P, P, i32, i32, P, P, P, i32, P, P, P, P, P]),
        "engram_gather_bounded": (C.c_int, [P, P, P, i64, i64, P, P]),
        "engram_row_cache_reset": (C.c_int, [P, P, P]),
        "engram_packed_weights_size": (sz, [P]),
        "engram_pack_weights": (C.c_int, [P, P, P, P, sz, P]),
        "engram_stage_rows_cached": (C.c_int, [P, P, i64, P, P, P, i32, P, P, P, P, P, P]),
        "engram_gate_conv": (C.c_int, [P, P, P, P, i32, i32, P, P, P, P, sz, P]),
        "engram_forward": (C.c_int, [P, P, P, P, P, i32, i32, P, P, P, P, P, P, sz, P, P]),
        "engram_gate_conv_noalloc": (C.c_int, [P, P, P, P, i32, i32, P, P, P, P]),
        "engram_device_status": (C.c_int, [P, C.c_int]),
        "engram_forward_path": (C.c_int, [P, i32, i32, P]),
        "engram_synchronize": (C.c_int, [P]),
        "engram_selftest_wait_timeout": (C.c_int, [P, P, P, P, i64, P, sz, C.c_uint64, P]),
        "engram_last_error": (C.c_char_p, []),
        "engram_version": (C.c_char_p, []),
        "engram_sizeof": (sz, [C.c_char_p]),
        "engram_kernel_launches": (C.c_uint64, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    for name, cls in (("engram_config", engram_config), ("engram_plan", engram_plan),
                      ("engram_weights", engram_weights), ("engram_row_cache", engram_row_cache)):
        n = L.engram_sizeof(name.encode())
        if n != C.sizeof(cls):
            raise ImportError(f"ABI mismatch: sizeof({name}) is {n} in the library, {C.sizeof(cls)} here")
    return L


lib = _load()


def last_error() -> str:
    return lib.engram_last_error().decode()


def version() -> str:
    return lib.engram_version().decode()


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far (engram_kernel_launches)."""
    return int(lib.engram_kernel_launches())


def _check(rc: int):
    if rc != ENGRAM_OK:
        raise EngramError(rc, last_error())


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)


# ---------------------------------------------------------------------------------------
class Plan:
    """A validated lookup configuration (engram_plan), built by engram_init."""

    def __init__(self, *, orders: Sequence[int], heads_per_order: int, table_rows: Sequence[int],
                 row_dim: int, hidden_dim: int, vocab_in: int, vocab_out: int, hash_seed: int,
                 eps: float = 1e-6, conv_kernel: int = 4, table_location: int = ENGRAM_TABLES_DEVICE,
                 flags: int = 0, table_dtype: int = ENGRAM_TABLE_BF16,
                 table_scale: Optional[Sequence[float]] = None, num_branches: int = 1):
        cfg = engram_config()
        cfg.num_orders = len(orders)
        for i, o in enumerate(orders):
            cfg.orders[i] = int(o)
        cfg.heads_per_order = int(heads_per_order)
        for i, p in enumerate(table_rows):
            cfg.table_rows[i] = int(p)
        cfg.row_dim = int(row_dim)
        cfg.hidden_dim = int(hidden_dim)
        cfg.vocab_in = int(vocab_in)
        cfg.vocab_out = int(vocab_out)
        cfg.pad_id = int(vocab_out)
        cfg.conv_kernel = int(conv_kernel)
        cfg.conv_dilation = int(max(orders)) if len(orders) else 0
        cfg.table_location = int(table_location)
        cfg.hash_seed = int(hash_seed) & 0xFFFFFFFFFFFFFFFF
        cfg.eps = float(eps)
        cfg.flags = int(flags)
        cfg.table_dtype = int(table_dtype)
        cfg.num_branches = int(num_branches)
        for i, sc in enumerate(table_scale or ()):
            cfg.table_scale[i] = float(sc)
        self.cfg = cfg
        self.plan = engram_plan()
        _check(lib.engram_init(C.byref(cfg), C.byref(self.plan)))

    @classmethod
    def from_workload(cls, wl, **kw) -> "Plan":
        loc = ENGRAM_TABLES_HOST_MAPPED if kw.pop("host_tables", False) else ENGRAM_TABLES_DEVICE
        fp8 = getattr(wl, "table_dtype", "bf16") == "fp8"
        return cls(orders=wl.orders, heads_per_order=wl.K, table_rows=wl.primes, row_dim=wl.d_e,
                   hidden_dim=wl.d_h, vocab_in=wl.vocab_in, vocab_out=wl.vocab_out,
                   hash_seed=wl.hash_seed, eps=wl.eps, conv_kernel=wl.conv_kernel,
                   table_location=loc, table_dtype=ENGRAM_TABLE_FP8_E4M3 if fp8 else ENGRAM_TABLE_BF16,
                   table_scale=[float(wl.table_scale(h)) for h in range(wl.H)] if fp8 else None,
                   num_branches=getattr(wl, "branches", 1), **kw)

    @property
    def num_tables(self) -> int:
        return self.plan.num_tables

    @property
    def mem_dim(self) -> int:
        return self.plan.mem_dim

    @property
    def num_branches(self) -> int:
        return self.plan.num_branches

    @property
    def hist_len(self) -> int:
        return self.plan.hist_len

    @property
    def state_len(self) -> int:
        return self.plan.state_len

    @property
    def _as_parameter_(self):
        return C.byref(self.plan)


class Weights:
    """Device tensors of the gate and conv, bundled as engram_weights.  `packed`: optional
    copy of [W_k ; W_v] made by pack_weights (streamed by the projections instead)."""

    def __init__(self, w_k, w_v, gamma_q, gamma_k, gamma_c, conv_w, packed=None):
        self.tensors = (w_k, w_v, gamma_q, gamma_k, gamma_c, conv_w, packed)
        names = ("w_k", "w_v", "gamma_q", "gamma_k", "gamma_c", "conv_w")
        ptrs = [_ptr(t, _BF16, n) for t, n in zip(self.tensors[:6], names)]
        ptrs.append(None if packed is None else _ptr(packed, None, "packed"))
        self.struct = engram_weights(*ptrs)

    @property
    def _as_parameter_(self):
        return C.byref(self.struct)


def engram_packed_weights_size(plan: Plan) -> int:
    return int(lib.engram_packed_weights_size(plan))


def pack_weights(plan: Plan, w_k: torch.Tensor, w_v: torch.Tensor, stream=None) -> torch.Tensor:
    """The projection weights re-laid as pre-swizzled 256 x 64 tiles (engram_pack_weights)."""
    n = engram_packed_weights_size(plan)
    if n == 0:
        raise EngramError(ENGRAM_ERR_UNSUPPORTED, "no packed form for this hidden size")
    out = torch.empty(n, dtype=torch.uint8, device=w_k.device)
    _check(lib.engram_pack_weights(plan, _ptr(w_k, _BF16, "w_k"), _ptr(w_v, _BF16, "w_v"),
                                   _ptr(out, None, "packed"), n, _stream(stream)))
    return out


def _table_array(tables, plan: Optional[Plan] = None):
    """Pointer array of tables (tensors or raw addresses).  With a plan, tensors must hold the
    plan's table element type: 2-byte bf16 patterns, or 1-byte e4m3 codes."""
    want = None
    if plan is not None:
        want = 1 if plan.cfg.table_dtype == ENGRAM_TABLE_FP8_E4M3 else 2
    arr = (C.c_void_p * len(tables))()
    for i, t in enumerate(tables):
        if not isinstance(t, int) and want is not None and t.element_size() != want:
            raise ValueError(f"tables[{i}] has {t.element_size()}-byte elements; the plan's tables have {want}")
        arr[i] = t if isinstance(t, int) else t.data_ptr()
    return arr


# ---------------------------------------------------------------------------------------
def engram_workspace_size(plan: Plan, n_tok: int) -> int:
    return int(lib.engram_workspace_size(plan, int(n_tok)))


def engram_remap(plan: Plan, ids: torch.Tensor, remap: torch.Tensor, out: torch.Tensor, stream=None):
    _check(lib.engram_remap(plan, _ptr(ids, torch.int32, "ids"), ids.numel(),
                            _ptr(remap, torch.int32, "remap"), _ptr(out, torch.int32, "out"),
                            _stream(stream)))


def engram_hash(plan: Plan, ids_remapped: torch.Tensor, idx: torch.Tensor,
                history: Optional[torch.Tensor] = None, stream=None):
    B, T = ids_remapped.shape
    _check(lib.engram_hash(plan, _ptr(ids_remapped, torch.int32, "ids_remapped"), B, T,
                           _ptr(history, torch.int32, "history"),
                           _ptr(idx, (torch.int32, torch.uint32), "idx"), _stream(stream)))


def engram_advance_history(plan: Plan, ids_remapped: torch.Tensor, history: torch.Tensor, stream=None):
    B, T = ids_remapped.shape
    _check(lib.engram_advance_history(plan, _ptr(ids_remapped, torch.int32, "ids_remapped"), B, T,
                                      _ptr(history, torch.int32, "history"), _stream(stream)))


def engram_gather(plan: Plan, idx: torch.Tensor, tables, m: torch.Tensor, stream=None, rows_bound: int = 0):
    """rows_bound > 0: every table holds only that many rows (device staging buffers from
    engram_stage_rows); row ids at or beyond it read a zero row and raise the status bit."""
    arr = _table_array(tables, plan)
    if rows_bound:
        _check(lib.engram_gather_bounded(plan, _ptr(idx, (torch.int32, torch.uint32), "idx"), arr, idx.shape[0],
                                         int(rows_bound), _ptr(m, _BF16, "m"), _stream(stream)))
        return
    _check(lib.engram_gather(plan, _ptr(idx, (torch.int32, torch.uint32), "idx"), arr, idx.shape[0],
                             _ptr(m, _BF16, "m"), _stream(stream)))


def engram_stage_rows(plan: Plan, idx: torch.Tensor, tables, staging, staged_idx: torch.Tensor,
                      unique_rows: torch.Tensor, n_unique: torch.Tensor, stream=None):
    """Copy each distinct row the batch needs from (host-mapped) tables into device staging."""
    n_tok = idx.shape[0]
    cap = staging[0].shape[0]
    _check(lib.engram_stage_rows(plan, _ptr(idx, (torch.int32, torch.uint32), "idx"), n_tok,
                                 _table_array(tables, plan), _table_array(staging, plan), cap,
                                 _ptr(staged_idx, (torch.int32, torch.uint32), "staged_idx"),
                                 _ptr(unique_rows, (torch.int32, torch.uint32), "unique_rows"),
                                 _ptr(n_unique, torch.int32, "n_unique"), _stream(stream)))


def engram_stage_rows_from_ids(plan: Plan, ids: torch.Tensor, tables, staging, idx: torch.Tensor,
                               staged_idx: torch.Tensor, unique_rows: torch.Tensor, n_unique: torch.Tensor,
                               remap: Optional[torch.Tensor] = None, history: Optional[torch.Tensor] = None,
                               stream=None):
    """Hash the ids (into idx) and stage the batch's distinct rows from the (host-mapped)
    tables, in one kernel for decode-sized batches."""
    B, T = ids.shape
    cap = staging[0].shape[0]
    _check(lib.engram_stage_rows_from_ids(plan, _ptr(ids, torch.int32, "ids"), _ptr(remap, torch.int32, "remap"),
                                          B, T, _ptr(history, torch.int32, "history"), _table_array(tables, plan),
                                          _table_array(staging, plan), cap,
                                          _ptr(idx, (torch.int32, torch.uint32), "idx"),
                                          _ptr(staged_idx, (torch.int32, torch.uint32), "staged_idx"),
                                          _ptr(unique_rows, (torch.int32, torch.uint32), "unique_rows"),
                                          _ptr(n_unique, torch.int32, "n_unique"), _stream(stream)))


def _check_rows(plan: Plan, n_tok: int, **tensors):
    """h / out / delta hold one d_h-wide row per (token, branch)."""
    want = n_tok * plan.num_branches * plan.cfg.hidden_dim
    for name, t in tensors.items():
        if t is not None and t.numel() != want:
            raise ValueError(f"{name} has {t.numel()} elements; {n_tok} tokens x {plan.num_branches} branches x "
                             f"{plan.cfg.hidden_dim} need {want}")


class RowCache:
    """Device buffers of an HBM row cache (engram_row_cache) for the plan's tables: per table
    `slots` rows of the table element type, uint32 tags and claims.  Created empty."""

    def __init__(self, plan: Plan, slots: int, device="cuda", stream=None):
        if slots < 1 or slots & (slots - 1):
            raise ValueError("slots must be a power of two")
        elem = torch.uint8 if plan.cfg.table_dtype == ENGRAM_TABLE_FP8_E4M3 else torch.bfloat16
        H, d_e = plan.num_tables, plan.cfg.row_dim
        self.data = [torch.empty((slots, d_e), dtype=elem, device=device) for _ in range(H)]
        self.tags = [torch.empty((slots,), dtype=torch.int32, device=device) for _ in range(H)]
        self.claim = [torch.empty((slots,), dtype=torch.int32, device=device) for _ in range(H)]
        self.struct = engram_row_cache()
        for hh in range(H):
            self.struct.data[hh] = self.data[hh].data_ptr()
            self.struct.tags[hh] = self.tags[hh].data_ptr()
            self.struct.claim[hh] = self.claim[hh].data_ptr()
        self.struct.slots = int(slots)
        self.plan = plan
        self.reset(stream)

    def reset(self, stream=None):
        _check(lib.engram_row_cache_reset(self.plan, C.byref(self.struct), _stream(stream)))

    @property
    def _as_parameter_(self):
        return C.byref(self.struct)


def engram_stage_rows_cached(plan: Plan, idx: torch.Tensor, tables, cache: RowCache, staging,
                             staged_idx: torch.Tensor, unique_rows: torch.Tensor, n_unique: torch.Tensor,
                             row_flags: torch.Tensor, n_hits: torch.Tensor, stream=None):
    """engram_stage_rows with the HBM row cache in front of the (host-mapped) tables; n_hits
    accumulates the distinct rows served from the cache."""
    n_tok = idx.shape[0]
    cap = staging[0].shape[0]
    _check(lib.engram_stage_rows_cached(plan, _ptr(idx, (torch.int32, torch.uint32), "idx"), n_tok,
                                        _table_array(tables, plan), cache, _table_array(staging, plan), cap,
                                        _ptr(staged_idx, (torch.int32, torch.uint32), "staged_idx"),
                                        _ptr(unique_rows, (torch.int32, torch.uint32), "unique_rows"),
                                        _ptr(n_unique, torch.int32, "n_unique"),
                                        _ptr(row_flags, (torch.int32, torch.uint32), "row_flags"),
                                        _ptr(n_hits, torch.int32, "n_hits"), _stream(stream)))


def engram_gate_conv(plan: Plan, weights: Weights, h: torch.Tensor, m: torch.Tensor, B: int, T: int,
                     out: torch.Tensor, workspace: torch.Tensor, conv_state: Optional[torch.Tensor] = None,
                     delta_dbg: Optional[torch.Tensor] = None, stream=None):
    _check_rows(plan, B * T, h=h, out=out, delta_dbg=delta_dbg)
    _check(lib.engram_gate_conv(plan, weights, _ptr(h, _BF16, "h"), _ptr(m, _BF16, "m"), B, T,
                                _ptr(conv_state, _BF16, "conv_state"), _ptr(out, _BF16, "out"),
                                _ptr(delta_dbg, torch.float32, "delta_dbg"),
                                _ptr(workspace, None, "workspace"),
                                workspace.numel() * workspace.element_size(), _stream(stream)))


def engram_gate_conv_noalloc(plan: Plan, weights: Weights, h: torch.Tensor, m: torch.Tensor, B: int, T: int,
                             out: torch.Tensor, conv_state: Optional[torch.Tensor] = None,
                             delta_dbg: Optional[torch.Tensor] = None, stream=None):
    """engram_gate_conv without a workspace, for hosts that cannot allocate device memory
    (their scratch is the library's fixed per-GPU array of ENGRAM_NOALLOC_SCRATCH_BYTES)."""
    _check_rows(plan, B * T, h=h, out=out, delta_dbg=delta_dbg)
    _check(lib.engram_gate_conv_noalloc(plan, weights, _ptr(h, _BF16, "h"), _ptr(m, _BF16, "m"), B, T,
                                        _ptr(conv_state, _BF16, "conv_state"), _ptr(out, _BF16, "out"),
                                        _ptr(delta_dbg, torch.float32, "delta_dbg"), _stream(stream)))


def engram_forward(plan: Plan, weights: Weights, tables, ids: torch.Tensor, h: torch.Tensor,
                   out: torch.Tensor, workspace: torch.Tensor, remap: Optional[torch.Tensor] = None,
                   history: Optional[torch.Tensor] = None, conv_state: Optional[torch.Tensor] = None,
                   delta_dbg: Optional[torch.Tensor] = None, stream=None, stage_events=None):
    B, T = ids.shape
    _check_rows(plan, B * T, h=h, out=out, delta_dbg=delta_dbg)
    arr = _table_array(tables, plan)
    ev = None
    if stage_events is not None:
        if len(stage_events) != ENGRAM_FORWARD_STAGES + 1:
            raise ValueError(f"stage_events needs {ENGRAM_FORWARD_STAGES + 1} events")
        ev = (C.c_void_p * len(stage_events))(*[e._as_parameter_.value for e in stage_events])
    _check(lib.engram_forward(plan, weights, arr, _ptr(ids, torch.int32, "ids"),
                              _ptr(remap, torch.int32, "remap"), B, T,
                              _ptr(history, torch.int32, "history"), _ptr(conv_state, _BF16, "conv_state"),
                              _ptr(h, _BF16, "h"), _ptr(out, _BF16, "out"),
                              _ptr(delta_dbg, torch.float32, "delta_dbg"), _ptr(workspace, None, "workspace"),
                              workspace.numel() * workspace.element_size(), _stream(stream), ev))


def engram_device_status(clear: bool = True) -> int:
    s = C.c_uint32(0)
    _check(lib.engram_device_status(C.byref(s), int(clear)))
    return int(s.value)


def engram_forward_path(plan: Plan, B: int, T: int) -> int:
    """ENGRAM_PATH_* bits: which kernels engram_forward runs for B sequences of T tokens."""
    bits = C.c_uint32(0)
    _check(lib.engram_forward_path(plan, int(B), int(T), C.byref(bits)))
    return int(bits.value)


def engram_synchronize(stream=None):
    """Wait for the stream; raises EngramError(ENGRAM_ERR_TIMEOUT) if a bounded wait inside a
    kernel gave up since the device status word was last cleared."""
    _check(lib.engram_synchronize(_stream(stream)))


def engram_selftest_wait_timeout(plan: Plan, weights: Weights, h: torch.Tensor, m: torch.Tensor,
                                 workspace: torch.Tensor, wait_limit_ns: int, stream=None):
    """Run the projection with its loads stalled so that every bounded wait runs out after
    wait_limit_ns (the failure path of engram_selftest_wait_timeout)."""
    _check(lib.engram_selftest_wait_timeout(plan, weights, _ptr(h, _BF16, "h"), _ptr(m, _BF16, "m"), m.shape[0],
                                            _ptr(workspace, None, "workspace"),
                                            workspace.numel() * workspace.element_size(), int(wait_limit_ns),
                                            _stream(stream)))


def alloc_workspace(plan: Plan, n_tok: int, device="cuda") -> torch.Tensor:
    """A workspace tensor of the size engram_workspace_size reports (torch allocations are
    at least 256-byte aligned)."""
    n = engram_workspace_size(plan, n_tok)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)
