"""The workloads the lookup is exercised and measured on (shapes, seeds, distributions).

Geometry follows the pages' model where it fixes it (hidden 2560; 2-gram and 3-gram heads;
prime-sized bf16 tables; ~20M rows x 2560 = 51.2B parameters = ~95.4 GiB) and the stated
workload list otherwise.  Seeds: ids 1000+c, tables 2000+c, weights 3000+c, hidden and
decode state 4000+c for workload c.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import numpy as np

from .fill import FillSpec, fp8_scale_for_sigma
from .streams import zipf_ids, uniform_ids, remap_table, phrase_stream


def is_prime(n: int) -> bool:
    if n < 2:
        return False
    if n % 2 == 0:
        return n == 2
    f = 3
    while f * f <= n:
        if n % f == 0:
            return False
        f += 2
    return True


def largest_prime_below(n: int) -> int:
    p = n - 1
    while not is_prime(p):
        p -= 1
    return p


# tensor ids within a weight / hidden seed
T_WK, T_WV, T_CONV_W, T_H, T_STATE = 100, 101, 102, 103, 104


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    vocab_in: int
    vocab_out: int          # V' (compressed); pad id = V'
    B: int
    T: int
    orders: Tuple[int, ...]
    K: int
    primes: Tuple[int, ...]  # one per table, order-major then head-minor
    d_e: int
    d_h: int
    ids_kind: str = "zipf"   # zipf | uniform | phrases
    zipf_s: float = 1.1
    identity_remap: bool = False
    decode: bool = False     # history + conv state carried across calls
    host_tables: bool = False
    hash_seed: int = 0x5EED
    eps: float = 1e-6
    conv_kernel: int = 4
    sigma_table: float = 0.02
    sigma_w: float = 0.02
    sigma_h: float = 1.0
    sigma_conv: float = 0.25
    index: int = 0
    table_dtype: str = "bf16"  # bf16 | fp8 (e4m3 codes with one dequantisation scale per table)
    branches: int = 1          # M: residual-stream branches, each with its own key projection

    @property
    def H(self) -> int:
        return len(self.orders) * self.K

    @property
    def d_m(self) -> int:
        return self.H * self.d_e

    @property
    def n_tok(self) -> int:
        return self.B * self.T

    @property
    def h_rows(self) -> int:
        """Rows of the hidden-state (and output) matrix: one per (token, branch)."""
        return self.n_tok * self.branches

    @property
    def conv_dilation(self) -> int:
        return max(self.orders)

    @property
    def hist_len(self) -> int:
        return max(self.orders) - 1

    @property
    def state_len(self) -> int:
        return (self.conv_kernel - 1) * self.conv_dilation

    @property
    def pad_id(self) -> int:
        return self.vocab_out

    @property
    def table_elem_bytes(self) -> int:
        return 1 if self.table_dtype == "fp8" else 2

    @property
    def table_bytes(self) -> int:
        return sum(self.primes) * self.d_e * self.table_elem_bytes

    def seeds(self):
        c = self.index
        return dict(ids=1000 + c, tables=2000 + c, weights=3000 + c, hidden=4000 + c)

    # ---- fill specs -------------------------------------------------------------------
    def table_spec(self, h: int) -> FillSpec:
        return FillSpec(self.seeds()["tables"], h, self.sigma_table)

    def table_sigma(self, h: int) -> float:
        """FP8 tables: table h is dequantised to ~N(0, sigma_h^2), sigma_h growing with h so that
        every table has its own scale."""
        return self.sigma_table * (1.0 + 0.125 * h)

    def table_scale(self, h: int):
        """Dequantisation scale of FP8 table h (float32)."""
        return fp8_scale_for_sigma(self.table_sigma(h))

    def wk_spec(self) -> FillSpec:
        """W_k as [branches * d_h, d_m] (the key projections of the branches stacked)."""
        return FillSpec(self.seeds()["weights"], T_WK, self.sigma_w)

    def wv_spec(self) -> FillSpec:
        return FillSpec(self.seeds()["weights"], T_WV, self.sigma_w)

    def conv_spec(self) -> FillSpec:
        return FillSpec(self.seeds()["weights"], T_CONV_W, self.sigma_conv)

    def h_spec(self, step: int = 0) -> FillSpec:
        return FillSpec(self.seeds()["hidden"] + 1_000_003 * step, T_H, self.sigma_h)

    def state_spec(self) -> FillSpec:
        return FillSpec(self.seeds()["hidden"], T_STATE, 1.0)

    # ---- host-side inputs -------------------------------------------------------------
    def remap(self) -> np.ndarray:
        if self.identity_remap:
            return np.arange(self.vocab_in, dtype=np.int32)
        return remap_table(self.vocab_in, self.vocab_out, self.seeds()["ids"] + 500)

    def ids(self, step: int = 0) -> np.ndarray:
        seed = self.seeds()["ids"] + 7 * step
        shape = (self.B, self.T)
        if self.ids_kind == "uniform":
            return uniform_ids(self.vocab_in, shape, seed)
        if self.ids_kind == "phrases":
            return phrase_stream(self.vocab_in, self.zipf_s, self.B, self.T, seed)
        return zipf_ids(self.vocab_in, self.zipf_s, shape, seed)

    def history(self) -> Optional[np.ndarray]:
        """Decode: the 2 remapped ids before the first step, drawn from the same stream."""
        if not self.decode:
            return None
        prev = zipf_ids(self.vocab_in, self.zipf_s, (self.B, self.hist_len), self.seeds()["ids"] + 99991)
        return self.remap()[prev].astype(np.int32)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


P_C1 = (10007, 10009, 10037, 10039)
P_1M = largest_prime_below(1_000_000)      # 999,983
P_10M = largest_prime_below(10_000_000)    # 9,999,991
P_20M = largest_prime_below(20_000_000)    # 19,999,999

WORKLOADS = {
    "tiny": Workload(
        name="tiny", index=0,
        description="vocab 1,000 remapped to 770; 1x512 Zipf(1.1); orders {2,3}, K=2; "
                    "4 prime tables x 32 dims; memory 128; hidden 256",
        vocab_in=1000, vocab_out=770, B=1, T=512, orders=(2, 3), K=2, primes=P_C1,
        d_e=32, d_h=256),
    "layer2560": Workload(
        name="layer2560", index=1,
        description="vocab 128,000 remapped to 98,560; 8x4096 Zipf(1.1); orders {2,3}, K=8; "
                    "16 tables of 999,983 rows x 160 dims; memory 2560; hidden 2560",
        vocab_in=128_000, vocab_out=98_560, B=8, T=4096, orders=(2, 3), K=8,
        primes=(P_1M,) * 16, d_e=160, d_h=2560),
    "decode20m": Workload(
        name="decode20m", index=2,
        description="vocab 248,320 (no compression); 256 sequences x 1 token, 2-id history; "
                    "orders {2,3}, K=1; 2 tables of 9,999,991 rows x 2560 dims (95.4 GiB); hidden 2560",
        vocab_in=248_320, vocab_out=248_320, B=256, T=1, orders=(2, 3), K=1,
        primes=(P_10M,) * 2, d_e=2560, d_h=2560, identity_remap=True, decode=True),
    "prefill20m": Workload(
        name="prefill20m", index=3,
        description="as decode20m tables; 32x8192 tokens, Zipf(1.1) with 30% of positions "
                    "copied from 5,000 seeded phrases",
        vocab_in=248_320, vocab_out=248_320, B=32, T=8192, orders=(2, 3), K=1,
        primes=(P_10M,) * 2, d_e=2560, d_h=2560, identity_remap=True, ids_kind="phrases"),
    "hostpinned20m": Workload(
        name="hostpinned20m", index=4,
        description="as decode20m tables, kept in pinned host memory; 64 tokens per step; "
                    "ids uniform or Zipf(1.3)",
        vocab_in=248_320, vocab_out=248_320, B=64, T=1, orders=(2, 3), K=1,
        primes=(P_10M,) * 2, d_e=2560, d_h=2560, identity_remap=True, decode=True,
        host_tables=True, ids_kind="uniform", zipf_s=1.3),
    # the pages' own geometry: 8 two-gram + 8 three-gram heads, ~20M rows per table, 160
    # values per row (16 x 20M x 160 = 51.2B parameters, ~102 GB): small rows spread over a
    # huge table, the hardest case for DRAM efficiency of the row gather
    # the layer2560 workload on a 4-branch residual stream: tables, memory vectors and the
    # value projection shared, one key projection per branch
    "layer2560x4": Workload(
        name="layer2560x4", index=6,
        description="as layer2560 with 4 residual-stream branches (hidden states [32768, 4, 2560], "
                    "4 key projections, shared value projection)",
        vocab_in=128_000, vocab_out=98_560, B=8, T=4096, orders=(2, 3), K=8,
        primes=(P_1M,) * 16, d_e=160, d_h=2560, branches=4),
    "ngram16x20m": Workload(
        name="ngram16x20m", index=5,
        description="vocab 248,320 (no compression); 8x4096 Zipf(1.1); orders {2,3}, K=8; "
                    "16 tables of 19,999,999 rows x 160 dims (102 GB); memory 2560; hidden 2560",
        vocab_in=248_320, vocab_out=248_320, B=8, T=4096, orders=(2, 3), K=8,
        primes=(P_20M,) * 16, d_e=160, d_h=2560, identity_remap=True),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]
