"""Seeded synthetic inputs for paged decode attention.

This module is shared by the CUDA-path tests, the oracle tests and the
benchmark.  It only draws random numbers and lays them out in the library's
storage format; it contains none of the attention arithmetic.

Recipe (one ``torch.Generator`` per workload, seed = 20261202 + index):
  * q, K, V ~ N(0, 1) drawn in fp32, then rounded (RNE) to the workload dtype;
    the MLA workload scales every value by 1/sqrt(576) before rounding;
  * paged cache of 64-token blocks; the physical blocks of all sequences are
    a random permutation of the pool (``torch.randperm``) unless an identity
    ("contiguous") table is asked for; unused table entries hold -1;
  * ragged lengths T_b ~ U[1024, 131072] (``torch.randint``).
Small inputs are drawn on the CPU generator; full-size inputs may be drawn
directly on a CUDA generator with the same seed (a different but equally
fixed stream of numbers).
"""
import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

BLOCK_SIZE = 64
SEED_BASE = 20261202


@dataclass(frozen=True)
class GQAConfig:
    name: str
    B: int
    H_q: int
    H_kv: int
    d: int
    seq_lens: Optional[List[int]] = None   # None -> every sequence has length T
    T: int = 0
    dtype: torch.dtype = torch.bfloat16
    window: int = 0
    sink: int = 0                          # global tokens kept visible (with a window)
    ring: int = 0                          # ring table of this many blocks after the sink ones
    kv_fp8: bool = False                   # fp8 (E4M3 + per-row scale) cache, bf16 q
    contiguous: bool = False               # identity block table
    seed: int = SEED_BASE
    ragged: Optional[tuple] = None         # (lo, hi) inclusive range of T_b
    n_global: int = 0                      # explicit global positions per sequence (global_rows)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


@dataclass(frozen=True)
class MLAConfig:
    name: str
    B: int
    H: int = 128
    d_c: int = 512
    d_r: int = 64
    T: int = 8192
    seq_lens: Optional[List[int]] = None
    value_scale: float = 1.0 / math.sqrt(576.0)
    seed: int = SEED_BASE + 4
    dtype: torch.dtype = torch.bfloat16
    kv_fp8: bool = False                   # fp8 latent cache (E4M3 codes + row scales)

    @property
    def scale(self) -> float:
        # per-head content + rope key width d_c' + d_R = 128 + 64
        return 1.0 / math.sqrt(192.0)


# The five workloads of the benchmark plan, by what they are.
TINY = GQAConfig("tiny_gqa_fp32_B1_Hq4_Hkv2_d16_T64", B=1, H_q=4, H_kv=2,
                 d=16, T=64, dtype=torch.float32, contiguous=True,
                 seed=SEED_BASE + 0)
LLAMA3_8B = GQAConfig("llama3_8b_gqa_bf16_B16_Hq32_Hkv8_d128_T4096", B=16,
                      H_q=32, H_kv=8, d=128, T=4096, seed=SEED_BASE + 1)


def sweep_config(H_kv: int, B: int) -> GQAConfig:
    return GQAConfig(f"sweep_bf16_B{B}_Hq32_Hkv{H_kv}_d128_T32768", B=B,
                     H_q=32, H_kv=H_kv, d=128, T=32768, seed=SEED_BASE + 2)


SWEEP = [sweep_config(hkv, b) for hkv in (32, 8, 1) for b in (1, 8, 32)]


def ragged_config(window: int) -> GQAConfig:
    tag = "full" if window <= 0 else f"w{window}"
    return GQAConfig(f"ragged_gqa_bf16_B8_Hq24_Hkv4_d256_{tag}", B=8, H_q=24,
                     H_kv=4, d=256, ragged=(1024, 131072), window=window,
                     seed=SEED_BASE + 3)


RAGGED_FULL = ragged_config(0)
RAGGED_WINDOW = ragged_config(4096)
# The Llama-3-8B shape over an fp8 (E4M3 + per-row scale) KV cache.
LLAMA3_8B_FP8 = GQAConfig("llama3_8b_gqa_fp8kv_B16_Hq32_Hkv8_d128_T4096", B=16, H_q=32,
                          H_kv=8, d=128, T=4096, kv_fp8=True, seed=SEED_BASE + 1)
# MQA at B = 8, T = 32768 over an fp8 cache (the tensor-core fp8 kernel's shape).
MQA_B8_FP8 = GQAConfig("sweep_fp8_B8_Hq32_Hkv1_d128_T32768", B=8, H_q=32, H_kv=1, d=128,
                       T=32768, kv_fp8=True, seed=SEED_BASE + 2)
# Window plus 64 global tokens on the same shape; and the same on a ring table
# that keeps only the 1 sink block and the 65 blocks a 4096-key window can reach.
RAGGED_WINDOW_SINK = GQAConfig("ragged_gqa_bf16_B8_Hq24_Hkv4_d256_w4096_g64", B=8, H_q=24,
                               H_kv=4, d=256, ragged=(1024, 131072), window=4096, sink=64,
                               seed=SEED_BASE + 3)
RAGGED_WINDOW_RING = GQAConfig("ragged_gqa_bf16_B8_Hq24_Hkv4_d256_w4096_g64_ring65", B=8,
                               H_q=24, H_kv=4, d=256, ragged=(1024, 131072), window=4096,
                               sink=64, ring=65, seed=SEED_BASE + 3)
RAGGED_WINDOW_GLOBAL = GQAConfig("ragged_gqa_bf16_B8_Hq24_Hkv4_d256_w4096_G16", B=8, H_q=24,
                                 H_kv=4, d=256, ragged=(1024, 131072), window=4096,
                                 n_global=16, seed=SEED_BASE + 3)
MLA_DSV2 = MLAConfig("mla_absorbed_bf16_B32_H128_dc512_dr64_T8192", B=32)
# The DeepSeek-V2 shape over an fp8 latent cache.
MLA_DSV2_FP8 = MLAConfig("mla_absorbed_fp8latent_B32_H128_dc512_dr64_T8192", B=32, kv_fp8=True)

WORKLOADS = {c.name: c for c in [TINY, LLAMA3_8B, *SWEEP, RAGGED_FULL,
                                 RAGGED_WINDOW, RAGGED_WINDOW_SINK, RAGGED_WINDOW_RING,
                                 RAGGED_WINDOW_GLOBAL, LLAMA3_8B_FP8, MQA_B8_FP8, MLA_DSV2,
                                 MLA_DSV2_FP8]}


def global_rows(seq_lens, n: int) -> torch.Tensor:
    """[B][n] int32 global positions: per sequence of T tokens the first 4
    positions and n - 4 positions spread evenly over [0, T) (a prompt's
    leading tokens and periodic summary tokens), ascending, -1 padded."""
    rows = []
    for T in seq_lens:
        pos = set(range(min(4, T))) | {T * k // (n - 3) for k in range(1, n - 3)}
        pos = sorted(p for p in pos if 0 <= p < T)[:n]
        rows.append(pos + [-1] * (n - len(pos)))
    return torch.tensor(rows, dtype=torch.int32)


def _generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def draw_seq_lens(cfg, g: torch.Generator) -> List[int]:
    if cfg.seq_lens is not None:
        return list(cfg.seq_lens)
    if getattr(cfg, "ragged", None):
        lo, hi = cfg.ragged
        t = torch.randint(lo, hi + 1, (cfg.B,), generator=g,
                          device=g.device)
        return [int(v) for v in t.cpu()]
    return [cfg.T] * cfg.B


def make_block_table(seq_lens, g: torch.Generator, contiguous=False,
                     extra_blocks_per_seq=0, pool_slack=0):
    """Block table [B][max_blocks] (int32, on the generator's device).

    Each sequence b owns ceil(T_b / 64) + extra_blocks_per_seq physical
    blocks.  Physical ids are a random permutation of a pool of all owned
    blocks plus ``pool_slack`` unowned ones, or consecutive ids when
    ``contiguous``.  Entries past a sequence's blocks are -1.
    Returns (table, num_blocks).
    """
    B = len(seq_lens)
    owned = [(t + BLOCK_SIZE - 1) // BLOCK_SIZE + extra_blocks_per_seq
             for t in seq_lens]
    max_blocks = max(1, max(owned) if owned else 1)
    total = sum(owned)
    num_blocks = total + pool_slack
    if contiguous:
        ids = torch.arange(num_blocks, dtype=torch.int64, device=g.device)
    else:
        ids = torch.randperm(num_blocks, generator=g, device=g.device)
    table = torch.full((B, max_blocks), -1, dtype=torch.int32,
                       device=g.device)
    off = 0
    for b, n in enumerate(owned):
        if n:
            table[b, :n] = ids[off:off + n].to(torch.int32)
        off += n
    return table, max(num_blocks, 1)


def randn(shape, g: torch.Generator, dtype, scale: float = 1.0):
    x = torch.randn(shape, generator=g, device=g.device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


@dataclass
class GQAInputs:
    cfg: GQAConfig
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    seq_lens: torch.Tensor
    block_table: torch.Tensor
    num_blocks: int
    window: int
    scale: float
    seq_list: List[int] = field(default_factory=list)
    k_scale: Optional[torch.Tensor] = None   # fp8 cache: [num_blocks][H_kv][64] row scales
    v_scale: Optional[torch.Tensor] = None
    global_pos: Optional[torch.Tensor] = None   # [B][n_global] int32 (cfg.n_global > 0)

    def to(self, device):
        mv = (lambda t: None if t is None else t.to(device))
        return GQAInputs(self.cfg, self.q.to(device), self.k_cache.to(device),
                         self.v_cache.to(device), self.seq_lens.to(device),
                         self.block_table.to(device), self.num_blocks,
                         self.window, self.scale, list(self.seq_list),
                         mv(self.k_scale), mv(self.v_scale), mv(self.global_pos))


def make_gqa_inputs(cfg: GQAConfig, device="cpu", seed: Optional[int] = None,
                    extra_blocks_per_seq=0, pool_slack=0,
                    window: Optional[int] = None) -> GQAInputs:
    g = _generator(cfg.seed if seed is None else seed, device)
    seq = draw_seq_lens(cfg, g)
    if cfg.ring > 0:
        # Every sequence owns the sink blocks and the ring slots, whatever T.
        slots = (cfg.sink + BLOCK_SIZE - 1) // BLOCK_SIZE + cfg.ring
        table, nblk = make_block_table([slots * BLOCK_SIZE] * cfg.B, g, cfg.contiguous,
                                       extra_blocks_per_seq, pool_slack)
    else:
        table, nblk = make_block_table(seq, g, cfg.contiguous,
                                       extra_blocks_per_seq, pool_slack)
    q = randn((cfg.B, cfg.H_q, cfg.d), g, cfg.dtype)
    sl = torch.tensor(seq, dtype=torch.int32, device=g.device)
    win = cfg.window if window is None else window
    if cfg.kv_fp8:
        # Stand-in quantised rows: uniform E4M3 codes (the two NaN codes
        # replaced by +-448) with row scales of N(0,1)-like rows (amax ~3).
        shape = (nblk, cfg.H_kv, BLOCK_SIZE, cfg.d)
        codes = []
        for _ in range(2):
            c = torch.randint(0, 256, shape, generator=g, device=g.device, dtype=torch.int32)
            c = torch.where((c & 0x7F) == 0x7F, c - 1, c)
            codes.append(c.to(torch.uint8))
        scales = [(torch.rand(shape[:3], generator=g, device=g.device) * 2 + 2) / 448
                  for _ in range(2)]
        return GQAInputs(cfg, q, codes[0], codes[1], sl, table, nblk, win, cfg.scale, seq,
                         scales[0], scales[1])
    k = randn((nblk, cfg.H_kv, BLOCK_SIZE, cfg.d), g, cfg.dtype)
    v = randn((nblk, cfg.H_kv, BLOCK_SIZE, cfg.d), g, cfg.dtype)
    gp = global_rows(seq, cfg.n_global).to(g.device) if cfg.n_global > 0 else None
    return GQAInputs(cfg, q, k, v, sl, table, nblk, win, cfg.scale, seq, global_pos=gp)


@dataclass
class MLAInputs:
    cfg: MLAConfig
    q_lat: torch.Tensor
    q_rope: torch.Tensor
    latent_cache: torch.Tensor
    seq_lens: torch.Tensor
    block_table: torch.Tensor
    num_blocks: int
    scale: float
    seq_list: List[int] = field(default_factory=list)
    latent_scale: Optional[torch.Tensor] = None   # fp8 cache: [num_blocks][64] row scales

    def to(self, device):
        return MLAInputs(self.cfg, self.q_lat.to(device),
                         self.q_rope.to(device), self.latent_cache.to(device),
                         self.seq_lens.to(device), self.block_table.to(device),
                         self.num_blocks, self.scale, list(self.seq_list),
                         None if self.latent_scale is None else self.latent_scale.to(device))


def make_mla_inputs(cfg: MLAConfig, device="cpu", seed: Optional[int] = None,
                    extra_blocks_per_seq=0) -> MLAInputs:
    g = _generator(cfg.seed if seed is None else seed, device)
    seq = draw_seq_lens(cfg, g)
    table, nblk = make_block_table(seq, g, False, extra_blocks_per_seq)
    vs = cfg.value_scale
    q_lat = randn((cfg.B, cfg.H, cfg.d_c), g, cfg.dtype, vs)
    q_rope = randn((cfg.B, cfg.H, cfg.d_r), g, cfg.dtype, vs)
    sl = torch.tensor(seq, dtype=torch.int32, device=g.device)
    if cfg.kv_fp8:
        # Stand-in quantised rows: uniform E4M3 codes (the two NaN codes
        # replaced by +-448) with row scales of rows like N(0,1)*value_scale
        # (amax ~3.2 value_scale).
        shape = (nblk, BLOCK_SIZE, cfg.d_c + cfg.d_r)
        c = torch.randint(0, 256, shape, generator=g, device=g.device, dtype=torch.int32)
        c = torch.where((c & 0x7F) == 0x7F, c - 1, c).to(torch.uint8)
        sc = (torch.rand(shape[:2], generator=g, device=g.device) * 0.8 + 2.8) * vs / 448
        return MLAInputs(cfg, q_lat, q_rope, c, sl, table, nblk, cfg.scale, seq, sc)
    cache = randn((nblk, BLOCK_SIZE, cfg.d_c + cfg.d_r), g, cfg.dtype, vs)
    return MLAInputs(cfg, q_lat, q_rope, cache, sl, table, nblk, cfg.scale,
                     seq)


@dataclass
class MLAAbsorbInputs:
    q_c: torch.Tensor     # [B][H][d_h] per-head content query (before absorption)
    U_K: torch.Tensor     # [H][d_c][d_h] key up-projection, k^C_j = c_j U^K_h
    U_V: torch.Tensor     # [H][d_c][d_v] value up-projection, v_j = c_j U^V_h

    def to(self, device):
        return MLAAbsorbInputs(self.q_c.to(device), self.U_K.to(device), self.U_V.to(device))


def make_mla_absorb_inputs(cfg: MLAConfig, d_h=128, d_v=128, device="cpu",
                           seed: Optional[int] = None) -> MLAAbsorbInputs:
    """Random stand-ins for the per-head projections on either side of the
    absorbed decode (no trained weights exist here): q_c ~ N(0,1), U^K ~
    N(0,1)/(2 sqrt(d_h)) (q_c (U^K)^T has standard deviation 1/2, so even its
    extremes over a full batch stay below ~2.5, where bf16 storage keeps the
    1e-2 max-abs bar), U^V ~ N(0,1)/sqrt(d_c); bf16 like the cache."""
    g = _generator((cfg.seed if seed is None else seed) + 7919, device)
    q_c = randn((cfg.B, cfg.H, d_h), g, cfg.dtype, 1.0)
    U_K = randn((cfg.H, cfg.d_c, d_h), g, cfg.dtype, 0.5 / math.sqrt(d_h))
    U_V = randn((cfg.H, cfg.d_c, d_v), g, cfg.dtype, 1.0 / math.sqrt(cfg.d_c))
    return MLAAbsorbInputs(q_c, U_K, U_V)
