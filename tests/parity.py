"""Shared helpers for GPU-vs-oracle parity tests (no arithmetic of the method).

Tolerances (stated by the benchmark plan and written here once):
  bf16 inputs, fp32 accumulation: max-abs <= 1e-2 and relative L2 <= 2e-3;
  fp32 inputs: max-abs <= 1e-5.
"""
import numpy as np
import torch

import oracle as orc
from workloads import BLOCK_SIZE

BF16_MAX_ABS = 1e-2
BF16_REL_L2 = 2e-3
F32_MAX_ABS = 1e-5


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff)) / denom if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_parity(got, ref, dtype, what=""):
    max_abs, rel = errors(got, ref)
    if dtype == torch.float32:
        assert max_abs <= F32_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {F32_MAX_ABS}"
    else:
        assert max_abs <= BF16_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {BF16_MAX_ABS}"
        assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e} > {BF16_REL_L2}"
    return max_abs, rel


def oracle_gqa_sequences(inp, seqs):
    """Oracle output for the listed sequences of a (device-resident) workload.

    Gathers each sequence's owned blocks with torch indexing (plumbing, not
    the library), lays them out with an identity table and runs the oracle.
    Returns {b: array [H_q][d]}.
    """
    res = {}
    for b in seqs:
        T = int(inp.seq_list[b])
        nb = max(1, (T + BLOCK_SIZE - 1) // BLOCK_SIZE)
        ids = inp.block_table[b, :nb].long()
        if (ids < 0).any():
            # blocks outside a window may be deliberately invalid: gather only
            # the valid ones and zero-fill the rest (never visible)
            valid = ids >= 0
            kc = torch.zeros((nb,) + tuple(inp.k_cache.shape[1:]),
                             dtype=inp.k_cache.dtype, device=inp.k_cache.device)
            vc = torch.zeros_like(kc)
            kc[valid] = inp.k_cache[ids[valid]]
            vc[valid] = inp.v_cache[ids[valid]]
        else:
            kc = inp.k_cache[ids]
            vc = inp.v_cache[ids]
        q = inp.q[b:b + 1]
        table = torch.arange(nb, dtype=torch.int32).reshape(1, nb)
        out = orc.decode_gqa(q.cpu(), kc.cpu(), vc.cpu(),
                             torch.tensor([T], dtype=torch.int32), table,
                             inp.scale, window=inp.window)
        res[b] = out[0]
    return res


def oracle_mla_sequences(inp, seqs):
    res = {}
    for b in seqs:
        T = int(inp.seq_list[b])
        nb = max(1, (T + BLOCK_SIZE - 1) // BLOCK_SIZE)
        ids = inp.block_table[b, :nb].long()
        cache = inp.latent_cache[ids]
        table = torch.arange(nb, dtype=torch.int32).reshape(1, nb)
        out = orc.decode_mla(inp.q_lat[b:b + 1].cpu(), inp.q_rope[b:b + 1].cpu(),
                             cache.cpu(), torch.tensor([T], dtype=torch.int32),
                             table, inp.scale)
        res[b] = out[0]
    return res
