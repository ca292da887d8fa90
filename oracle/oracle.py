"""ctypes binding of the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the library.  Inputs are CPU torch
tensors (fp32, bf16 or fp64) or numpy arrays (fp32/fp64); outputs are numpy
fp64 arrays.  Marshalling only -- all arithmetic lives in oracle.c.
"""
import ctypes
import os

import numpy as np
import torch

from . import build_oracle

_F32, _BF16, _F64 = 0, 1, 2
_lib = None


def _load():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        lib = ctypes.CDLL(path)
        c_p, c_i, c_d = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        lib.orc_decode_gqa.argtypes = [c_p] * 7 + [c_i] * 7 + [c_d, c_i, c_i]
        lib.orc_decode_gqa.restype = c_i
        lib.orc_decode_gqa_vis.argtypes = ([c_p] * 7 + [c_i] * 7 + [c_d, c_i, c_i, c_i, c_i] +
                                           [c_p, c_i])
        lib.orc_decode_gqa_vis.restype = c_i
        lib.orc_e4m3_value.argtypes = [c_i]
        lib.orc_e4m3_value.restype = c_d
        lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        lib.orc_e4m3_encode.restype = c_i
        lib.orc_quantize_rows_e4m3.argtypes = [c_p, c_i, c_i, c_p, c_p]
        lib.orc_quantize_rows_e4m3.restype = None
        lib.orc_decode_mla.argtypes = [c_p] * 7 + [c_i] * 7 + [c_d, c_i]
        lib.orc_decode_mla.restype = c_i
        lib.orc_mla_explicit.argtypes = [c_p] * 8 + [c_i] * 8 + [c_d]
        lib.orc_mla_explicit.restype = c_i
        lib.orc_bytes_kv.argtypes = [c_d] * 5
        lib.orc_bytes_kv.restype = c_d
        lib.orc_bytes_mla.argtypes = [c_d] * 5
        lib.orc_bytes_mla.restype = c_d
        lib.orc_visible_range.argtypes = [c_i, c_i, ctypes.POINTER(c_i),
                                          ctypes.POINTER(c_i)]
        lib.orc_visible_range.restype = None
        lib.orc_slot_offset.argtypes = [c_p, c_i, c_i, c_i, c_i, c_i, c_i, c_i,
                                        ctypes.POINTER(ctypes.c_int64)]
        lib.orc_slot_offset.restype = c_i
        lib.orc_set_threads.argtypes = [c_i]
        lib.orc_set_threads.restype = None
        lib.orc_get_threads.argtypes = []
        lib.orc_get_threads.restype = c_i
        _lib = lib
    return _lib


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def get_threads() -> int:
    return int(_load().orc_get_threads())


def _as_input(x):
    """(keepalive, pointer, dtype code) for a CPU tensor / numpy array."""
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    if x.device.type != "cpu":
        raise ValueError("oracle inputs must live in host memory")
    x = x.contiguous()
    code = {torch.float32: _F32, torch.bfloat16: _BF16,
            torch.float64: _F64}.get(x.dtype)
    if code is None:
        raise TypeError(f"oracle does not read dtype {x.dtype}")
    return x, x.data_ptr(), code


def _as_i32(x):
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    x = x.to("cpu", torch.int32).contiguous()
    return x, x.data_ptr()


def visible_range(T: int, window: int):
    lo, hi = ctypes.c_int(), ctypes.c_int()
    _load().orc_visible_range(int(T), int(window), ctypes.byref(lo),
                              ctypes.byref(hi))
    return lo.value, hi.value


def decode_gqa(q, k_cache, v_cache, seq_lens, block_table, scale, window=0,
               return_probs=False):
    """out [B][H_q][d] (fp64) = decode attention over the paged K/V cache.

    q [B][H_q][d]; k_cache/v_cache [num_blocks][H_kv][block_size][d];
    seq_lens [B]; block_table [B][max_blocks].  With return_probs, also the
    softmax weights [B][H_q][max_T] (zero outside each visible range).
    """
    B, H_q, d = q.shape
    _, H_kv, bs, d2 = k_cache.shape
    assert d2 == d and tuple(v_cache.shape) == tuple(k_cache.shape)
    qa, qp, dt = _as_input(q)
    ka, kp, dt_k = _as_input(k_cache)
    va, vp, dt_v = _as_input(v_cache)
    if not (dt == dt_k == dt_v):
        raise TypeError("q, k_cache and v_cache must share one dtype")
    sl, slp = _as_i32(seq_lens)
    bt, btp = _as_i32(block_table)
    max_blocks = bt.shape[1]
    out = np.zeros((B, H_q, d), dtype=np.float64)
    max_T = int(sl.max().item()) if return_probs and B > 0 else 0
    probs = np.zeros((B, H_q, max_T), dtype=np.float64) if return_probs else None
    rc = _load().orc_decode_gqa(
        qp, kp, vp, slp, btp, out.ctypes.data,
        probs.ctypes.data if probs is not None else None, max_T,
        B, H_q, H_kv, d, bs, max_blocks, float(scale), int(window), dt)
    if rc != 0:
        raise RuntimeError(f"oracle decode_gqa failed with status {rc}")
    return (out, probs) if return_probs else out


def decode_gqa_vis(q, k_cache, v_cache, seq_lens, block_table, scale, window=0,
                   sink=0, ring=0, return_probs=False, global_pos=None):
    """decode_gqa with global tokens and a ring-buffer table (fp64).

    Key j < T is visible when window <= 0, j >= T - window, j < sink, j is in
    the sequence's global set, or T - 1 is in it (attention-head article, §3:
    a global query sees the whole history).  global_pos: int [B][n_g], each
    row ascending and read up to its first entry that does not exceed the one
    before (pad with -1).  With ring > 0 and no global set, logical block i
    lives in table slot i for i < A = ceil(sink / block_size) (the sink
    blocks) and in slot A + i % ring after them.  With ring > 0 and a global
    set (sink must be 0), slots [0, n_g) are global slots -- slot k holds the
    block of position global_pos[b][k] -- a visible key in a block before the
    window's first block is read through its own position's global slot, and
    block i from the window's first block on sits in slot n_g + i % ring; a
    global query with T > window is refused (the ring no longer holds the
    history it would see).  Same arrays as decode_gqa.
    """
    B, H_q, d = q.shape
    _, H_kv, bs, d2 = k_cache.shape
    assert d2 == d and tuple(v_cache.shape) == tuple(k_cache.shape)
    qa, qp, dt = _as_input(q)
    ka, kp, dt_k = _as_input(k_cache)
    va, vp, dt_v = _as_input(v_cache)
    if not (dt == dt_k == dt_v):
        raise TypeError("q, k_cache and v_cache must share one dtype")
    sl, slp = _as_i32(seq_lens)
    bt, btp = _as_i32(block_table)
    out = np.zeros((B, H_q, d), dtype=np.float64)
    max_T = int(sl.max().item()) if return_probs and B > 0 else 0
    probs = np.zeros((B, H_q, max_T), dtype=np.float64) if return_probs else None
    if global_pos is None:
        gp, gpp, n_g = None, None, 0
    else:
        gp, gpp = _as_i32(global_pos)
        if gp.ndim != 2 or gp.shape[0] != B:
            raise ValueError("global_pos must be [B][n_g]")
        n_g = gp.shape[1]
    rc = _load().orc_decode_gqa_vis(
        qp, kp, vp, slp, btp, out.ctypes.data,
        probs.ctypes.data if probs is not None else None, max_T,
        B, H_q, H_kv, d, bs, bt.shape[1], float(scale), int(window), int(sink), int(ring), dt,
        gpp, n_g)
    if rc != 0:
        raise RuntimeError(f"oracle decode_gqa_vis failed with status {rc}")
    return (out, probs) if return_probs else out


def decode_mla(q_lat, q_rope, latent_cache, seq_lens, block_table, scale,
               return_probs=False):
    """z [B][H][d_c] (fp64): absorbed MLA decode over the paged latent cache.

    q_lat [B][H][d_c]; q_rope [B][H][d_r];
    latent_cache [num_blocks][block_size][d_c + d_r].
    """
    B, H, d_c = q_lat.shape
    d_r = q_rope.shape[2]
    _, bs, width = latent_cache.shape
    assert width == d_c + d_r
    qa, qp, dt = _as_input(q_lat)
    ra, rp, dt_r = _as_input(q_rope)
    ca, cp, dt_c = _as_input(latent_cache)
    if not (dt == dt_r == dt_c):
        raise TypeError("q_lat, q_rope and latent_cache must share one dtype")
    sl, slp = _as_i32(seq_lens)
    bt, btp = _as_i32(block_table)
    out = np.zeros((B, H, d_c), dtype=np.float64)
    max_T = int(sl.max().item()) if return_probs and B > 0 else 0
    probs = np.zeros((B, H, max_T), dtype=np.float64) if return_probs else None
    rc = _load().orc_decode_mla(
        qp, rp, cp, slp, btp, out.ctypes.data,
        probs.ctypes.data if probs is not None else None, max_T,
        B, H, d_c, d_r, bs, bt.shape[1], float(scale), dt)
    if rc != 0:
        raise RuntimeError(f"oracle decode_mla failed with status {rc}")
    return (out, probs) if return_probs else out


def mla_explicit(q_c, q_rope, latent_cache, seq_lens, block_table, U_K, U_V,
                 scale):
    """o [B][H][d_v] (fp64): MLA with per-head K/V expanded from the latents.

    q_c [B][H][d_h]; q_rope [B][H][d_r]; latent_cache [nb][bs][d_c+d_r];
    U_K [H][d_c][d_h]; U_V [H][d_c][d_v].  All fp64.
    """
    q_c = np.ascontiguousarray(q_c, dtype=np.float64)
    q_rope = np.ascontiguousarray(q_rope, dtype=np.float64)
    latent_cache = np.ascontiguousarray(latent_cache, dtype=np.float64)
    U_K = np.ascontiguousarray(U_K, dtype=np.float64)
    U_V = np.ascontiguousarray(U_V, dtype=np.float64)
    B, H, d_h = q_c.shape
    d_r = q_rope.shape[2]
    _, bs, width = latent_cache.shape
    d_c = width - d_r
    d_v = U_V.shape[2]
    sl, slp = _as_i32(seq_lens)
    bt, btp = _as_i32(block_table)
    out = np.zeros((B, H, d_v), dtype=np.float64)
    rc = _load().orc_mla_explicit(
        q_c.ctypes.data, q_rope.ctypes.data, latent_cache.ctypes.data, slp,
        btp, U_K.ctypes.data, U_V.ctypes.data, out.ctypes.data,
        B, H, d_c, d_r, d_h, d_v, bs, bt.shape[1], float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle mla_explicit failed with status {rc}")
    return out


def e4m3_table():
    """Values of the 256 OCP FP8 E4M3 codes (fp64; NaN for the two NaN codes)."""
    lib = _load()
    return np.array([lib.orc_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(x):
    """Nearest E4M3 code of fp32 x (ties to even, saturating at 448)."""
    return _load().orc_e4m3_encode(float(np.float32(x)))


def quantize_rows_e4m3(x):
    """(codes uint8 [..., d], scales fp32 [...]) of the fp8 cache row
    quantisation: scale = amax / 448, codes = E4M3(x * (448 / amax)) in fp32."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    d = x.shape[-1]
    rows = int(np.prod(x.shape[:-1])) if x.ndim > 1 else 1
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros(x.shape[:-1], dtype=np.float32)
    _load().orc_quantize_rows_e4m3(x.ctypes.data, rows, d, codes.ctypes.data,
                                   scales.ctypes.data)
    return codes, scales


def dequantize_e4m3(codes, scales):
    """fp64 cache rows: code value times its row scale."""
    return e4m3_table()[np.asarray(codes)] * np.asarray(scales, dtype=np.float64)[..., None]


def mla_absorb_q(q_c, U_K):
    """q_latent [B][H][d_c] (fp64) = q^C_h (U^K_h)^T per head: the key
    up-projection folded into the query (attention-head §5.2, absorption).

    q_c [B][H][d_h]; U_K [H][d_c][d_h] (k^C_j = c_j U^K_h).  A plain batched
    product; pinned by the absorbed == explicit invariant.
    """
    q_c = np.asarray(q_c, dtype=np.float64)
    U_K = np.asarray(U_K, dtype=np.float64)
    return np.einsum("bhi,hci->bhc", q_c, U_K)


def mla_project_out(z, U_V):
    """o [B][H][d_v] (fp64) = z_h U^V_h per head: the value up-projection
    applied after the attention in latent space (attention-head §5.2).

    z [B][H][d_c]; U_V [H][d_c][d_v].  A plain batched product; pinned by the
    absorbed == explicit invariant.
    """
    z = np.asarray(z, dtype=np.float64)
    U_V = np.asarray(U_V, dtype=np.float64)
    return np.einsum("bhc,hcv->bhv", z, U_V)


def bytes_kv(B, T, H_kv, d, s):
    return _load().orc_bytes_kv(float(B), float(T), float(H_kv), float(d),
                                float(s))


def bytes_mla(B, T, r, d_r, s):
    return _load().orc_bytes_mla(float(B), float(T), float(r), float(d_r),
                                 float(s))


def slot_offset(block_table, b, pos, block_size, n_heads, head, row_width):
    bt, btp = _as_i32(block_table)
    off = ctypes.c_int64()
    rc = _load().orc_slot_offset(btp, bt.shape[1], int(b), int(pos),
                                 int(block_size), int(n_heads), int(head),
                                 int(row_width), ctypes.byref(off))
    if rc != 0:
        raise ValueError("position outside the block table")
    return off.value


__all__ = [name for name in dir() if not name.startswith("_")
           and name not in ("ctypes", "os", "np", "torch", "build_oracle")]
