"""Paged decode attention on NVIDIA B200 -- thin Python binding of the C ABI.

The work happens in libattn_decode.so (hand-written sm_100a CUDA, declared in
include/attn_decode.h).  This module only marshals torch tensors into the
C calls: it checks dtypes, shapes and devices, passes raw device pointers and
the current CUDA stream, and raises AttnError on a failing status.  There is
no fallback: if the library is missing, ``load()`` raises.
"""
import ctypes
import os

import torch

from . import planner  # noqa: F401  (host model of the split partition)

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn_decode.so")
BLOCK_SIZE = 64

OK, ERR_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BAD_BLOCK, \
    ERR_BAD_SEQLEN = 0, -1, -2, -3, -4, -5, -6
F32, BF16, FP8_E4M3 = 0, 1, 2

# Every entry point include/attn_decode.h declares.
C_SYMBOLS = (
    "attn_decode_gqa", "attn_decode_mla", "kv_append", "kv_append_mla",
    "attn_decode_plan", "attn_decode_gqa_config", "attn_set_num_ctas",
    "attn_set_gqa_path", "attn_set_profile_events",
    "attn_debug_force_timeout", "attn_decode_last_error",
    "attn_status_string", "attn_version", "attn_decode_gqa_noalloc",
    "attn_mla_absorb_q", "attn_mla_project_out", "attn_decode_gqa_ext", "kv_append_ext",
    "attn_decode_gqa_fp8", "kv_append_fp8", "attn_decode_mla_fp8", "kv_append_mla_fp8",
)


class Visibility(ctypes.Structure):
    """attn_visibility: window, global (sink) tokens, ring table (blocks),
    explicit global positions (device int32 [B][n_global])."""
    _fields_ = [("window", ctypes.c_int), ("sink_tokens", ctypes.c_int),
                ("ring_blocks", ctypes.c_int), ("global_pos", ctypes.c_void_p),
                ("n_global", ctypes.c_int)]


def _visibility(window, sink_tokens, ring_blocks, global_pos=None, B=None):
    if global_pos is None:
        return Visibility(int(window), int(sink_tokens), int(ring_blocks), None, 0)
    if global_pos.dim() != 2 or (B is not None and global_pos.shape[0] != B):
        raise ValueError("global_pos must be [B][n_global]")
    return Visibility(int(window), int(sink_tokens), int(ring_blocks),
                      _dev(global_pos, "global_pos", torch.int32).value, int(global_pos.shape[1]))

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        name = load().attn_status_string(status).decode()
        super().__init__(f"{what}: {name} ({status})" if what else name)


def load():
    """Load libattn_decode.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m decode_attention_kv_paged_b200.build_lib` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    p, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_decode_gqa.argtypes = [p] * 6 + [i] * 4 + [f, i, p, i, i, i]
    lib.attn_decode_mla.argtypes = [p] * 6 + [i] * 4 + [f, p, i, i]
    lib.attn_decode_gqa_noalloc.argtypes = lib.attn_decode_gqa.argtypes
    lib.attn_decode_gqa_ext.argtypes = ([p] * 6 + [i] * 4 +
                                        [f, ctypes.POINTER(Visibility), p, i, i, i])
    lib.kv_append_ext.argtypes = [p] * 6 + [i] * 6 + [ctypes.POINTER(Visibility), p]
    lib.attn_decode_gqa_fp8.argtypes = ([p] * 8 + [i] * 4 +
                                        [f, ctypes.POINTER(Visibility), p, i, i])
    lib.kv_append_fp8.argtypes = [p] * 8 + [i] * 5 + [ctypes.POINTER(Visibility), p]
    lib.attn_decode_mla_fp8.argtypes = [p] * 7 + [i] * 4 + [f, p, i, i]
    lib.kv_append_mla_fp8.argtypes = [p] * 5 + [i] * 5 + [p]
    lib.attn_mla_absorb_q.argtypes = [p] * 3 + [i] * 4 + [p]
    lib.attn_mla_project_out.argtypes = [p] * 3 + [i] * 4 + [p]
    lib.kv_append.argtypes = [p] * 6 + [i] * 6 + [p]
    lib.kv_append_mla.argtypes = [p] * 4 + [i] * 5 + [p]
    lib.attn_decode_plan.argtypes = [p, i, i, i, i, i, p, p]
    lib.attn_decode_gqa_config.argtypes = [i] * 5 + [ctypes.POINTER(i)] * 3
    lib.attn_set_num_ctas.argtypes = [i]
    lib.attn_set_gqa_path.argtypes = [i]
    lib.attn_set_profile_events.argtypes = [p, p, i]
    lib.attn_debug_force_timeout.argtypes = [i, ctypes.c_longlong]
    lib.attn_decode_last_error.argtypes = [p]
    lib.attn_status_string.argtypes = [i]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    for name in C_SYMBOLS:
        fn = getattr(lib, name)
        if name != "attn_status_string":
            fn.restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status, what):
    if status != OK:
        raise AttnError(status, what)


def _stream_ptr(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _dtype_code(dt):
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {dt} (bf16 or fp32)")


def decode_gqa(q, k_cache, v_cache, seq_lens, block_table, scale, window=0,
               out=None, stream=None):
    """out [B][H_q][d] = paged decode attention (MHA/GQA/MQA, optional window).

    q [B][H_q][d]; k_cache, v_cache [num_blocks][H_kv][64][d] (bf16 or fp32);
    seq_lens int32 [B]; block_table int32 [B][max_blocks].
    """
    B, H_q, d = q.shape
    nblk, H_kv, bs, d2 = k_cache.shape
    if bs != BLOCK_SIZE or d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("cache must be [num_blocks][H_kv][64][d] for K and V")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B][max_blocks]")
    dt = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    rc = load().attn_decode_gqa(
        _dev(q, "q"), _dev(k_cache, "k_cache", q.dtype),
        _dev(v_cache, "v_cache", q.dtype), _dev(seq_lens, "seq_lens", torch.int32),
        _dev(block_table, "block_table", torch.int32), _dev(out, "out", q.dtype),
        B, H_q, H_kv, d, float(scale), int(window), _stream_ptr(stream),
        block_table.shape[1], nblk, dt)
    _check(rc, "attn_decode_gqa")
    return out


def decode_gqa_ext(q, k_cache, v_cache, seq_lens, block_table, scale, window=0,
                   sink_tokens=0, ring_blocks=0, out=None, stream=None, global_pos=None):
    """decode_gqa with global tokens and a ring-buffer block table: key
    j < T is visible when window <= 0, j >= T - window, j < sink_tokens, j is
    in the sequence's row of global_pos (int32 [B][n_global], ascending, -1
    padded), or T - 1 is in it (a global query sees everything); with
    ring_blocks > 0 logical block i lives in table slot i for the sink
    blocks and in slot A + i % ring_blocks after them (A = ceil(sink / 64));
    with ring_blocks > 0 and global_pos, slots [0, n_global) hold the blocks
    of the global positions (read for blocks before the window) and A =
    n_global."""
    B, H_q, d = q.shape
    nblk, H_kv, bs, d2 = k_cache.shape
    if bs != BLOCK_SIZE or d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("cache must be [num_blocks][H_kv][64][d] for K and V")
    dt = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    vis = _visibility(window, sink_tokens, ring_blocks, global_pos, B)
    rc = load().attn_decode_gqa_ext(
        _dev(q, "q"), _dev(k_cache, "k_cache", q.dtype),
        _dev(v_cache, "v_cache", q.dtype), _dev(seq_lens, "seq_lens", torch.int32),
        _dev(block_table, "block_table", torch.int32), _dev(out, "out", q.dtype),
        B, H_q, H_kv, d, float(scale), ctypes.byref(vis), _stream_ptr(stream),
        block_table.shape[1], nblk, dt)
    _check(rc, "attn_decode_gqa_ext")
    return out


def decode_gqa_fp8(q, k_cache, v_cache, k_scale, v_scale, seq_lens, block_table, scale,
                   window=0, sink_tokens=0, ring_blocks=0, out=None, stream=None,
                   global_pos=None):
    """out [B][H_q][d] (bf16) = decode attention over an fp8 cache: k_cache /
    v_cache uint8 E4M3 codes [num_blocks][H_kv][64][d], k_scale / v_scale
    fp32 row scales [num_blocks][H_kv][64] (value = code * row scale)."""
    B, H_q, d = q.shape
    nblk, H_kv, bs, d2 = k_cache.shape
    if bs != BLOCK_SIZE or d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("cache must be [num_blocks][H_kv][64][d] for K and V")
    if tuple(k_scale.shape) != (nblk, H_kv, bs) or tuple(v_scale.shape) != (nblk, H_kv, bs):
        raise ValueError("scales must be [num_blocks][H_kv][64]")
    bf, u8, f32 = torch.bfloat16, torch.uint8, torch.float32
    if out is None:
        out = torch.empty_like(q)
    vis = _visibility(window, sink_tokens, ring_blocks, global_pos, B)
    rc = load().attn_decode_gqa_fp8(
        _dev(q, "q", bf), _dev(k_cache, "k_cache", u8), _dev(v_cache, "v_cache", u8),
        _dev(k_scale, "k_scale", f32), _dev(v_scale, "v_scale", f32),
        _dev(seq_lens, "seq_lens", torch.int32), _dev(block_table, "block_table", torch.int32),
        _dev(out, "out", bf), B, H_q, H_kv, d, float(scale), ctypes.byref(vis),
        _stream_ptr(stream), block_table.shape[1], nblk)
    _check(rc, "attn_decode_gqa_fp8")
    return out


def kv_append_fp8(k_new, v_new, k_cache, v_cache, k_scale, v_scale, positions, block_table,
                  window=0, sink_tokens=0, ring_blocks=0, stream=None):
    """Quantise the current token's K/V rows (bf16 [B][H_kv][d]) to E4M3 with
    one scale per row (amax / 448) and write them at positions[b]."""
    B, H_kv, d = k_new.shape
    bf, u8, f32 = torch.bfloat16, torch.uint8, torch.float32
    vis = _visibility(window, sink_tokens, ring_blocks)
    rc = load().kv_append_fp8(
        _dev(k_new, "k_new", bf), _dev(v_new, "v_new", bf), _dev(k_cache, "k_cache", u8),
        _dev(v_cache, "v_cache", u8), _dev(k_scale, "k_scale", f32),
        _dev(v_scale, "v_scale", f32), _dev(positions, "positions", torch.int32),
        _dev(block_table, "block_table", torch.int32), B, H_kv, d, block_table.shape[1],
        k_cache.shape[0], ctypes.byref(vis), _stream_ptr(stream))
    _check(rc, "kv_append_fp8")


def decode_gqa_noalloc(q, k_cache, v_cache, seq_lens, block_table, scale,
                       window=0, out=None, stream=None):
    """decode_gqa through attn_decode_gqa_noalloc: same result, but the split
    scratch is the library's fixed device array, so the call never allocates
    device memory (for callers that must not allocate while running).  Calls
    share that array: keep them on one stream."""
    B, H_q, d = q.shape
    nblk, H_kv, bs, d2 = k_cache.shape
    if bs != BLOCK_SIZE or d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("cache must be [num_blocks][H_kv][64][d] for K and V")
    dt = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    rc = load().attn_decode_gqa_noalloc(
        _dev(q, "q"), _dev(k_cache, "k_cache", q.dtype),
        _dev(v_cache, "v_cache", q.dtype), _dev(seq_lens, "seq_lens", torch.int32),
        _dev(block_table, "block_table", torch.int32), _dev(out, "out", q.dtype),
        B, H_q, H_kv, d, float(scale), int(window), _stream_ptr(stream),
        block_table.shape[1], nblk, dt)
    _check(rc, "attn_decode_gqa_noalloc")
    return out


def decode_mla(q_latent, q_rope, latent_cache, seq_lens, block_table, scale,
               out=None, stream=None):
    """z [B][H][d_c] = absorbed MLA decode over the paged latent cache (bf16).

    q_latent [B][H][d_c]; q_rope [B][H][d_r];
    latent_cache [num_blocks][64][d_c + d_r].
    """
    B, H, d_c = q_latent.shape
    d_r = q_rope.shape[2]
    nblk, bs, width = latent_cache.shape
    if bs != BLOCK_SIZE or width != d_c + d_r:
        raise ValueError("latent_cache must be [num_blocks][64][d_c + d_r]")
    if out is None:
        out = torch.empty_like(q_latent)
    bf = torch.bfloat16
    rc = load().attn_decode_mla(
        _dev(q_latent, "q_latent", bf), _dev(q_rope, "q_rope", bf),
        _dev(latent_cache, "latent_cache", bf),
        _dev(seq_lens, "seq_lens", torch.int32),
        _dev(block_table, "block_table", torch.int32), _dev(out, "out", bf),
        B, H, d_c, d_r, float(scale), _stream_ptr(stream), block_table.shape[1],
        nblk)
    _check(rc, "attn_decode_mla")
    return out


def decode_mla_fp8(q_latent, q_rope, latent_codes, latent_scale, seq_lens, block_table,
                   scale, out=None, stream=None):
    """z [B][H][d_c] (bf16) = absorbed MLA decode over an fp8 latent cache:
    latent_codes uint8 E4M3 [num_blocks][64][d_c + d_r], latent_scale fp32
    [num_blocks][64] (value = code value * row scale)."""
    B, H, d_c = q_latent.shape
    d_r = q_rope.shape[2]
    nblk, bs, width = latent_codes.shape
    if bs != BLOCK_SIZE or width != d_c + d_r:
        raise ValueError("latent_codes must be [num_blocks][64][d_c + d_r]")
    if tuple(latent_scale.shape) != (nblk, bs):
        raise ValueError("latent_scale must be [num_blocks][64]")
    if out is None:
        out = torch.empty_like(q_latent)
    bf = torch.bfloat16
    rc = load().attn_decode_mla_fp8(
        _dev(q_latent, "q_latent", bf), _dev(q_rope, "q_rope", bf),
        _dev(latent_codes, "latent_codes", torch.uint8),
        _dev(latent_scale, "latent_scale", torch.float32),
        _dev(seq_lens, "seq_lens", torch.int32),
        _dev(block_table, "block_table", torch.int32), _dev(out, "out", bf),
        B, H, d_c, d_r, float(scale), _stream_ptr(stream), block_table.shape[1], nblk)
    _check(rc, "attn_decode_mla_fp8")
    return out


def kv_append_mla_fp8(latent_new, latent_codes, latent_scale, positions, block_table,
                      d_c=512, stream=None):
    """Quantise latent_new [B][d_c + d_r] (bf16) to E4M3 with one scale per row
    and write it into the fp8 latent cache at positions[b]."""
    B, width = latent_new.shape
    rc = load().kv_append_mla_fp8(
        _dev(latent_new, "latent_new", torch.bfloat16),
        _dev(latent_codes, "latent_codes", torch.uint8),
        _dev(latent_scale, "latent_scale", torch.float32),
        _dev(positions, "positions", torch.int32),
        _dev(block_table, "block_table", torch.int32), B, d_c, width - d_c,
        block_table.shape[1], latent_codes.shape[0], _stream_ptr(stream))
    _check(rc, "kv_append_mla_fp8")


def mla_absorb_q(q_c, u_k, out=None, stream=None):
    """q_latent [B][H][d_c] = q_c (U^K_h)^T per head (bf16).

    q_c [B][H][d_h]; u_k [H][d_c][d_h]."""
    B, H, d_h = q_c.shape
    d_c = u_k.shape[1]
    if tuple(u_k.shape) != (H, d_c, d_h):
        raise ValueError("u_k must be [H][d_c][d_h]")
    bf = torch.bfloat16
    if out is None:
        out = torch.empty((B, H, d_c), dtype=bf, device=q_c.device)
    _check(load().attn_mla_absorb_q(_dev(q_c, "q_c", bf), _dev(u_k, "u_k", bf),
                                    _dev(out, "out", bf), B, H, d_c, d_h,
                                    _stream_ptr(stream)), "attn_mla_absorb_q")
    return out


def mla_project_out(z, u_v, out=None, stream=None):
    """o [B][H][d_v] = z U^V_h per head (bf16).  z [B][H][d_c]; u_v [H][d_c][d_v]."""
    B, H, d_c = z.shape
    d_v = u_v.shape[2]
    if tuple(u_v.shape) != (H, d_c, d_v):
        raise ValueError("u_v must be [H][d_c][d_v]")
    bf = torch.bfloat16
    if out is None:
        out = torch.empty((B, H, d_v), dtype=bf, device=z.device)
    _check(load().attn_mla_project_out(_dev(z, "z", bf), _dev(u_v, "u_v", bf),
                                       _dev(out, "out", bf), B, H, d_c, d_v,
                                       _stream_ptr(stream)), "attn_mla_project_out")
    return out


def kv_append_ext(k_new, v_new, k_cache, v_cache, positions, block_table,
                  window=0, sink_tokens=0, ring_blocks=0, stream=None, global_pos=None):
    """kv_append through the table mapping of a visibility record (sink or
    global slots, then the ring): with a ring, writing past the window
    overwrites the block that left it."""
    B, H_kv, d = k_new.shape
    vis = _visibility(window, sink_tokens, ring_blocks, global_pos, B)
    rc = load().kv_append_ext(
        _dev(k_new, "k_new"), _dev(v_new, "v_new", k_new.dtype),
        _dev(k_cache, "k_cache", k_new.dtype), _dev(v_cache, "v_cache", k_new.dtype),
        _dev(positions, "positions", torch.int32),
        _dev(block_table, "block_table", torch.int32), B, H_kv, d,
        block_table.shape[1], k_cache.shape[0], _dtype_code(k_new.dtype),
        ctypes.byref(vis), _stream_ptr(stream))
    _check(rc, "kv_append_ext")


def kv_append(k_new, v_new, k_cache, v_cache, positions, block_table,
              stream=None):
    """Write k_new/v_new [B][H_kv][d] into the paged caches at positions[b]."""
    B, H_kv, d = k_new.shape
    rc = load().kv_append(
        _dev(k_new, "k_new"), _dev(v_new, "v_new", k_new.dtype),
        _dev(k_cache, "k_cache", k_new.dtype),
        _dev(v_cache, "v_cache", k_new.dtype),
        _dev(positions, "positions", torch.int32),
        _dev(block_table, "block_table", torch.int32), B, H_kv, d,
        block_table.shape[1], k_cache.shape[0], _dtype_code(k_new.dtype),
        _stream_ptr(stream))
    _check(rc, "kv_append")


def kv_append_mla(latent_new, latent_cache, positions, block_table, d_c=512,
                  stream=None):
    """Write latent_new [B][d_c + d_r] into latent_cache at positions[b]."""
    B, width = latent_new.shape
    bf = torch.bfloat16
    rc = load().kv_append_mla(
        _dev(latent_new, "latent_new", bf), _dev(latent_cache, "latent_cache", bf),
        _dev(positions, "positions", torch.int32),
        _dev(block_table, "block_table", torch.int32), B, d_c, width - d_c,
        block_table.shape[1], latent_cache.shape[0], _stream_ptr(stream))
    _check(rc, "kv_append_mla")


def plan(seq_lens, units_per_seq, window, max_blocks, num_ctas, stream=None):
    """Run the device split planner alone; returns the int64 plan tensor."""
    B = seq_lens.shape[0]
    out = torch.empty(1 + 4 * num_ctas + B + 1, dtype=torch.int64,
                      device=seq_lens.device)
    rc = load().attn_decode_plan(
        _dev(seq_lens, "seq_lens", torch.int32), B, units_per_seq, int(window),
        max_blocks, num_ctas, _dev(out, "plan_out"), _stream_ptr(stream))
    _check(rc, "attn_decode_plan")
    return out


def gqa_config(B, H_q, H_kv, d, dtype=torch.bfloat16):
    """(num_ctas, heads_per_cta, path) the GQA call uses for this problem;
    path 0 = CUDA-core kernel, 1 = M=128 tensor-core kernel, 2 = M=64
    tensor-core kernel.  dtype "fp8" asks about decode_gqa_fp8."""
    n, h, pth = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    code = FP8_E4M3 if dtype == "fp8" else _dtype_code(dtype)
    rc = load().attn_decode_gqa_config(B, H_q, H_kv, d, code,
                                       ctypes.byref(n), ctypes.byref(h),
                                       ctypes.byref(pth))
    _check(rc, "attn_decode_gqa_config")
    return n.value, h.value, pth.value


def set_num_ctas(n):
    _check(load().attn_set_num_ctas(int(n)), "attn_set_num_ctas")


def set_gqa_path(path):
    """Testing/tuning hook: -1 automatic (bf16: CUDA cores for groups of up
    to 4 heads, else the tensor cores), 0 CUDA cores, 1 tensor cores (the
    M=128 kernel where it applies, else M=64), 2 the M=64 tensor-core kernel."""
    _check(load().attn_set_gqa_path(int(path)), "attn_set_gqa_path")


def debug_force_timeout(enable=True, timeout_ns=20_000_000):
    _check(load().attn_debug_force_timeout(int(enable), int(timeout_ns)),
           "attn_debug_force_timeout")


def last_error(stream=None):
    """Synchronise the stream, read and clear the device error word."""
    return load().attn_decode_last_error(_stream_ptr(stream))


class ProfileEvents:
    """Context manager: the library records CUDA events around its main
    split-KV kernel for the next n calls; ``times_ms()`` returns them."""

    def __init__(self, n):
        self.n = n
        self.start = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        self.stop = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in self.start + self.stop:
            e.record()          # materialise the underlying cudaEvent_t
        torch.cuda.synchronize()
        arr = ctypes.c_void_p * n
        self._s = arr(*[e.cuda_event for e in self.start])
        self._e = arr(*[e.cuda_event for e in self.stop])

    def __enter__(self):
        _check(load().attn_set_profile_events(self._s, self._e, self.n),
               "attn_set_profile_events")
        return self

    def __exit__(self, *exc):
        load().attn_set_profile_events(None, None, 0)
        return False

    def times_ms(self, count=None):
        torch.cuda.synchronize()
        k = self.n if count is None else count
        return [self.start[i].elapsed_time(self.stop[i]) for i in range(k)]
