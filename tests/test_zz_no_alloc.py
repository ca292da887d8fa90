"""attn_decode_gqa_noalloc: the decode entry point for callers that must not
allocate device memory while running (e.g. a server that gives all device
memory to its own pool at start-up).  Its scratch is a fixed array inside the
library; these tests call it through the C ABI and check it, on two
consecutive calls, against the regular attn_decode_gqa and against the fp64
oracle (both within the bf16 parity bars).  This file is collected last so
that a stop-at-first-failure run has already run everything else; it also
passes on its own in a fresh process."""
import ctypes

import pytest
import torch

from tests.parity import assert_parity, oracle_gqa_sequences
from workloads import GQAConfig, make_gqa_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call_noalloc(lib, x, out):
    """Direct C-ABI call of attn_decode_gqa_noalloc."""
    c = lib.load()
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return c.attn_decode_gqa_noalloc(
        ptr(x.q), ptr(x.k_cache), ptr(x.v_cache), ptr(x.seq_lens), ptr(x.block_table),
        ptr(out), x.q.shape[0], x.q.shape[1], x.k_cache.shape[1], x.q.shape[2],
        ctypes.c_float(x.scale), x.window,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
        x.block_table.shape[1], x.k_cache.shape[0], 1 if x.q.dtype == torch.bfloat16 else 0)


def test_noalloc_matches_regular_entry_point_on_two_calls(lib):
    first = make_gqa_inputs(GQAConfig("na1", B=6, H_q=32, H_kv=8, d=128,
                                      seq_lens=[4096, 1, 700, 64, 2000, 129],
                                      seed=71), device=DEV)
    second = make_gqa_inputs(GQAConfig("na2", B=3, H_q=24, H_kv=4, d=256,
                                       seq_lens=[5000, 333, 4097], window=1000,
                                       seed=72), device=DEV)
    for x in (first, second):            # two calls in a row, different shapes
        ref = lib.decode_gqa(x.q, x.k_cache, x.v_cache, x.seq_lens, x.block_table,
                             x.scale, window=x.window)
        out = torch.full_like(x.q, float("nan"))
        assert _call_noalloc(lib, x, out) == lib.OK
        assert lib.last_error() == lib.OK
        got = out.float().cpu().numpy()
        assert_parity(got, ref.float().cpu().numpy(), torch.bfloat16,
                      "noalloc vs attn_decode_gqa")
        for b, r in oracle_gqa_sequences(x, range(x.cfg.B)).items():
            assert_parity(got[b], r, torch.bfloat16, f"noalloc vs oracle b={b}")


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    x = make_gqa_inputs(GQAConfig("na3", B=1, H_q=8, H_kv=8, d=128, seq_lens=[64],
                                  seed=73), device=DEV)
    c = lib.load()
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    # B = 100000 sequences of 8 heads would need ~400 MB of scratch; the call
    # is refused before anything is launched or dereferenced.
    rc = c.attn_decode_gqa_noalloc(
        ptr(x.q), ptr(x.k_cache), ptr(x.v_cache), ptr(x.seq_lens), ptr(x.block_table),
        ptr(x.q), 100000, 8, 8, 128, ctypes.c_float(0.1), 0,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), 1, 1, 1)
    assert rc == lib.ERR_UNSUPPORTED
    assert c.attn_decode_gqa_noalloc(None, ptr(x.k_cache), ptr(x.v_cache),
                                     ptr(x.seq_lens), ptr(x.block_table), ptr(x.q),
                                     1, 8, 8, 128, ctypes.c_float(0.1), 0, None, 1, 1,
                                     1) == lib.ERR_ARG
