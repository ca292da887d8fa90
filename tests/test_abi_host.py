"""CPU-only checks of the boundary: the library loads, exports every symbol the
header declares, validates arguments on the host; the host planner model is
self-consistent.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import decode_attention_kv_paged_b200 as attn
from decode_attention_kv_paged_b200 import planner

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "attn_decode.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"^(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", src, flags=re.M))


def test_library_exports_every_declared_symbol():
    lib = attn.load()
    declared = _declared_symbols()
    assert declared == set(attn.C_SYMBOLS), declared ^ set(attn.C_SYMBOLS)
    for name in declared:
        assert hasattr(lib, name), name
    assert lib.attn_version() >= 100
    assert lib.attn_status_string(-5) == b"ATTN_ERR_BAD_BLOCK"


def test_null_and_shape_arguments_rejected_before_any_launch():
    lib = attn.load()
    p = ctypes.c_void_p(16)      # never dereferenced: validation fails first
    n = ctypes.c_void_p(0)
    assert lib.attn_decode_gqa(n, p, p, p, p, p, 1, 4, 2, 128, 1.0, 0, n, 1, 1,
                               1) == attn.ERR_ARG
    assert lib.attn_decode_gqa(p, p, p, p, p, p, 1, 6, 4, 128, 1.0, 0, n, 1, 1,
                               1) == attn.ERR_ARG           # 6 % 4
    assert lib.attn_decode_gqa(p, p, p, p, p, p, 0, 4, 2, 128, 1.0, 0, n, 1, 1,
                               1) == attn.ERR_ARG           # B = 0
    assert lib.attn_decode_gqa(ctypes.c_void_p(8), p, p, p, p, p, 1, 4, 2, 128,
                               1.0, 0, n, 1, 1, 1) == attn.ERR_ARG  # misaligned
    assert lib.attn_decode_gqa(p, p, p, p, p, p, 1, 4, 2, 128, float("nan"), 0,
                               n, 1, 1, 1) == attn.ERR_ARG
    assert lib.attn_decode_gqa(p, p, p, p, p, p, 1, 4, 2, 128, 1.0, 0, n, 1, 1,
                               7) == attn.ERR_ARG           # dtype
    assert lib.attn_decode_mla(n, p, p, p, p, p, 1, 128, 512, 64, 1.0, n, 1,
                               1) == attn.ERR_ARG
    assert lib.kv_append(n, p, p, p, p, p, 1, 1, 128, 1, 1, 1, n) == attn.ERR_ARG
    assert lib.kv_append_mla(n, p, p, p, 1, 512, 64, 1, 1, n) == attn.ERR_ARG
    assert lib.attn_decode_plan(n, 1, 1, 0, 1, 1, p, n) == attn.ERR_ARG
    assert lib.attn_set_num_ctas(-1) == attn.ERR_ARG
    assert lib.attn_set_gqa_path(5) == attn.ERR_ARG


def test_unsupported_head_dim_reported():
    lib = attn.load()
    p = ctypes.c_void_p(16)
    n = ctypes.c_void_p(0)
    assert lib.attn_decode_gqa(p, p, p, p, p, p, 1, 4, 2, 96, 1.0, 0, n, 1, 1,
                               1) == attn.ERR_UNSUPPORTED
    assert lib.attn_decode_gqa(p, p, p, p, p, p, 1, 4, 2, 256, 1.0, 0, n, 1, 1,
                               0) == attn.ERR_UNSUPPORTED  # fp32 d=256
    assert lib.attn_decode_mla(p, p, p, p, p, p, 1, 128, 256, 64, 1.0, n, 1,
                               1) == attn.ERR_UNSUPPORTED


@pytest.mark.parametrize("lens,units,window,P", [
    ([4096] * 16, 8, 0, 148), ([0, 1, 64, 65, 4097, 0], 3, 0, 7),
    ([131072, 1024, 5000], 4, 4096, 148), ([5] * 300, 2, 0, 64),
    ([100, 0, 0], 1, 0, 1000), ([0, 0], 2, 0, 5)])
def test_host_planner_partition_properties(lens, units, window, P):
    """CTA ranges tile [0, W) exactly; each (unit, CTA) slot u + i is unique
    and below U + P; windowed sequences list only blocks with visible keys."""
    mb = max(1, max((t + 63) // 64 for t in lens))
    p = planner.plan(lens, units, window, mb, P)
    W = p[0]
    rows = [p[1 + 4 * i: 5 + 4 * i] for i in range(P)]
    assert rows[0][0] == 0 and rows[-1][1] == W
    for a, b in zip(rows, rows[1:]):
        assert a[1] == b[0]
    prefix = p[1 + 4 * P:]
    slots = set()
    U = len(lens) * units
    for b, T in enumerate(lens):
        first, nb = planner.visible_blocks(T, window, mb)
        if window > 0 and nb:
            lo = max(0, T - window)
            assert first == lo // 64 and first * 64 + nb * 64 >= T
        for u in range(units):
            for c in planner.splits_of_unit(lens, units, window, mb, P, b, u):
                s = b * units + u + c
                assert s not in slots and s < U + P
                slots.add(s)
