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


def test_visibility_struct_layout_matches_header(tmp_path):
    """The Python binding's attn_visibility has the header's layout (field
    offsets and size, as a C compiler lays it out)."""
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "attn_decode.h"\n'
                   'int main(void) { printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(attn_visibility),'
                   ' offsetof(attn_visibility, window), offsetof(attn_visibility, sink_tokens),'
                   ' offsetof(attn_visibility, ring_blocks), offsetof(attn_visibility, global_pos),'
                   ' offsetof(attn_visibility, n_global)); return 0; }\n')
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    V = attn.Visibility
    want = [ctypes.sizeof(V), V.window.offset, V.sink_tokens.offset, V.ring_blocks.offset,
            V.global_pos.offset, V.n_global.offset]
    assert got == want


def test_global_set_validated_on_the_host():
    """An explicit global set with sink tokens, with a ring that does not fit
    the table row after its global slots, a null set, or more than 64
    positions is refused before any launch."""
    lib = attn.load()
    p = ctypes.c_void_p(16)      # never dereferenced: validation fails first
    g = ctypes.c_void_p(64)

    def call(vis):
        return lib.attn_decode_gqa_ext(p, p, p, p, p, p, 1, 8, 2, 64, ctypes.c_float(0.1),
                                       ctypes.byref(vis), None, 4, 8, attn.BF16)
    V = attn.Visibility
    assert call(V(10, 4, 0, g.value, 2)) == attn.ERR_ARG        # with sink tokens
    assert call(V(64, 0, 3, g.value, 2)) == attn.ERR_ARG        # 2 global + 3 ring slots > 4
    assert call(V(64, 4, 2, g.value, 2)) == attn.ERR_ARG        # sink tokens and a ring
    assert call(V(200, 0, 2, g.value, 2)) == attn.ERR_ARG       # ring shorter than the window
    assert call(V(10, 0, 0, None, 2)) == attn.ERR_ARG           # no positions
    assert call(V(10, 0, 0, g.value, -1)) == attn.ERR_ARG       # negative count
    assert call(V(10, 0, 0, ctypes.c_void_p(66).value, 2)) == attn.ERR_ARG   # misaligned
    assert call(V(10, 0, 0, g.value, 65)) == attn.ERR_UNSUPPORTED
