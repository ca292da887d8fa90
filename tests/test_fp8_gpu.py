"""GPU parity of the fp8 (OCP E4M3 + per-row fp32 scale) KV cache, through
the C ABI, vs the oracle: the append's quantisation is bit-exact (codes and
scales are integer/byte results of fp32 arithmetic both sides do alike), and
the decode matches the oracle's decode over the dequantised cache within the
bf16 bars (max-abs <= 1e-2, rel-L2 <= 2e-3), on both kernels that read an
fp8 cache: the CUDA-core split kernel (path 0) and the M = 128 tensor-core
kernel that widens the codes to f16 on the chip (path 1, d <= 128)."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.parity import assert_parity
from workloads import BLOCK_SIZE

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fp8_cache(seed, n_blocks, H_kv, d):
    """Random bf16 K/V rows, row magnitudes varied over [0.05, 0.5] x N(0,1)
    (so a one-token output stays where bf16 rounding fits the 1e-2 max-abs
    bar), quantised on the host by the oracle."""
    g = torch.Generator().manual_seed(seed)
    shape = (n_blocks, H_kv, BLOCK_SIZE, d)
    mags = torch.rand((n_blocks, H_kv, BLOCK_SIZE, 1), generator=g) * 0.45 + 0.05
    k = (torch.randn(shape, generator=g) * mags).bfloat16()
    v = (torch.randn(shape, generator=g) * mags).bfloat16()
    kc, ks = orc.quantize_rows_e4m3(k.float().numpy())
    vc, vs = orc.quantize_rows_e4m3(v.float().numpy())
    return kc, ks, vc, vs


def test_append_quantisation_is_bit_exact(lib):
    B, H_kv, d = 3, 4, 128
    g = torch.Generator().manual_seed(81)
    rows_k = (torch.randn((B, H_kv, d), generator=g) *
              torch.tensor([0.01, 1.0, 300.0]).view(3, 1, 1)).bfloat16()
    rows_v = (torch.randn((B, H_kv, d), generator=g) * 2).bfloat16()
    rows_k[1, 2] = 0                                     # a zero row
    table = torch.tensor([[2, 5], [0, 1], [4, 3]], dtype=torch.int32)
    pos = torch.tensor([70, 3, 127], dtype=torch.int32)
    kc = torch.zeros((6, H_kv, BLOCK_SIZE, d), dtype=torch.uint8, device=DEV)
    vc = torch.zeros_like(kc)
    ks = torch.zeros((6, H_kv, BLOCK_SIZE), dtype=torch.float32, device=DEV)
    vs = torch.zeros_like(ks)
    lib.kv_append_fp8(rows_k.to(DEV), rows_v.to(DEV), kc, vc, ks, vs, pos.to(DEV),
                      table.to(DEV))
    assert lib.last_error() == lib.OK
    ek, eks = orc.quantize_rows_e4m3(rows_k.float().numpy())
    ev, evs = orc.quantize_rows_e4m3(rows_v.float().numpy())
    kc, vc, ks, vs = kc.cpu().numpy(), vc.cpu().numpy(), ks.cpu().numpy(), vs.cpu().numpy()
    for b in range(B):
        phys = int(table[b, int(pos[b]) // 64])
        r = int(pos[b]) % 64
        assert np.array_equal(kc[phys, :, r], ek[b]), b
        assert np.array_equal(vc[phys, :, r], ev[b]), b
        assert np.array_equal(ks[phys, :, r].view(np.uint32), eks[b].view(np.uint32)), b
        assert np.array_equal(vs[phys, :, r].view(np.uint32), evs[b].view(np.uint32)), b


FP8_CASES = [
    # (H_q, H_kv, d, lens, window, sink)
    (32, 8, 128, [1000, 65, 1], 0, 0),
    (8, 8, 64, [700, 300], 0, 0),
    (24, 4, 256, [3000, 129], 0, 0),
    (32, 1, 128, [600, 64], 0, 0),
    (32, 8, 128, [2000, 90], 300, 16),
]


class _path:
    """Force a GQA kernel for the calls inside the block."""

    def __init__(self, lib, path):
        self.lib, self.path = lib, path

    def __enter__(self):
        self.lib.set_gqa_path(self.path)

    def __exit__(self, *exc):
        self.lib.set_gqa_path(-1)


PATHS = pytest.mark.parametrize("path", [0, 1], ids=["cuda_core", "tcgen05"])


@PATHS
@pytest.mark.parametrize("H_q,H_kv,d,lens,window,sink", FP8_CASES,
                         ids=[f"q{c[0]}_kv{c[1]}_d{c[2]}_w{c[4]}_g{c[5]}" for c in FP8_CASES])
def test_fp8_decode_matches_oracle(lib, path, H_q, H_kv, d, lens, window, sink):
    if path == 1 and d > 128:
        pytest.skip("the tensor-core fp8 kernel takes d <= 128")
    B = len(lens)
    slots = max((T + 63) // 64 for T in lens)
    n_blocks = B * slots + 2
    kc, ks, vc, vs = _fp8_cache(8100 + H_q + d, n_blocks, H_kv, d)
    g = torch.Generator().manual_seed(8200 + d)
    q = torch.randn((B, H_q, d), generator=g).bfloat16()
    table = torch.randperm(n_blocks, generator=g)[: B * slots].reshape(B, slots).to(torch.int32)
    scale = 1.0 / np.sqrt(d)
    with _path(lib, path):
        got = lib.decode_gqa_fp8(q.to(DEV), torch.from_numpy(kc).to(DEV),
                                 torch.from_numpy(vc).to(DEV), torch.from_numpy(ks).to(DEV),
                                 torch.from_numpy(vs).to(DEV),
                                 torch.tensor(lens, dtype=torch.int32, device=DEV), table.to(DEV),
                                 scale, window=window, sink_tokens=sink)
        assert lib.last_error() == lib.OK
    ref = orc.decode_gqa_vis(q.double().numpy(), orc.dequantize_e4m3(kc, ks),
                             orc.dequantize_e4m3(vc, vs), np.asarray(lens, dtype=np.int32),
                             table.numpy(), scale, window=window, sink=sink)
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, "fp8 decode")


def test_fp8_append_then_decode(lib):
    """The current token appended with kv_append_fp8 is read by the decode
    exactly as the oracle quantises it."""
    B, H_q, H_kv, d, T = 2, 16, 4, 128, 333
    nb = (T + 63) // 64
    kc, ks, vc, vs = _fp8_cache(8300, B * nb, H_kv, d)
    table = torch.arange(B * nb, dtype=torch.int32).reshape(B, nb)
    g = torch.Generator().manual_seed(8301)
    q = torch.randn((B, H_q, d), generator=g).bfloat16()
    k_new = torch.randn((B, H_kv, d), generator=g).bfloat16() * 2
    v_new = torch.randn((B, H_kv, d), generator=g).bfloat16() * 0.5
    dk, dv = torch.from_numpy(kc).to(DEV), torch.from_numpy(vc).to(DEV)
    dks, dvs = torch.from_numpy(ks).to(DEV), torch.from_numpy(vs).to(DEV)
    pos = torch.full((B,), T - 1, dtype=torch.int32, device=DEV)
    lib.kv_append_fp8(k_new.to(DEV), v_new.to(DEV), dk, dv, dks, dvs, pos, table.to(DEV))
    lens = torch.full((B,), T, dtype=torch.int32, device=DEV)
    got = lib.decode_gqa_fp8(q.to(DEV), dk, dv, dks, dvs, lens, table.to(DEV), 0.1)
    assert lib.last_error() == lib.OK
    ek, eks = orc.quantize_rows_e4m3(k_new.float().numpy())
    ev, evs = orc.quantize_rows_e4m3(v_new.float().numpy())
    for b in range(B):
        phys, r = int(table[b, (T - 1) // 64]), (T - 1) % 64
        kc[phys, :, r], ks[phys, :, r] = ek[b], eks[b]
        vc[phys, :, r], vs[phys, :, r] = ev[b], evs[b]
    ref = orc.decode_gqa(q.double().numpy(), orc.dequantize_e4m3(kc, ks),
                         orc.dequantize_e4m3(vc, vs), np.full(B, T, dtype=np.int32),
                         table.numpy(), 0.1)
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, "fp8 append+decode")


@PATHS
def test_fp8_decode_with_global_positions(lib, path):
    """The fp8 cache under a window plus an explicit global set."""
    lens, window = [2000, 700], 300
    rows = [[0, 5, 640, 1650], [699, -1, -1, -1]]
    H_q, H_kv, d = 32, 8, 128
    B = len(lens)
    slots = max((T + 63) // 64 for T in lens)
    n_blocks = B * slots + 2
    kc, ks, vc, vs = _fp8_cache(8400, n_blocks, H_kv, d)
    g = torch.Generator().manual_seed(8401)
    q = torch.randn((B, H_q, d), generator=g).bfloat16()
    table = torch.randperm(n_blocks, generator=g)[: B * slots].reshape(B, slots).to(torch.int32)
    gp = torch.tensor(rows, dtype=torch.int32)
    with _path(lib, path):
        got = lib.decode_gqa_fp8(q.to(DEV), torch.from_numpy(kc).to(DEV),
                                 torch.from_numpy(vc).to(DEV), torch.from_numpy(ks).to(DEV),
                                 torch.from_numpy(vs).to(DEV),
                                 torch.tensor(lens, dtype=torch.int32, device=DEV), table.to(DEV),
                                 0.09, window=window, global_pos=gp.to(DEV))
        assert lib.last_error() == lib.OK
    ref = orc.decode_gqa_vis(q.double().numpy(), orc.dequantize_e4m3(kc, ks),
                             orc.dequantize_e4m3(vc, vs), np.asarray(lens, dtype=np.int32),
                             table.numpy(), 0.09, window=window, global_pos=gp.numpy())
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, "fp8 global set")


def _fp8_unit_cache(seed, n_blocks, H_kv, d):
    """Unit-variance bf16 K/V rows (no magnitude narrowing), quantised by the
    oracle."""
    g = torch.Generator().manual_seed(seed)
    shape = (n_blocks, H_kv, BLOCK_SIZE, d)
    k = torch.randn(shape, generator=g).bfloat16()
    v = torch.randn(shape, generator=g).bfloat16()
    kc, ks = orc.quantize_rows_e4m3(k.float().numpy())
    vc, vs = orc.quantize_rows_e4m3(v.float().numpy())
    return kc, ks, vc, vs


def _within_one_bf16_ulp(got, ref, slack):
    """|got - ref| within one bf16 ulp of ref (the output's own rounding)
    plus an absolute slack for the fp32 arithmetic before it."""
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    return np.abs(np.asarray(got, dtype=np.float64) - ref) <= ulp + slack


@PATHS
@pytest.mark.parametrize("H_q,H_kv,d,lens", [(32, 8, 128, [1, 2, 700, 4097]),
                                             (32, 1, 128, [3000, 64]),
                                             (16, 16, 64, [1500, 3])],
                         ids=["gqa8_d128", "mqa_d128", "mha_d64"])
def test_fp8_unit_variance_rows(lib, path, H_q, H_kv, d, lens):
    """Unit-variance K/V rows and queries, no narrowing of the input ranges
    (one-token outputs reach |o| of 3-4, where a bf16 ulp is 2^-6): judged by
    rel-L2 and by agreement with the exact result to one bf16 ulp plus 2e-3."""
    B = len(lens)
    slots = max((T + 63) // 64 for T in lens)
    n_blocks = B * slots + 2
    kc, ks, vc, vs = _fp8_unit_cache(8500 + H_q + d, n_blocks, H_kv, d)
    g = torch.Generator().manual_seed(8501 + d)
    q = torch.randn((B, H_q, d), generator=g).bfloat16()
    table = torch.randperm(n_blocks, generator=g)[: B * slots].reshape(B, slots).to(torch.int32)
    scale = 1.0 / np.sqrt(d)
    with _path(lib, path):
        got = lib.decode_gqa_fp8(q.to(DEV), torch.from_numpy(kc).to(DEV),
                                 torch.from_numpy(vc).to(DEV), torch.from_numpy(ks).to(DEV),
                                 torch.from_numpy(vs).to(DEV),
                                 torch.tensor(lens, dtype=torch.int32, device=DEV), table.to(DEV),
                                 scale)
        assert lib.last_error() == lib.OK
    ref = orc.decode_gqa(q.double().numpy(), orc.dequantize_e4m3(kc, ks),
                         orc.dequantize_e4m3(vc, vs), np.asarray(lens, dtype=np.int32),
                         table.numpy(), scale)
    got = got.float().cpu().numpy()
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel <= 2e-3, rel
    ok = _within_one_bf16_ulp(got, ref, 2e-3)
    assert ok.all(), f"{(~ok).sum()} outputs off by more than one bf16 ulp + 2e-3"


@pytest.mark.parametrize("H_q,H_kv,d", [(32, 1, 128), (64, 1, 128), (8, 2, 64), (4, 4, 128),
                                        (24, 4, 64)],
                         ids=["mqa32", "mqa64", "g4_d64", "mha", "g6_d64"])
def test_fp8_tensor_core_many_tiles_and_splits(lib, H_q, H_kv, d):
    """The tensor-core fp8 kernel over long, ragged sequences whose tiles wrap
    the stage ring many times, with 3 and 148 CTAs (segments crossing units
    and sequences), groups from 1 to 64 heads (64: two 32-head units)."""
    lens = [5000, 777, 64, 65, 2100]
    B = len(lens)
    slots = max((T + 63) // 64 for T in lens)
    n_blocks = B * slots + 2
    kc, ks, vc, vs = _fp8_cache(8600 + H_q + d, n_blocks, H_kv, d)
    g = torch.Generator().manual_seed(8601 + H_q)
    q = torch.randn((B, H_q, d), generator=g).bfloat16()
    table = torch.randperm(n_blocks, generator=g)[: B * slots].reshape(B, slots).to(torch.int32)
    ref = orc.decode_gqa(q.double().numpy(), orc.dequantize_e4m3(kc, ks),
                         orc.dequantize_e4m3(vc, vs), np.asarray(lens, dtype=np.int32),
                         table.numpy(), 0.08)
    args = (q.to(DEV), torch.from_numpy(kc).to(DEV), torch.from_numpy(vc).to(DEV),
            torch.from_numpy(ks).to(DEV), torch.from_numpy(vs).to(DEV),
            torch.tensor(lens, dtype=torch.int32, device=DEV), table.to(DEV), 0.08)
    for ctas in (3, 0):
        lib.set_num_ctas(ctas)
        try:
            with _path(lib, 1):
                got = lib.decode_gqa_fp8(*args)
                assert lib.last_error() == lib.OK
        finally:
            lib.set_num_ctas(0)
        assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, f"fp8 tc, {ctas} CTAs")


def test_fp8_tensor_core_bad_block_is_flagged(lib):
    """A block id outside the pool on the tensor-core fp8 kernel sets the
    bad-block error and is never dereferenced."""
    H_q, H_kv, d, lens = 32, 1, 128, [300, 200]
    n_blocks = 12
    kc, ks, vc, vs = _fp8_cache(8700, n_blocks, H_kv, d)
    q = torch.randn((2, H_q, d)).bfloat16()
    table = torch.arange(10, dtype=torch.int32).reshape(2, 5)
    table[1, 2] = 1 << 20                                 # outside the pool
    with _path(lib, 1):
        lib.decode_gqa_fp8(q.to(DEV), torch.from_numpy(kc).to(DEV), torch.from_numpy(vc).to(DEV),
                           torch.from_numpy(ks).to(DEV), torch.from_numpy(vs).to(DEV),
                           torch.tensor(lens, dtype=torch.int32, device=DEV), table.to(DEV), 0.1)
        assert lib.last_error() == lib.ERR_BAD_BLOCK
