"""GPU parity of the GQA/MQA/MHA decode path (through the C ABI) vs the oracle.

Inputs are the seeded workloads of ``workloads``; the oracle receives the same
(dtype-rounded) values.  Bars: bf16 max-abs <= 1e-2 and rel-L2 <= 2e-3,
fp32 max-abs <= 1e-5; planner and cache placement bit-exact.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from tests.parity import assert_parity, oracle_gqa_sequences
from workloads import (BLOCK_SIZE, GQAConfig, LLAMA3_8B, RAGGED_FULL,
                       RAGGED_WINDOW, SWEEP, TINY, make_gqa_inputs)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_gpu(attn, inp):
    d = inp.to(DEV) if inp.q.device.type != "cuda" else inp
    out = attn.decode_gqa(d.q, d.k_cache, d.v_cache, d.seq_lens, d.block_table,
                          d.scale, window=d.window)
    assert attn.last_error() == attn.OK
    return out


def full_oracle(inp):
    return orc.decode_gqa(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(),
                          inp.seq_lens.cpu(), inp.block_table.cpu(), inp.scale,
                          window=inp.window)


# ------------------------------------------------------------ tiny, fp32
def test_tiny_fp32_contiguous(lib):
    """B=1, H_q=4, H_kv=2, d=16, T=64, fp32, identity table, scale 1/4."""
    inp = make_gqa_inputs(TINY)
    got = run_gpu(lib, inp).cpu().numpy()
    assert_parity(got, full_oracle(inp), torch.float32, "tiny fp32")


# --------------------------------------------- small cases spanning tiles
SMALL = [
    # (B, H_q, H_kv, d, dtype, lens, window)
    (3, 8, 2, 128, torch.bfloat16, [1, 64, 65], 0),
    (4, 32, 8, 128, torch.bfloat16, [300, 129, 64, 1000], 0),
    (2, 32, 32, 128, torch.bfloat16, [513, 77], 0),          # MHA
    (2, 32, 1, 128, torch.bfloat16, [700, 131], 0),          # MQA (G=32)
    (2, 24, 4, 256, torch.bfloat16, [999, 4097], 0),         # groups of 6
    (2, 24, 4, 256, torch.bfloat16, [999, 4097], 300),       # + window
    (3, 12, 4, 64, torch.bfloat16, [5, 190, 257], 64),       # G=3, window = 1 block
    (2, 16, 2, 32, torch.bfloat16, [33, 200], 1),            # window of 1
    (2, 10, 2, 16, torch.bfloat16, [64, 129], 0),            # G=5 -> 1 head/CTA
    (2, 16, 2, 128, torch.float32, [100, 300], 0),           # fp32 G=8
    (2, 4, 4, 64, torch.float32, [77, 1], 50),               # fp32 MHA window
    (5, 8, 1, 128, torch.bfloat16, [0, 100, 0, 64, 1], 0),   # empty sequences
]


@pytest.mark.parametrize("B,H_q,H_kv,d,dtype,lens,window", SMALL,
                         ids=[f"B{c[0]}_q{c[1]}_kv{c[2]}_d{c[3]}_"
                              f"{'bf16' if c[4] == torch.bfloat16 else 'f32'}_w{c[6]}"
                              for c in SMALL])
def test_small_cases_match_oracle(lib, B, H_q, H_kv, d, dtype, lens, window):
    cfg = GQAConfig("small", B=B, H_q=H_q, H_kv=H_kv, d=d, seq_lens=lens,
                    dtype=dtype, window=window, seed=1234 + B * 7 + d)
    inp = make_gqa_inputs(cfg)
    got = run_gpu(lib, inp).float().cpu().numpy()
    ref = full_oracle(inp)
    assert_parity(got, ref, dtype, "small")
    for b, T in enumerate(lens):
        if T == 0:
            assert np.all(got[b] == 0)


@pytest.mark.parametrize("num_ctas", [1, 3, 148, 1000])
def test_split_count_invariance(lib, num_ctas):
    """Any number of split CTAs gives the oracle's result (split-KV + LSE
    combine); 1000 CTAs splits single blocks of a unit across CTAs."""
    cfg = GQAConfig("split", B=3, H_q=16, H_kv=4, d=128, seq_lens=[2000, 1, 640],
                    seed=99)
    inp = make_gqa_inputs(cfg)
    ref = full_oracle(inp)
    lib.set_num_ctas(num_ctas)
    try:
        got = run_gpu(lib, inp).float().cpu().numpy()
    finally:
        lib.set_num_ctas(0)
    assert_parity(got, ref, torch.bfloat16, f"{num_ctas} CTAs")


def test_deterministic_repeat(lib):
    inp = make_gqa_inputs(GQAConfig("det", B=4, H_q=32, H_kv=8, d=128,
                                    seq_lens=[4096, 33, 2048, 1000], seed=5)).to(DEV)
    a = run_gpu(lib, inp).clone()
    b = run_gpu(lib, inp)
    assert torch.equal(a, b)


def test_permuted_table_matches_identity_table(lib):
    """Paging only relocates blocks: a permuted table gives the same result as
    the contiguous layout of the same logical cache (bit-identical)."""
    cfg = GQAConfig("perm", B=2, H_q=8, H_kv=2, d=128, seq_lens=[1000, 700],
                    seed=17, contiguous=True)
    inp = make_gqa_inputs(cfg).to(DEV)
    a = run_gpu(lib, inp)
    nb = inp.num_blocks
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(3)).to(DEV)
    k2 = torch.empty_like(inp.k_cache)
    v2 = torch.empty_like(inp.v_cache)
    k2[perm] = inp.k_cache
    v2[perm] = inp.v_cache
    table2 = torch.where(inp.block_table >= 0, perm[inp.block_table.long().clamp(min=0)],
                         inp.block_table.long()).to(torch.int32)
    b = lib.decode_gqa(inp.q, k2, v2, inp.seq_lens, table2, inp.scale)
    assert torch.equal(a, b)


def test_window_never_reads_masked_blocks(lib):
    """Blocks wholly before the window get invalid ids; the kernel must skip
    them (a read would raise ATTN_ERR_BAD_BLOCK) and still match the oracle
    (attention-head article §3: masked tiles are skipped, not computed)."""
    w = 300
    cfg = GQAConfig("win", B=3, H_q=24, H_kv=4, d=256, seq_lens=[5000, 301, 2049],
                    window=w, seed=41)
    inp = make_gqa_inputs(cfg)
    ref = full_oracle(inp)
    table = inp.block_table.clone()
    for b, T in enumerate(inp.seq_list):
        lo = max(0, T - w)
        table[b, : lo // BLOCK_SIZE] = -1
    inp.block_table = table
    got = run_gpu(lib, inp).float().cpu().numpy()
    assert_parity(got, ref, torch.bfloat16, "window")


def test_window_at_least_T_equals_full(lib):
    cfg = GQAConfig("wfull", B=2, H_q=8, H_kv=2, d=64, seq_lens=[500, 64], seed=8)
    inp = make_gqa_inputs(cfg).to(DEV)
    full = run_gpu(lib, inp).clone()
    inp.window = 500
    assert torch.equal(run_gpu(lib, inp), full)


# --------------------------------------------------------------- planner
@pytest.mark.parametrize("lens,units,window,P", [
    ([4096] * 16, 8, 0, 148),
    ([0, 1, 64, 65, 4097, 0], 3, 0, 7),
    ([131072, 1024, 5000, 77777], 4, 4096, 148),
    ([5] * 300, 2, 0, 64),
    ([100, 0, 0], 1, 0, 1000),
    ([64 * (i % 5) + i for i in range(32)], 3, 0, 148),     # B = 32: one-warp planner
    ([64 * (i % 5) + i for i in range(33)], 3, 100, 148),   # B = 33: block-wide planner
])
def test_device_planner_matches_host_model(lib, lens, units, window, P):
    from decode_attention_kv_paged_b200 import planner
    max_blocks = max(1, max((t + 63) // 64 for t in lens))
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    got = lib.plan(sl, units, window, max_blocks, P).cpu().tolist()
    assert got == planner.plan(lens, units, window, max_blocks, P)


# ------------------------------------------------------------ kv_append
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64),
                                     (torch.bfloat16, 256)])
def test_kv_append_places_rows_exactly(lib, dtype, d):
    cfg = GQAConfig("app", B=4, H_q=8, H_kv=4, d=d, seq_lens=[1, 64, 65, 300],
                    dtype=dtype, seed=23)
    inp = make_gqa_inputs(cfg, extra_blocks_per_seq=1).to(DEV)
    g = torch.Generator(device=DEV).manual_seed(2)
    k_new = torch.randn((4, 4, d), generator=g, device=DEV).to(dtype)
    v_new = torch.randn((4, 4, d), generator=g, device=DEV).to(dtype)
    pos = torch.tensor([0, 64, 127, 300], dtype=torch.int32, device=DEV)
    k0, v0 = inp.k_cache.clone(), inp.v_cache.clone()
    lib.kv_append(k_new, v_new, inp.k_cache, inp.v_cache, pos, inp.block_table)
    assert lib.last_error() == lib.OK
    kf, vf = k0.view(-1), v0.view(-1)
    table = inp.block_table.cpu()
    for b in range(4):
        for h in range(4):
            off = orc.slot_offset(table, b, int(pos[b]), BLOCK_SIZE, 4, h, d)
            kf[off:off + d] = k_new[b, h]
            vf[off:off + d] = v_new[b, h]
    assert torch.equal(inp.k_cache, k0)
    assert torch.equal(inp.v_cache, v0)


def test_append_then_decode_sees_new_token(lib):
    """A decode step: append the current token's K/V at position T-1, then
    attend over [0, T) -- the appended row takes part."""
    cfg = GQAConfig("step", B=2, H_q=8, H_kv=2, d=128, seq_lens=[130, 64], seed=31)
    inp = make_gqa_inputs(cfg).to(DEV)
    g = torch.Generator(device=DEV).manual_seed(9)
    k_new = torch.randn((2, 2, 128), generator=g, device=DEV).to(torch.bfloat16) * 4
    v_new = torch.randn((2, 2, 128), generator=g, device=DEV).to(torch.bfloat16)
    pos = (inp.seq_lens - 1).contiguous()
    lib.kv_append(k_new, v_new, inp.k_cache, inp.v_cache, pos, inp.block_table)
    got = run_gpu(lib, inp).float().cpu().numpy()
    assert_parity(got, full_oracle(inp), torch.bfloat16, "append+decode")


# ------------------------------------------------------------ error paths
def test_bad_block_id_is_flagged_not_dereferenced(lib):
    cfg = GQAConfig("bad", B=2, H_q=8, H_kv=2, d=128, seq_lens=[200, 100], seed=3)
    inp = make_gqa_inputs(cfg).to(DEV)
    inp.block_table[1, 0] = 10 ** 6
    lib.decode_gqa(inp.q, inp.k_cache, inp.v_cache, inp.seq_lens, inp.block_table,
                   inp.scale)
    assert lib.last_error() == lib.ERR_BAD_BLOCK
    inp.block_table[1, 0] = -7
    lib.decode_gqa(inp.q, inp.k_cache, inp.v_cache, inp.seq_lens, inp.block_table,
                   inp.scale)
    assert lib.last_error() == lib.ERR_BAD_BLOCK
    assert lib.last_error() == lib.OK            # cleared


def test_bad_seq_len_is_flagged(lib):
    cfg = GQAConfig("badlen", B=2, H_q=8, H_kv=2, d=128, seq_lens=[200, 100], seed=4)
    inp = make_gqa_inputs(cfg).to(DEV)
    inp.seq_lens[0] = 64 * inp.block_table.shape[1] + 1
    out = lib.decode_gqa(inp.q, inp.k_cache, inp.v_cache, inp.seq_lens,
                         inp.block_table, inp.scale)
    assert lib.last_error() == lib.ERR_BAD_SEQLEN
    assert torch.all(out[0] == 0)


def test_forced_timeout_returns_status_and_context_survives(lib):
    """Fault injection: the kernel waits on a barrier nobody signals, gives up
    after 20 ms, reports ATTN_ERR_TIMEOUT; the next call is correct."""
    cfg = GQAConfig("to", B=2, H_q=8, H_kv=2, d=128, seq_lens=[1000, 300], seed=6)
    inp = make_gqa_inputs(cfg)
    ref = full_oracle(inp)
    d = inp.to(DEV)
    lib.debug_force_timeout(True, 20_000_000)
    lib.decode_gqa(d.q, d.k_cache, d.v_cache, d.seq_lens, d.block_table, d.scale)
    assert lib.last_error() == lib.ERR_TIMEOUT
    got = run_gpu(lib, d).float().cpu().numpy()
    assert_parity(got, ref, torch.bfloat16, "after timeout")


def test_host_validation_rejects_bad_arguments(lib):
    inp = make_gqa_inputs(GQAConfig("v", B=1, H_q=6, H_kv=4, d=128, seq_lens=[10],
                                    seed=1)).to(DEV)
    with pytest.raises(lib.AttnError) as e:      # 6 % 4 != 0
        lib.decode_gqa(inp.q, inp.k_cache[:, :4], inp.v_cache[:, :4],
                       inp.seq_lens, inp.block_table, 0.1)
    assert e.value.status == lib.ERR_ARG


# ------------------------------------------------- full-size workloads
def _sampled(lib, cfg, seqs, **kw):
    inp = make_gqa_inputs(cfg, device=DEV, **kw)
    got = run_gpu(lib, inp).float().cpu().numpy()
    ref = oracle_gqa_sequences(inp, seqs)
    for b in seqs:
        assert_parity(got[b], ref[b], torch.bfloat16, f"{cfg.name} b={b}")
    return inp


def test_llama3_8b_shape_full_output(lib):
    """B=16, H_q=32, H_kv=8, d=128, T=4096, bf16, random-permutation table:
    every output compared with the oracle."""
    inp = make_gqa_inputs(LLAMA3_8B)
    got = run_gpu(lib, inp).float().cpu().numpy()
    assert_parity(got, full_oracle(inp), torch.bfloat16, LLAMA3_8B.name)


@pytest.mark.parametrize("cfg", SWEEP, ids=[c.name for c in SWEEP])
def test_head_sharing_sweep_sampled(lib, cfg):
    """H_q=32, d=128, T=32768, H_kv in {32,8,1} x B in {1,8,32}: sampled
    sequences (first and last) vs the oracle."""
    seqs = sorted({0, cfg.B - 1})
    inp = _sampled(lib, cfg, seqs)
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", [RAGGED_FULL, RAGGED_WINDOW],
                         ids=["full", "window4096"])
def test_ragged_qwen_shape_sampled(lib, cfg):
    """H_q=24, H_kv=4 (groups of 6), d=256, B=8, T ~ U[1024, 131072]; full
    causal and w=4096.  The longest and the shortest sequence are checked."""
    inp = make_gqa_inputs(cfg, device=DEV)
    lens = inp.seq_list
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens))})
    if cfg.window > 0:
        table = inp.block_table.clone()
        for b, T in enumerate(lens):
            table[b, : max(0, T - cfg.window) // BLOCK_SIZE] = -1
        inp.block_table = table
    got = run_gpu(lib, inp).float().cpu().numpy()
    ref = oracle_gqa_sequences(inp, seqs)
    for b in seqs:
        assert_parity(got[b], ref[b], torch.bfloat16, f"{cfg.name} b={b}")
    # every output row is a convex combination of V rows: finite and bounded
    assert np.isfinite(got).all()


# ------------------------------------------- both kernels, forced per case
PATH_CASES = [
    # (H_q, H_kv, d, lens, window)
    (8, 8, 128, [300, 65], 0),            # MHA
    (8, 4, 64, [129, 1000], 0),           # G=2
    (16, 4, 128, [700, 64, 1], 0),        # G=4
    (24, 4, 256, [999, 4097], 700),       # G=6 + window
    (32, 4, 128, [2000, 130], 0),         # G=8
    (32, 1, 128, [1500, 63, 64], 0),      # MQA G=32
    (16, 1, 128, [333, 2050, 17], 50),    # G=16: four head copies, window
    (24, 1, 128, [1200, 40], 0),          # G=24: two copies, padded rows
    (48, 1, 64, [900, 129], 0),           # G=48: one copy, padded rows
    (64, 1, 64, [800, 257], 100),         # G=64 + window
    (128, 1, 128, [520, 77], 0),          # G=128: two 64-head passes
]


@pytest.mark.parametrize("path", [0, 1, 2], ids=["cuda_core", "tcgen05", "tcgen05_m64"])
@pytest.mark.parametrize("H_q,H_kv,d,lens,window", PATH_CASES,
                         ids=[f"q{c[0]}_kv{c[1]}_d{c[2]}_w{c[4]}" for c in PATH_CASES])
def test_each_kernel_matches_oracle(lib, path, H_q, H_kv, d, lens, window):
    """The CUDA-core and the tensor-core (tcgen05) kernels each reproduce the
    oracle for every group size, whichever one the library would pick."""
    cfg = GQAConfig("paths", B=len(lens), H_q=H_q, H_kv=H_kv, d=d, seq_lens=lens,
                    window=window, seed=4000 + H_q + d)
    inp = make_gqa_inputs(cfg)
    ref = full_oracle(inp)
    lib.set_gqa_path(path)
    try:
        n, hc, used = lib.gqa_config(len(lens), H_q, H_kv, d)
        # path 1 takes the M=128 kernel where it applies, else the M=64 one
        assert used == path or (path == 1 and used == 2)
        got = run_gpu(lib, inp).float().cpu().numpy()
    finally:
        lib.set_gqa_path(-1)
    assert_parity(got, ref, torch.bfloat16, f"path {path}")


MANY_TILE_CASES = [
    # (H_q, H_kv, d, lens, window): few CTAs, so each walks many tiles and
    # several units -- the tensor-core kernels' rings wrap many times.
    (32, 4, 256, [2000, 700], 0),          # G=8, d=256: two-stage ring
    (48, 2, 256, [1500, 64], 300),         # G=24, d=256, window
    (32, 1, 128, [3000, 129], 0),          # MQA
    (16, 2, 64, [2500, 1], 0),             # G=8, d=64
]


@pytest.mark.parametrize("path", [1, 2], ids=["tcgen05", "tcgen05_m64"])
@pytest.mark.parametrize("H_q,H_kv,d,lens,window", MANY_TILE_CASES,
                         ids=[f"q{c[0]}_kv{c[1]}_d{c[2]}_w{c[4]}" for c in MANY_TILE_CASES])
def test_tensor_core_kernels_many_tiles_per_cta(lib, path, H_q, H_kv, d, lens, window):
    """Three CTAs for the whole batch: every CTA streams tens of tiles through
    its ring and crosses unit boundaries, against the oracle."""
    cfg = GQAConfig("many", B=len(lens), H_q=H_q, H_kv=H_kv, d=d, seq_lens=lens,
                    window=window, seed=4500 + H_q + d)
    inp = make_gqa_inputs(cfg)
    ref = full_oracle(inp)
    lib.set_gqa_path(path)
    lib.set_num_ctas(3)
    try:
        got = run_gpu(lib, inp).float().cpu().numpy()
    finally:
        lib.set_gqa_path(-1)
        lib.set_num_ctas(0)
    assert_parity(got, ref, torch.bfloat16, f"path {path}, 3 CTAs")


@pytest.mark.parametrize("H_q,H_kv,d,expect", [
    (32, 32, 128, 0), (32, 16, 128, 0), (32, 8, 128, 0), (24, 4, 128, 1), (32, 4, 128, 1),
    (16, 2, 64, 1), (24, 4, 256, 2), (36, 4, 128, 1), (32, 1, 128, 1), (48, 1, 64, 2),
    (128, 1, 64, 2), (48, 2, 256, 2)])
def test_automatic_kernel_choice(lib, H_q, H_kv, d, expect):
    """bf16: CUDA cores up to groups of 4 heads; above, the M=128 tensor-core
    kernel where it applies (d <= 128, units of <= 32 heads), else the M=64
    one (the measured crossovers)."""
    _, _, used = lib.gqa_config(4, H_q, H_kv, d)
    assert used == expect


def test_two_streams_run_concurrently_with_their_own_workspaces(lib):
    """Decodes issued alternately on two streams (so they can overlap on the
    GPU) each use their own split workspace and counters: both results match
    the oracle, on every repetition."""
    from tests.parity import oracle_gqa_sequences
    xa = make_gqa_inputs(GQAConfig("s2a", B=4, H_q=32, H_kv=8, d=128,
                                   seq_lens=[3000, 65, 1900, 700], seed=131), device=DEV)
    xb = make_gqa_inputs(GQAConfig("s2b", B=3, H_q=16, H_kv=16, d=64,
                                   seq_lens=[5000, 1, 2500], seed=132), device=DEV)
    refs = [oracle_gqa_sequences(x, range(x.cfg.B)) for x in (xa, xb)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [[torch.empty_like(x.q) for _ in range(6)] for x in (xa, xb)]
    torch.cuda.synchronize()
    for r in range(6):
        for k, (x, s) in enumerate(zip((xa, xb), streams)):
            with torch.cuda.stream(s):
                lib.decode_gqa(x.q, x.k_cache, x.v_cache, x.seq_lens, x.block_table, x.scale,
                               out=outs[k][r], stream=s)
    torch.cuda.synchronize()
    for s in streams:
        assert lib.last_error(s) == lib.OK
    for k, x in enumerate((xa, xb)):
        for r in range(6):
            got = outs[k][r].float().cpu().numpy()
            for b, ref in refs[k].items():
                assert_parity(got[b], ref, torch.bfloat16, f"stream {k} rep {r} b={b}")
