"""GPU parity of the fp8 latent cache for MLA, through the C ABI, vs the
oracle.

The fp8 cache stores each shared latent row (c_j followed by kR_j, 576
values; attention-head §5.4) as OCP E4M3 codes with one fp32 scale per row.
  * kv_append_mla_fp8 must quantise bit for bit like the oracle's row
    quantiser (amax / 448 scale, round-to-nearest-even codes, saturation);
  * attn_decode_mla_fp8 must match the fp64 oracle decode over the dequantised
    cache (code value x row scale) within the bf16 bars: max-abs <= 1e-2,
    rel-L2 <= 2e-3.  The decode is judged on the attention arithmetic; the
    quantisation is checked separately, exactly."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.parity import assert_parity
from workloads import BLOCK_SIZE, MLA_DSV2_FP8, MLAConfig, make_mla_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _quantised(x):
    """(codes, scales) of the bf16 latent cache of x, quantised by the oracle."""
    codes, scales = orc.quantize_rows_e4m3(x.latent_cache.float().numpy())
    return torch.from_numpy(codes), torch.from_numpy(scales)


def _oracle_fp8(x, codes, scales):
    deq = orc.dequantize_e4m3(codes.numpy(), scales.numpy())
    return orc.decode_mla(x.q_lat.double().numpy(), x.q_rope.double().numpy(), deq,
                          x.seq_lens.numpy(), x.block_table.numpy(), x.scale)


def _run(lib, x, codes, scales):
    d = x.to(DEV)
    out = lib.decode_mla_fp8(d.q_lat, d.q_rope, codes.to(DEV), scales.to(DEV), d.seq_lens,
                             d.block_table, d.scale)
    assert lib.last_error() == lib.OK
    return out.float().cpu().numpy()


@pytest.mark.parametrize("lens", [[64], [1], [300, 64], [65, 1, 700], [2048, 5, 129, 64]],
                         ids=lambda v: "T" + "_".join(map(str, v)))
def test_mla_fp8_small_cases_match_oracle(lib, lens):
    x = make_mla_inputs(MLAConfig("mla8", B=len(lens), seq_lens=lens, seed=600 + len(lens)))
    codes, scales = _quantised(x)
    assert_parity(_run(lib, x, codes, scales), _oracle_fp8(x, codes, scales), torch.bfloat16,
                  f"mla fp8 {lens}")


@pytest.mark.parametrize("clusters", [1, 3, 74, 300])
def test_mla_fp8_cluster_count_invariance(lib, clusters):
    x = make_mla_inputs(MLAConfig("mla8s", B=3, seq_lens=[1500, 70, 640], seed=78))
    codes, scales = _quantised(x)
    ref = _oracle_fp8(x, codes, scales)
    lib.set_num_ctas(clusters)
    try:
        got = _run(lib, x, codes, scales)
    finally:
        lib.set_num_ctas(0)
    assert_parity(got, ref, torch.bfloat16, f"fp8 {clusters} clusters")


def test_mla_fp8_unit_variance_rows_and_subnormal_codes(lib):
    """Unit-variance latent rows whose first RoPE value is 1e5 (the matching
    q_rope component is zero, so scores are unaffected): the row scale is set
    by that value, so nearly every content code is an E4M3 subnormal, which
    exercises the exact widening of subnormal codes; judged by the bf16 bars
    (the outputs are averages of O(1) values)."""
    cfg = MLAConfig("mla8u", B=2, seq_lens=[777, 1200], seed=611, value_scale=1.0)
    x = make_mla_inputs(cfg)
    cache = x.latent_cache.float()
    cache[:, :, 512] = 1e5
    x.latent_cache = cache.bfloat16()
    q_rope = x.q_rope.float()
    q_rope[:, :, 0] = 0.0
    x.q_rope = q_rope.bfloat16()
    x.q_lat = (x.q_lat.float() / 24.0).bfloat16()      # scores O(1)
    codes, scales = _quantised(x)
    c = codes.numpy()[:, :, :512]
    subnormal = ((c & 0x78) == 0) & ((c & 0x07) != 0)
    assert subnormal.mean() > 0.5
    assert_parity(_run(lib, x, codes, scales), _oracle_fp8(x, codes, scales), torch.bfloat16,
                  "mla fp8 subnormal codes")


def test_mla_fp8_rescale_path(lib):
    """Scores that grow along the sequence (rows scaled up by a ramp) force the
    running-max rescale with per-row scales in play."""
    cfg = MLAConfig("mla8g", B=2, seq_lens=[1024, 900], seed=19, value_scale=1.0)
    x = make_mla_inputs(cfg)
    ramp = torch.linspace(0.025, 0.5, x.latent_cache.shape[0] * 64).reshape(-1, 64, 1)
    x.latent_cache = (x.latent_cache.float() * ramp).to(torch.bfloat16)
    x.q_lat = (x.q_lat.float() * 6.0).to(torch.bfloat16)
    codes, scales = _quantised(x)
    assert_parity(_run(lib, x, codes, scales), _oracle_fp8(x, codes, scales), torch.bfloat16,
                  "mla fp8 rescale")


def test_kv_append_mla_fp8_bit_exact(lib):
    """Appended rows: codes and scales identical to the oracle's quantiser;
    every other row of the cache untouched."""
    x = make_mla_inputs(MLAConfig("mla8a", B=4, seq_lens=[1, 64, 200, 129], seed=8),
                        extra_blocks_per_seq=1)
    codes, scales = _quantised(x)
    g = torch.Generator().manual_seed(44)
    new = torch.randn((4, 576), generator=g)
    new[1] *= 1e-3                                       # a small row
    new[2] = 0.0                                         # a zero row: scale 0, codes 0
    new[3, 7] = 1e4                                      # one large entry sets the scale
    new = new.bfloat16()
    pos = torch.tensor([0, 64, 199, 128], dtype=torch.int32)
    d_codes, d_scales = codes.to(DEV), scales.to(DEV)
    lib.kv_append_mla_fp8(new.to(DEV), d_codes, d_scales, pos.to(DEV), x.block_table.to(DEV))
    assert lib.last_error() == lib.OK
    want_c, want_s = orc.quantize_rows_e4m3(new.float().numpy())
    exp_codes, exp_scales = codes.clone(), scales.clone()
    table = x.block_table
    for b in range(4):
        p = int(pos[b])
        blk = int(table[b, p // BLOCK_SIZE])
        exp_codes[blk, p % BLOCK_SIZE] = torch.from_numpy(want_c[b])
        exp_scales[blk, p % BLOCK_SIZE] = float(want_s[b])
    assert torch.equal(d_codes.cpu(), exp_codes)
    assert torch.equal(d_scales.cpu(), exp_scales)


def test_mla_fp8_deepseek_v2_shape_sampled(lib):
    """The DeepSeek-V2 shape over an fp8 cache (B=32, T=8192): the first and
    last sequences against the oracle over the dequantised cache."""
    from workloads import MLAConfig as C
    cfg = C("dsv2_fp8_sampled", B=MLA_DSV2_FP8.B, T=MLA_DSV2_FP8.T, seed=MLA_DSV2_FP8.seed)
    x = make_mla_inputs(cfg, device=DEV)
    codes, scales = orc.quantize_rows_e4m3(x.latent_cache.float().cpu().numpy())
    codes_t = torch.from_numpy(codes).to(DEV)
    scales_t = torch.from_numpy(scales).to(DEV)
    got = lib.decode_mla_fp8(x.q_lat, x.q_rope, codes_t, scales_t, x.seq_lens, x.block_table,
                             x.scale).float().cpu().numpy()
    assert lib.last_error() == lib.OK
    assert np.isfinite(got).all()
    for b in (0, cfg.B - 1):
        T = int(x.seq_list[b])
        nb = (T + BLOCK_SIZE - 1) // BLOCK_SIZE
        ids = x.block_table[b, :nb].long().cpu().numpy()
        deq = orc.dequantize_e4m3(codes[ids], scales[ids])
        ref = orc.decode_mla(x.q_lat[b:b + 1].double().cpu().numpy(),
                             x.q_rope[b:b + 1].double().cpu().numpy(), deq,
                             np.array([T], dtype=np.int32),
                             np.arange(nb, dtype=np.int32).reshape(1, nb), x.scale)
        assert_parity(got[b], ref[0], torch.bfloat16, f"mla fp8 dsv2 b={b}")
