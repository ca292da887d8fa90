"""GPU parity of the MLA absorption products on either side of the latent
decode (attention-head §5.2), through the C ABI, vs the oracle.

Stages: q_latent = q_c (U^K_h)^T and o = z U^V_h each against the oracle's
fp64 products of the same bf16 inputs; then the whole absorbed pipeline
(absorb -> latent decode -> project) against the oracle run on the same
pipeline with the same bf16 storage of q_latent and z (the decode API takes
and returns bf16).  The oracle's absorbed pipeline equals explicit MLA in
fp64 (pinned on the CPU).  Bars: bf16 max-abs <= 1e-2, rel-L2 <= 2e-3."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.parity import assert_parity
from workloads import MLA_DSV2, MLAConfig, make_mla_absorb_inputs, make_mla_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16_round(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).bfloat16().double().numpy()


@pytest.mark.parametrize("B", [1, 5, 32, 100, 200])
def test_absorb_q_matches_oracle(lib, B):
    cfg = MLAConfig("absorb", B=B, seq_lens=[64] * B, seed=900 + B)
    w = make_mla_absorb_inputs(cfg)
    got = lib.mla_absorb_q(w.q_c.to(DEV), w.U_K.to(DEV)).float().cpu().numpy()
    ref = orc.mla_absorb_q(w.q_c.double().numpy(), w.U_K.double().numpy())
    assert got.shape == (B, 128, 512)
    assert_parity(got, ref, torch.bfloat16, f"absorb B={B}")


@pytest.mark.parametrize("B", [1, 5, 32, 100, 200])
def test_project_out_matches_oracle(lib, B):
    cfg = MLAConfig("project", B=B, seq_lens=[64] * B, seed=950 + B)
    w = make_mla_absorb_inputs(cfg)
    g = torch.Generator().manual_seed(17 + B)
    z = (torch.randn((B, 128, 512), generator=g) * 0.05).bfloat16()
    got = lib.mla_project_out(z.to(DEV), w.U_V.to(DEV)).float().cpu().numpy()
    ref = orc.mla_project_out(z.double().numpy(), w.U_V.double().numpy())
    assert got.shape == (B, 128, 128)
    assert_parity(got, ref, torch.bfloat16, f"project B={B}")


@pytest.mark.parametrize("lens", [[300, 129], [1, 64, 2050]],
                         ids=lambda v: "T" + "_".join(map(str, v)))
def test_absorbed_pipeline_matches_oracle(lib, lens):
    cfg = MLAConfig("pipeline", B=len(lens), seq_lens=lens, seed=990 + len(lens))
    x = make_mla_inputs(cfg)
    w = make_mla_absorb_inputs(cfg)
    d = x.to(DEV)
    q_lat = lib.mla_absorb_q(w.q_c.to(DEV), w.U_K.to(DEV))
    z = lib.decode_mla(q_lat, d.q_rope, d.latent_cache, d.seq_lens, d.block_table, d.scale)
    assert lib.last_error() == lib.OK
    o = lib.mla_project_out(z, w.U_V.to(DEV)).float().cpu().numpy()

    q_ref = _bf16_round(orc.mla_absorb_q(w.q_c.double().numpy(), w.U_K.double().numpy()))
    z_ref = orc.decode_mla(q_ref, x.q_rope.double().numpy(), x.latent_cache.double().numpy(),
                           x.seq_lens.numpy(), x.block_table.numpy(), x.scale)
    o_ref = orc.mla_project_out(_bf16_round(z_ref), w.U_V.double().numpy())
    assert_parity(o, o_ref, torch.bfloat16, f"pipeline {lens}")


def test_absorb_host_validation(lib):
    w = make_mla_absorb_inputs(MLAConfig("v", B=1, seq_lens=[1], seed=1))
    with pytest.raises(ValueError):
        lib.mla_absorb_q(w.q_c.to(DEV), w.U_K[:, :, :64].to(DEV))
    with pytest.raises(lib.AttnError) as e:        # d_h not a multiple of 64
        lib.mla_absorb_q(w.q_c[:, :, :48].contiguous().to(DEV),
                         w.U_K[:, :, :48].contiguous().to(DEV))
    assert e.value.status == lib.ERR_UNSUPPORTED
    with pytest.raises(lib.AttnError) as e:        # d_v not a multiple of 128
        z = torch.zeros((1, 128, 512), dtype=torch.bfloat16, device=DEV)
        lib.mla_project_out(z, w.U_V[:, :, :64].contiguous().to(DEV))
    assert e.value.status == lib.ERR_UNSUPPORTED


def _within_one_ulp(got, ref):
    """Every output is within one bf16 ulp of the exact product (the kernel
    rounds an fp32 accumulation once): a check that holds at any scale."""
    ref = np.asarray(ref, dtype=np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    return np.abs(np.asarray(got, dtype=np.float64) - ref) <= ulp + 1e-6


def test_absorb_q_unit_variance_weights(lib):
    """U^K ~ N(0, 1/d_h) (unit-variance products, extremes near 5): judged by
    the relative L2 bar and by one-ulp agreement with the exact fp64 product,
    instead of the max-abs bar that bf16 storage of values near 5 alone breaks."""
    g = torch.Generator().manual_seed(4242)
    B, H, d_c, d_h = 32, 128, 512, 128
    q_c = torch.randn((B, H, d_h), generator=g).bfloat16()
    U_K = (torch.randn((H, d_c, d_h), generator=g) / np.sqrt(d_h)).bfloat16()
    got = lib.mla_absorb_q(q_c.to(DEV), U_K.to(DEV)).float().cpu().numpy()
    ref = orc.mla_absorb_q(q_c.double().numpy(), U_K.double().numpy())
    assert np.abs(ref).max() > 3.0
    from tests.parity import errors
    _, rel = errors(got, ref)
    assert rel <= 2e-3, rel
    ok = _within_one_ulp(got, ref)
    assert ok.all(), f"{(~ok).sum()} outputs off by more than one bf16 ulp"


def test_project_out_unit_variance(lib):
    """z ~ N(0, 1), U^V ~ N(0, 1/d_c): the same one-ulp and rel-L2 checks."""
    g = torch.Generator().manual_seed(4343)
    B, H, d_c, d_v = 32, 128, 512, 128
    z = torch.randn((B, H, d_c), generator=g).bfloat16()
    U_V = (torch.randn((H, d_c, d_v), generator=g) / np.sqrt(d_c)).bfloat16()
    got = lib.mla_project_out(z.to(DEV), U_V.to(DEV)).float().cpu().numpy()
    ref = orc.mla_project_out(z.double().numpy(), U_V.double().numpy())
    from tests.parity import errors
    _, rel = errors(got, ref)
    assert rel <= 2e-3, rel
    ok = _within_one_ulp(got, ref)
    assert ok.all(), f"{(~ok).sum()} outputs off by more than one bf16 ulp"
