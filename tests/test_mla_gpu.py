"""GPU parity of the absorbed-MLA decode path (tcgen05, cluster pairs) vs the
oracle, through the C ABI.  Bars: bf16 max-abs <= 1e-2, rel-L2 <= 2e-3."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.parity import assert_parity, oracle_mla_sequences
from workloads import BLOCK_SIZE, MLA_DSV2, MLAConfig, make_mla_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_gpu(attn, x):
    d = x.to(DEV) if x.q_lat.device.type != "cuda" else x
    out = attn.decode_mla(d.q_lat, d.q_rope, d.latent_cache, d.seq_lens, d.block_table,
                          d.scale)
    assert attn.last_error() == attn.OK
    return out


def full_oracle(x):
    return orc.decode_mla(x.q_lat.cpu(), x.q_rope.cpu(), x.latent_cache.cpu(),
                          x.seq_lens.cpu(), x.block_table.cpu(), x.scale)


@pytest.mark.parametrize("lens", [[64], [1], [300, 64], [65, 1, 700], [2048, 5, 129, 64]],
                         ids=lambda v: "T" + "_".join(map(str, v)))
def test_mla_small_cases_match_oracle(lib, lens):
    x = make_mla_inputs(MLAConfig("mla_small", B=len(lens), seq_lens=lens, seed=500 + len(lens)))
    got = run_gpu(lib, x).float().cpu().numpy()
    assert_parity(got, full_oracle(x), torch.bfloat16, f"mla {lens}")


@pytest.mark.parametrize("clusters", [1, 2, 7, 74, 300])
def test_mla_cluster_count_invariance(lib, clusters):
    """Any number of cluster ranges (including ones that split a single
    block per cluster, and more clusters than blocks) gives the oracle."""
    x = make_mla_inputs(MLAConfig("mla_split", B=3, seq_lens=[1500, 70, 640], seed=77))
    ref = full_oracle(x)
    lib.set_num_ctas(clusters)
    try:
        got = run_gpu(lib, x).float().cpu().numpy()
    finally:
        lib.set_num_ctas(0)
    assert_parity(got, ref, torch.bfloat16, f"{clusters} clusters")


def test_mla_many_sequences_ragged_match_oracle(lib):
    """Enough sequences that the 8-head combine merges the cluster partials
    (few partials per sequence): ragged lengths, empty sequences, one-token
    and block-edge lengths; every sequence against the oracle."""
    lens = [0, 1, 64, 65, 700, 3000, 5, 128, 129, 2048, 0, 63, 1000, 17, 640, 4096]
    x = make_mla_inputs(MLAConfig("mla_many", B=len(lens), seq_lens=lens, seed=31))
    got = run_gpu(lib, x).float().cpu().numpy()
    ref = oracle_mla_sequences(x, [b for b, T in enumerate(lens) if T > 0])
    for b, T in enumerate(lens):
        if T == 0:
            assert np.all(got[b] == 0), f"empty sequence {b}"
        else:
            assert_parity(got[b], ref[b], torch.bfloat16, f"mla many b={b} T={T}")


def test_mla_combine_sequence_spanning_many_clusters(lib):
    """20 sequences over 140 clusters, one holding 95 % of the tiles: it
    spans more clusters than the 8-head combine keeps weights for in shared
    memory (its further weights are recomputed from the log-sum-exps)."""
    lens = [20000] + [64] * 18 + [0]
    x = make_mla_inputs(MLAConfig("mla_span", B=len(lens), seq_lens=lens, seed=41))
    tiles = [(T + BLOCK_SIZE - 1) // BLOCK_SIZE for T in lens]
    W, P = sum(tiles), 140
    last_cluster = (tiles[0] - 1) * P // W           # cluster of the long sequence's last tile
    assert last_cluster + 1 > 128                    # the case this test is for
    lib.set_num_ctas(P)
    try:
        got = run_gpu(lib, x).float().cpu().numpy()
    finally:
        lib.set_num_ctas(0)
    ref = oracle_mla_sequences(x, [0, 1, 18])
    for b, r in ref.items():
        assert_parity(got[b], r, torch.bfloat16, f"mla span b={b}")
    assert np.all(got[19] == 0)


def test_mla_empty_sequence_gives_zero_row(lib):
    x = make_mla_inputs(MLAConfig("mla_empty", B=3, seq_lens=[0, 100, 0], seed=5))
    got = run_gpu(lib, x).float().cpu().numpy()
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    assert_parity(got[1], full_oracle(x)[1], torch.bfloat16, "mla empty")


def test_mla_large_scores_rescale_path(lib):
    """Scores that grow along the sequence force the running-max rescale of
    the TMEM accumulator; the result must still match the oracle."""
    cfg = MLAConfig("mla_grow", B=2, seq_lens=[1024, 900], seed=9, value_scale=1.0)
    x = make_mla_inputs(cfg)
    # latent magnitudes grow 20x along the cache (scores too); outputs stay
    # below 2 so bf16 output rounding stays inside the max-abs bar
    ramp = torch.linspace(0.025, 0.5, x.latent_cache.shape[0] * 64).reshape(-1, 64, 1)
    x.latent_cache = (x.latent_cache.float() * ramp).to(torch.bfloat16)
    x.q_lat = (x.q_lat.float() * 6.0).to(torch.bfloat16)
    got = run_gpu(lib, x).float().cpu().numpy()
    assert_parity(got, full_oracle(x), torch.bfloat16, "mla rescale")


def test_mla_bad_block_flagged(lib):
    x = make_mla_inputs(MLAConfig("mla_bad", B=2, seq_lens=[200, 100], seed=3)).to(DEV)
    x.block_table[0, 1] = 10 ** 6
    lib.decode_mla(x.q_lat, x.q_rope, x.latent_cache, x.seq_lens, x.block_table, x.scale)
    assert lib.last_error() == lib.ERR_BAD_BLOCK


def test_mla_unsupported_shapes(lib):
    x = make_mla_inputs(MLAConfig("mla_h64", B=1, H=64, seq_lens=[64], seed=3)).to(DEV)
    with pytest.raises(lib.AttnError) as e:
        lib.decode_mla(x.q_lat, x.q_rope, x.latent_cache, x.seq_lens, x.block_table,
                       x.scale)
    assert e.value.status == lib.ERR_UNSUPPORTED


def test_kv_append_mla_places_rows_exactly(lib):
    x = make_mla_inputs(MLAConfig("mla_app", B=3, seq_lens=[1, 64, 200], seed=8),
                        extra_blocks_per_seq=1).to(DEV)
    g = torch.Generator(device=DEV).manual_seed(4)
    new = torch.randn((3, 576), generator=g, device=DEV).to(torch.bfloat16)
    pos = torch.tensor([0, 64, 199], dtype=torch.int32, device=DEV)
    before = x.latent_cache.clone()
    lib.kv_append_mla(new, x.latent_cache, pos, x.block_table)
    assert lib.last_error() == lib.OK
    flat = before.view(-1)
    table = x.block_table.cpu()
    for b in range(3):
        off = orc.slot_offset(table, b, int(pos[b]), BLOCK_SIZE, 1, 0, 576)
        flat[off:off + 576] = new[b]
    assert torch.equal(x.latent_cache, before)


def test_mla_deepseek_v2_shape_sampled(lib):
    """H=128, 512 + 64 latent, B=32, T=8192, values N(0,1)/sqrt(576), scale
    1/sqrt(192): first and last sequences against the oracle, all finite."""
    x = make_mla_inputs(MLA_DSV2, device=DEV)
    got = run_gpu(lib, x).float().cpu().numpy()
    ref = oracle_mla_sequences(x, [0, MLA_DSV2.B - 1])
    for b, r in ref.items():
        assert_parity(got[b], r, torch.bfloat16, f"mla full b={b}")
    assert np.isfinite(got).all()
