"""GPU parity of decode with global (sink) tokens and a ring-buffer block
table (attn_decode_gqa_ext, kv_append_ext) vs the oracle's decode_gqa_vis,
through the C ABI, on every GQA kernel.  Bars: bf16 max-abs <= 1e-2,
rel-L2 <= 2e-3."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.parity import assert_parity
from workloads import BLOCK_SIZE

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(seed, B, H_q, H_kv, d, n_blocks, slots):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, H_q, d), generator=g).bfloat16()
    k = torch.randn((n_blocks, H_kv, BLOCK_SIZE, d), generator=g).bfloat16()
    v = torch.randn((n_blocks, H_kv, BLOCK_SIZE, d), generator=g).bfloat16()
    table = torch.randperm(n_blocks, generator=g)[: B * slots].reshape(B, slots)
    return q, k, v, table.to(torch.int32)


def _oracle(q, k, v, lens, table, scale, window, sink, ring):
    return orc.decode_gqa_vis(q, k, v, np.asarray(lens, dtype=np.int32), table.numpy(), scale,
                              window=window, sink=sink, ring=ring)


VIS_CASES = [
    # (H_q, H_kv, d, lens, window, sink)
    (32, 8, 128, [1000, 70, 5, 4097], 100, 4),
    (32, 1, 128, [3000, 64, 130], 500, 64),
    (8, 8, 64, [700, 300, 1], 33, 100),
    (24, 4, 256, [5000, 129], 1000, 7),
]


@pytest.mark.parametrize("path", [0, 1, 2], ids=["cuda_core", "tcgen05", "tcgen05_m64"])
@pytest.mark.parametrize("H_q,H_kv,d,lens,window,sink", VIS_CASES,
                         ids=[f"q{c[0]}_kv{c[1]}_d{c[2]}_w{c[4]}_g{c[5]}" for c in VIS_CASES])
def test_window_plus_sink_matches_oracle(lib, path, H_q, H_kv, d, lens, window, sink):
    B = len(lens)
    slots = max((T + 63) // 64 for T in lens)
    q, k, v, table = _inputs(7000 + H_q + d + window, B, H_q, H_kv, d, B * slots + 3, slots)
    scale = 1.0 / np.sqrt(d)
    ref = _oracle(q, k, v, lens, table, scale, window, sink, 0)
    lib.set_gqa_path(path)
    try:
        got = lib.decode_gqa_ext(q.to(DEV), k.to(DEV), v.to(DEV),
                                 torch.tensor(lens, dtype=torch.int32, device=DEV),
                                 table.to(DEV), scale, window=window, sink_tokens=sink)
        assert lib.last_error() == lib.OK
    finally:
        lib.set_gqa_path(-1)
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, f"vis path {path}")


@pytest.mark.parametrize("path", [0, 1], ids=["cuda_core", "tcgen05"])
def test_ring_table_matches_oracle(lib, path):
    """Sequences far longer than the table row: the ring of 4 blocks after
    one sink block holds the window (w=150); the oracle reads the same cache
    through the same slot mapping."""
    lens, window, sink, ring = [9000, 640, 151, 20000], 150, 10, 4
    H_q, H_kv, d = 16, 2 if path == 0 else 1, 128
    slots = 1 + ring
    q, k, v, table = _inputs(7100 + path, len(lens), H_q, H_kv, d, len(lens) * slots + 5,
                             slots)
    scale = 0.09
    ref = _oracle(q, k, v, lens, table, scale, window, sink, ring)
    lib.set_gqa_path(path)
    try:
        got = lib.decode_gqa_ext(q.to(DEV), k.to(DEV), v.to(DEV),
                                 torch.tensor(lens, dtype=torch.int32, device=DEV),
                                 table.to(DEV), scale, window=window, sink_tokens=sink,
                                 ring_blocks=ring)
        assert lib.last_error() == lib.OK
    finally:
        lib.set_gqa_path(-1)
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, f"ring path {path}")


def test_ring_append_evicts_and_decode_matches_full_cache(lib):
    """Append every token of two sequences one step at a time into a ring
    table (window 100 + sink 5 in 1 + 3 slots): blocks that leave the window
    are overwritten, the sink block is kept, and the final decode equals the
    oracle over the full (never evicted) cache with the same visibility."""
    T, window, sink, ring, H_kv, H_q, d = 700, 100, 5, 3, 2, 8, 64
    B = 2
    g = torch.Generator().manual_seed(7200)
    k_all = torch.randn((B, T, H_kv, d), generator=g).bfloat16()
    v_all = torch.randn((B, T, H_kv, d), generator=g).bfloat16()
    q = torch.randn((B, H_q, d), generator=g).bfloat16()
    slots = 1 + ring
    table = torch.tensor([[3, 0, 6, 1], [7, 2, 4, 5]], dtype=torch.int32)
    kc = torch.zeros((8, H_kv, BLOCK_SIZE, d), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    td = table.to(DEV)
    kd, vd = k_all.to(DEV), v_all.to(DEV)
    for t in range(T):
        pos = torch.full((B,), t, dtype=torch.int32, device=DEV)
        lib.kv_append_ext(kd[:, t].contiguous(), vd[:, t].contiguous(), kc, vc, pos, td,
                          window=window, sink_tokens=sink, ring_blocks=ring)
    assert lib.last_error() == lib.OK
    lens = torch.full((B,), T, dtype=torch.int32, device=DEV)
    got = lib.decode_gqa_ext(q.to(DEV), kc, vc, lens, td, 0.15, window=window,
                             sink_tokens=sink, ring_blocks=ring)
    assert lib.last_error() == lib.OK
    # Full, never-evicted cache with an identity table per sequence.
    nb = (T + 63) // 64
    full_k = torch.zeros((B * nb, H_kv, BLOCK_SIZE, d), dtype=torch.bfloat16)
    full_v = torch.zeros_like(full_k)
    for b in range(B):
        for t in range(T):
            full_k[b * nb + t // 64, :, t % 64] = k_all[b, t]
            full_v[b * nb + t // 64, :, t % 64] = v_all[b, t]
    full_table = torch.arange(B * nb, dtype=torch.int32).reshape(B, nb)
    ref = _oracle(q, full_k, full_v, [T] * B, full_table, 0.15, window, sink, 0)
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, "ring append")


def test_visibility_host_validation(lib):
    q, k, v, table = _inputs(1, 1, 4, 2, 64, 8, 4)
    args = (q.to(DEV), k.to(DEV), v.to(DEV), torch.tensor([100], dtype=torch.int32,
                                                          device=DEV), table.to(DEV), 0.1)
    for kw in (dict(ring_blocks=2),                              # ring needs a window
               dict(window=200, ring_blocks=3),                  # ring too small for w
               dict(window=64, sink_tokens=65, ring_blocks=3),   # 2 sink + 3 ring > 4
               dict(window=10, sink_tokens=-1)):
        with pytest.raises(lib.AttnError) as e:
            lib.decode_gqa_ext(*args, **kw)
        assert e.value.status == lib.ERR_ARG, kw


GLOBAL_CASES = [
    # (H_q, H_kv, d, lens, window, global rows (-1 padded))
    (32, 8, 128, [1000, 300, 4097, 65],
     [[0, 5, 130, 700], [299, -1, -1, -1], [1, 2, 64, 3000], [-1, -1, -1, -1]], 200),
    (32, 1, 128, [3000, 640, 1],
     [[0, 70, 71, 200, 1500, 2990], [0, 639, -1, -1, -1, -1], [0, -1, -1, -1, -1, -1]], 100),
    (24, 4, 256, [5000, 129],
     [[10, 64 * 20 + 3, 64 * 40, 4000], [5, 6, 7, -1]], 700),
    (8, 8, 64, [700, 300], [[4, 7, 6, 600], [3] + [-1] * 3], 33),
]


@pytest.mark.parametrize("path", [0, 1, 2], ids=["cuda_core", "tcgen05", "tcgen05_m64"])
@pytest.mark.parametrize("H_q,H_kv,d,lens,rows,window", GLOBAL_CASES,
                         ids=[f"q{c[0]}_kv{c[1]}_d{c[2]}_w{c[5]}" for c in GLOBAL_CASES])
def test_global_positions_match_oracle(lib, path, H_q, H_kv, d, lens, rows, window):
    """Window plus an explicit global set per sequence (attention-head §3,
    G = {0, 5} in its figure): blocks before the window are read only where
    a global position lies, keys in them are masked to the set, and a query
    that is itself global sees everything; every kernel vs the oracle."""
    B = len(lens)
    slots = max((T + 63) // 64 for T in lens)
    q, k, v, table = _inputs(7300 + H_q + d, B, H_q, H_kv, d, B * slots + 3, slots)
    gp = torch.tensor(rows, dtype=torch.int32)
    scale = 1.0 / np.sqrt(d)
    ref = orc.decode_gqa_vis(q, k, v, np.asarray(lens, dtype=np.int32), table.numpy(), scale,
                             window=window, global_pos=gp.numpy())
    lib.set_gqa_path(path)
    try:
        got = lib.decode_gqa_ext(q.to(DEV), k.to(DEV), v.to(DEV),
                                 torch.tensor(lens, dtype=torch.int32, device=DEV),
                                 table.to(DEV), scale, window=window, global_pos=gp.to(DEV))
        assert lib.last_error() == lib.OK
    finally:
        lib.set_gqa_path(-1)
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, f"global set, path {path}")


def test_global_positions_many_tiles_per_cta(lib):
    """Three CTAs over the batch: global blocks and window runs of several
    sequences in one CTA's range, on both tensor-core kernels and CUDA cores."""
    lens = [2000, 1500, 700]
    rows = [[0, 1, 500, 1000], [64, 900, -1, -1], [699, -1, -1, -1]]
    for path, (H_q, H_kv, d) in ((0, (32, 8, 128)), (1, (32, 2, 128)), (2, (48, 2, 256))):
        B = len(lens)
        slots = max((T + 63) // 64 for T in lens)
        q, k, v, table = _inputs(7400 + path, B, H_q, H_kv, d, B * slots + 2, slots)
        gp = torch.tensor(rows, dtype=torch.int32)
        ref = orc.decode_gqa_vis(q, k, v, np.asarray(lens, dtype=np.int32), table.numpy(), 0.1,
                                 window=250, global_pos=gp.numpy())
        lib.set_gqa_path(path)
        lib.set_num_ctas(3)
        try:
            got = lib.decode_gqa_ext(q.to(DEV), k.to(DEV), v.to(DEV),
                                     torch.tensor(lens, dtype=torch.int32, device=DEV),
                                     table.to(DEV), 0.1, window=250, global_pos=gp.to(DEV))
            assert lib.last_error() == lib.OK
        finally:
            lib.set_gqa_path(-1)
            lib.set_num_ctas(0)
        assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, f"path {path}")


def test_global_positions_host_validation(lib):
    q, k, v, table = _inputs(2, 1, 4, 2, 64, 8, 4)
    args = (q.to(DEV), k.to(DEV), v.to(DEV), torch.tensor([100], dtype=torch.int32,
                                                          device=DEV), table.to(DEV), 0.1)
    gp = torch.tensor([[0, 5]], dtype=torch.int32, device=DEV)
    for kw, status in ((dict(window=10, sink_tokens=4, global_pos=gp), lib.ERR_ARG),
                       (dict(window=64, ring_blocks=3, global_pos=gp), lib.ERR_ARG),
                       (dict(window=10, global_pos=torch.zeros((1, 65), dtype=torch.int32,
                                                               device=DEV)),
                        lib.ERR_UNSUPPORTED)):
        with pytest.raises(lib.AttnError) as e:
            lib.decode_gqa_ext(*args, **kw)
        assert e.value.status == status, kw


def _global_ring_table(rng, B, lens, window, ring, rows, n_phys):
    """Per sequence: n_g global slots + `ring` ring slots.  Global slot k
    names one physical block per distinct block of the positions (slots of
    positions sharing a block share it; pads stay -1), ring slot n_g + i %
    ring names the block of logical block i for the blocks the window
    reaches.  All blocks are distinct; the pool holds spares nothing names."""
    n_g = len(rows[0])
    table = np.full((B, n_g + ring), -1, dtype=np.int32)
    perm = iter(rng.permutation(n_phys).tolist())
    for b in range(B):
        by_block = {}
        for k, pos in enumerate(rows[b]):
            if pos < 0:
                continue
            if pos // 64 not in by_block:
                by_block[pos // 64] = next(perm)
            table[b, k] = by_block[pos // 64]
        for r in range(ring):
            table[b, n_g + r] = next(perm)
    return torch.from_numpy(table)


GLOBAL_RING_CASES = [
    # (H_q, H_kv, d, lens, rows, window, ring)
    (16, 2, 128, [9000, 640, 151, 20000],
     [[0, 5, 70, 3000, 8990], [3, 600, -1, -1, -1], [0, 149, -1, -1, -1],
      [64, 65, 19000, 19950, -1]], 150, 4),
    (32, 1, 128, [5000, 130], [[1, 2, 4700, 4900], [129, -1, -1, -1]], 400, 8),
    (24, 4, 256, [3000, 2999], [[10, 1300, 2900, -1], [0, 2000, 2950, -1]], 100, 3),
]


@pytest.mark.parametrize("path", [0, 1, 2], ids=["cuda_core", "tcgen05", "tcgen05_m64"])
@pytest.mark.parametrize("H_q,H_kv,d,lens,rows,window,ring", GLOBAL_RING_CASES,
                         ids=[f"q{c[0]}_kv{c[1]}_d{c[2]}_w{c[5]}_r{c[6]}"
                              for c in GLOBAL_RING_CASES])
def test_global_set_with_ring_matches_oracle(lib, path, H_q, H_kv, d, lens, rows, window,
                                             ring):
    """A window layer that also keeps an explicit global set in a ring table
    (attention-head §3): global slots ahead of the ring, sequences far longer
    than the row; every kernel vs the oracle through the same table."""
    B = len(lens)
    n_phys = B * (len(rows[0]) + ring) + 4
    q, k, v, _ = _inputs(7500 + H_q + d, B, H_q, H_kv, d, n_phys, 1)
    table = _global_ring_table(np.random.default_rng(7500 + d), B, lens, window, ring, rows,
                               n_phys)
    gp = torch.tensor(rows, dtype=torch.int32)
    scale = 1.0 / np.sqrt(d)
    ref = orc.decode_gqa_vis(q, k, v, np.asarray(lens, dtype=np.int32), table.numpy(), scale,
                             window=window, ring=ring, global_pos=gp.numpy())
    lib.set_gqa_path(path)
    try:
        got = lib.decode_gqa_ext(q.to(DEV), k.to(DEV), v.to(DEV),
                                 torch.tensor(lens, dtype=torch.int32, device=DEV),
                                 table.to(DEV), scale, window=window, ring_blocks=ring,
                                 global_pos=gp.to(DEV))
        assert lib.last_error() == lib.OK
    finally:
        lib.set_gqa_path(-1)
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16,
                  f"global set + ring, path {path}")


@pytest.mark.parametrize("path", [0, 1], ids=["cuda_core", "tcgen05"])
def test_global_query_with_ring_is_flagged(lib, path):
    """A global query (T - 1 in G) with T > window needs history the ring no
    longer holds: that sequence is refused on the device (bad sequence
    length, zero output row) and the others are served."""
    lens, rows, window, ring = [3000, 1000], [[5, 2999], [7, -1]], 200, 5
    H_q, H_kv, d = 16, 2, 128
    B = len(lens)
    n_phys = B * (2 + ring) + 2
    q, k, v, _ = _inputs(7600 + path, B, H_q, H_kv, d, n_phys, 1)
    table = _global_ring_table(np.random.default_rng(7600), B, lens, window, ring, rows, n_phys)
    gp = torch.tensor(rows, dtype=torch.int32)
    ref1 = orc.decode_gqa_vis(q[1:], k, v, np.asarray(lens[1:], dtype=np.int32),
                              table[1:].numpy(), 0.1, window=window, ring=ring,
                              global_pos=gp[1:].numpy())
    lib.set_gqa_path(path)
    try:
        got = lib.decode_gqa_ext(q.to(DEV), k.to(DEV), v.to(DEV),
                                 torch.tensor(lens, dtype=torch.int32, device=DEV),
                                 table.to(DEV), 0.1, window=window, ring_blocks=ring,
                                 global_pos=gp.to(DEV))
        assert lib.last_error() == lib.ERR_BAD_SEQLEN
        assert lib.last_error() == lib.OK            # reading clears it
    finally:
        lib.set_gqa_path(-1)
    got = got.float().cpu()
    assert torch.count_nonzero(got[0]) == 0
    assert_parity(got[1:].numpy(), ref1, torch.bfloat16, f"served rows, path {path}")


def test_global_set_ring_append_then_decode_matches_full_cache(lib):
    """Append every token of two sequences one step at a time into a ring
    table with global slots, the caller keeping a global position's block
    alive (the ring slot gets a fresh block when it comes round): the final
    decode equals the oracle over the full, never-evicted cache with the
    same window and global set."""
    T, window, ring, H_kv, H_q, d = 900, 100, 3, 2, 8, 64
    rows = [[0, 5, 300, 301, 700], [64, 890, -1, -1, -1]]
    B, n_g = 2, len(rows[0])
    g = torch.Generator().manual_seed(7700)
    k_all = torch.randn((B, T, H_kv, d), generator=g).bfloat16()
    v_all = torch.randn((B, T, H_kv, d), generator=g).bfloat16()
    q = torch.randn((B, H_q, d), generator=g).bfloat16()
    n_phys = 32
    free = list(range(n_phys))[::-1]
    table = np.full((B, n_g + ring), -1, dtype=np.int32)
    pinned = [set() for _ in range(B)]
    kc = torch.zeros((n_phys, H_kv, BLOCK_SIZE, d), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    td = torch.from_numpy(table).to(DEV)
    gp = torch.tensor(rows, dtype=torch.int32, device=DEV)
    kd, vd = k_all.to(DEV), v_all.to(DEV)
    for t in range(T):
        if t % 64 == 0:                       # a new block: the cache manager's step
            i = t // 64
            for b in range(B):
                r = n_g + i % ring
                old = table[b, r]
                if old < 0 or old in pinned[b]:
                    table[b, r] = free.pop()  # fresh block; a pinned one stays alive
                for kk, pos in enumerate(rows[b]):
                    if pos >= 0 and pos // 64 == i:
                        table[b, kk] = table[b, r]
                        pinned[b].add(int(table[b, r]))
            td.copy_(torch.from_numpy(table))
        pos = torch.full((B,), t, dtype=torch.int32, device=DEV)
        lib.kv_append_ext(kd[:, t].contiguous(), vd[:, t].contiguous(), kc, vc, pos, td,
                          window=window, ring_blocks=ring, global_pos=gp)
    assert lib.last_error() == lib.OK
    lens = torch.full((B,), T, dtype=torch.int32, device=DEV)
    got = lib.decode_gqa_ext(q.to(DEV), kc, vc, lens, td, 0.15, window=window,
                             ring_blocks=ring, global_pos=gp)
    assert lib.last_error() == lib.OK
    nb = (T + 63) // 64
    full_k = torch.zeros((B * nb, H_kv, BLOCK_SIZE, d), dtype=torch.bfloat16)
    full_v = torch.zeros_like(full_k)
    for b in range(B):
        for t in range(T):
            full_k[b * nb + t // 64, :, t % 64] = k_all[b, t]
            full_v[b * nb + t // 64, :, t % 64] = v_all[b, t]
    full_table = np.arange(B * nb, dtype=np.int32).reshape(B, nb)
    ref = orc.decode_gqa_vis(q, full_k, full_v, np.array([T] * B, dtype=np.int32), full_table,
                             0.15, window=window, global_pos=np.asarray(rows, dtype=np.int32))
    assert_parity(got.float().cpu().numpy(), ref, torch.bfloat16, "global set ring append")
