"""Host logic of the benchmark's byte model: the visible-key and visible-tile
counts it divides by must follow the visibility definition (window plus
global tokens), checked against brute force on the CPU."""
import importlib.util
import os
import random
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_model", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_visible_keys_and_tiles_match_brute_force():
    b = _bench()
    rng = random.Random(5)
    for _ in range(3000):
        T = rng.randint(0, 700)
        w = rng.choice([0, 1, 5, 63, 64, 100, 700])
        g = rng.choice([0, 1, 3, 63, 64, 65, 200, 1000])
        keys = [j for j in range(T) if w <= 0 or j >= T - w or j < g]
        assert b.visible_keys(T, w, g) == len(keys), (T, w, g)
        assert b.visible_tiles(T, w, g) == len({j // 64 for j in keys}), (T, w, g)


def test_visible_key_and_tile_counts_with_global_sets():
    """The bench's byte model for explicit global sets counts exactly the
    keys (and 64-token blocks) the definition makes visible, brute force."""
    bench = _bench()
    rng = random.Random(5)
    for _ in range(3000):
        T = rng.randint(0, 400)
        w = rng.choice([0, 1, 5, 64, 100, 500])
        row = sorted(rng.sample(range(0, 450), rng.randint(0, 6))) + [-1] * 3
        if rng.random() < 0.2 and len(row) > 4:
            row[2], row[1] = row[1], row[2]        # a non-ascending entry ends the row
        G = bench._global_set(row)
        if T <= 0:
            keys = set()
        elif w <= 0 or (T - 1) in G:
            keys = set(range(T))
        else:
            keys = {j for j in range(T) if j >= T - w or j in G}
        assert bench.visible_keys_global(T, w, row) == len(keys), (T, w, row)
        assert bench.visible_tiles_global(T, w, row) == len({j // 64 for j in keys}), (T, w, row)
