"""GPU parity of the whole chunk step (selection and attention) on a fixed sweep of
randomly drawn small shapes: dtype, head_dim, group size, chunk length, batch, prefix and
budget per sequence, kept-query count and input recipe are drawn together, so the sweep
reaches combinations of paths (decode and chunk kernels, column groups, padded query
heads, empty prefixes, budgets below, at and above the prefix) that the hand-picked cases
do not.  The draw is seeded, so every run checks the same cases."""
import numpy as np
import pytest

from query_oriented_sparse_b200 import workloads as W

from gpu_harness import check_step, run_gpu

pytestmark = pytest.mark.gpu

N_CASES = 48


def _draw(i: int) -> W.Workload:
    rng = np.random.default_rng(5000 + i)
    dtype = "f32" if rng.random() < 0.3 else "bf16"
    head_dim = int(rng.choice([64, 128]))
    G = int(rng.choice([1, 2, 3, 4, 6, 8, 12, 16]))
    h_kv = int(rng.choice([1, 2, 4])) if G <= 8 else int(rng.choice([1, 2]))
    chunk = int(rng.choice([1, 2, 3, 5, 16, 31, 64, 100, 127, 200, 257, 300, 513]))
    batch = int(rng.integers(1, 4))
    prefix = tuple(int(p) for p in rng.integers(0, 5001, size=batch))
    prefix = tuple(0 if rng.random() < 0.15 else p for p in prefix)
    budget = tuple(int(min(rng.integers(0, 400), p + 50)) if rng.random() < 0.9 else p + 10
                   for p in prefix)
    nq = int(rng.integers(1, chunk + 11))
    recipe = str(rng.choice(["gauss", "rank4", "heavy"]))
    name = f"rand{i:02d}_{dtype}_d{head_dim}_g{G}x{h_kv}_c{chunk}_b{batch}_nq{nq}"
    return W.custom(name, h_q=G * h_kv, h_kv=h_kv, head_dim=head_dim, chunk=chunk, prefix=prefix,
                    nq=nq, budget=budget, dtype=dtype, seed=700 + i, recipe=recipe)


CASES = [_draw(i) for i in range(N_CASES)]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_random_shape_parity(w, cuda_device):
    t = W.generate(w)
    res = run_gpu(w, t)
    rep = check_step(w, t, res)
    print(w.name, w.prefix, w.budget, rep)
