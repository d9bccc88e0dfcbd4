"""The test-side row-parallel oracle driver returns exactly what one oracle call returns."""
import numpy as np

import oracle
import workloads
from gpu_helpers import oracle_forward_rows


def test_chunked_threads_equal_one_call():
    rng = np.random.default_rng(21)
    coords = workloads.uniform_coords(rng, 20, 3000)
    x = workloads.round_to_bf16(rng.standard_normal((3000, 32), dtype=np.float32))
    w = workloads.round_to_bf16(rng.standard_normal((27, 32, 16), dtype=np.float32) * 0.05)
    b = workloads.round_to_bf16(rng.standard_normal(16, dtype=np.float32) * 0.1)
    nbr = oracle.neighbor_map(coords, (20, 20, 20))
    whole = oracle.forward(nbr, x, w, b)
    assert np.array_equal(oracle_forward_rows(oracle, nbr, x, w, b, chunk=97), whole)
    rows = np.sort(rng.choice(3000, 700, replace=False))
    assert np.array_equal(oracle_forward_rows(oracle, nbr, x, w, None, rows=rows, chunk=50),
                          oracle.forward(nbr, x, w, None, rows=rows))
