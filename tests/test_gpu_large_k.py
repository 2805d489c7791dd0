"""Very large k (above the 4096 keys the shared-memory final top-k holds): the
global-memory final stage, bit-exact against the oracle, with padding, with
many equal scores, and with a cut bin too large to keep aside."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
from gpu_util import assert_parity, run_gpu, run_oracle
from workloads import small

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("k", [4097, 20000, 70000])
def test_large_k_matches_oracle(k):
    # masks that require nothing but two flags: about 80% of 100k items eligible
    data = small(n=100000, d=32, nlist=8, sig_bits=64, B=3, nprobe=8, k=k, seed=61, mask_flags=2,
                 mask_lang=False)
    assert_parity(run_gpu(data, 8, k), run_oracle(data, 8, k), f"k={k}")


def test_large_k_more_than_eligible_pads():
    data = small(n=30000, d=32, nlist=8, sig_bits=64, B=2, nprobe=4, k=50000, seed=62)
    got = run_gpu(data, 4, 50000)
    assert_parity(got, run_oracle(data, 4, 50000), "padding")
    assert (got[0][:, -1] == -1).all()


def test_large_k_identical_items():
    # every score equal: one long segment, ordered by id alone
    data = small(n=20000, d=16, nlist=2, sig_bits=64, B=2, nprobe=2, k=12000, seed=63, mask_flags=0,
                 mask_lang=False)
    data.items[:] = 3
    assert_parity(run_gpu(data, 2, 12000), run_oracle(data, 2, 12000), "identical")
