"""Calls with at least 2048 key blocks run their CTAs in clusters of two that split the proxy
scoring's reads of the pooled keys (each CTA scores half the key blocks for its own tiles and its
partner's, storing the partner's scores into the partner's shared memory).  Two edge cases of
that sharing, against the oracle:
  - an odd number of CTAs (1025 tile pairs plus the split of the last wave): the grid gets one
    extra CTA with no work unit, which only scores its partner's tiles;
  - clusters across a head boundary (1025 tile pairs per head): such a pair shares nothing and
    each CTA scores its own tiles over every key block; the partial last key block as well."""
import numpy as np
import pytest

from free_sparse_attention_block_b200 import inputs
from parity import check_parity, default_units, gpu_run

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("BH,N,beta", [(1, 64 * 2050, 1.5), (3, 64 * 2049 + 5, 1.0)])
def test_clustered_routing_against_oracle(BH, N, beta):
    q, k, v = inputs.small_workload(N, BH=BH, seed=BH + 40, f_max=4.0)
    Nq = (N + 63) // 64
    units = default_units(BH, Nq, per_head=10, seed=BH)
    if BH > 1:   # tiles around each head boundary: the last pair of a head and the first of the next
        extra = [bh * Nq + i for bh in range(BH) for i in (0, 1, Nq - 2, Nq - 1)]
        units = np.unique(np.concatenate([units, np.asarray(extra, np.int64)]))
    g = gpu_run(q, k, v, beta, units=units, with_proxy=True)
    rep = {}
    check_parity(q, k, v, beta, g, units, report=rep)
    print(f"BH={BH} N={N} beta={beta}: {rep}")
