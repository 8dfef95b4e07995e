"""Failure detection on the GPU without a GPU fault.

Every wait of the decode kernel's pipeline roles is bounded.  Here the bound
is made tiny (mla_set_wait_limit_ns), so waits run out on purpose: the kernel
must set MLA_STATUS_TIMEOUT, stop both CTAs of each cluster, wait for the
copies and tensor-core products it already issued (under the default bound),
free its tensor memory and return.  The context must stay usable: the next
call with the default bound matches the oracle."""
import pytest
import torch

from head_latent_attention_04_b200 import workloads as W
from tests.gpu_helpers import check_out, oracle_all, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lens,s_q,clusters", [([3000, 1000, 77], 1, 4), ([256, 256], 1, 74),
                                               ([2000, 70, 600], 2, 6)])
def test_wait_time_out_returns_and_the_context_recovers(lens, s_q, clusters):
    from head_latent_attention_04_b200 import mla
    w = W.make_workload(len(lens), s_q, 128, lens, seed=66 + s_q, pool="permuted")
    try:
        mla.set_wait_limit_ns(1)
        for _ in range(2):
            dec, res = run_gpu(w, num_clusters=clusters)       # returns: the kernel gives up instead of hanging
            assert res.status.item() & mla.STATUS_TIMEOUT
    finally:
        mla.set_wait_limit_ns(0)
    dec, res = run_gpu(w, num_clusters=clusters)
    assert res.status.item() == 0
    check_out(res.out, oracle_all(w)["out"])
