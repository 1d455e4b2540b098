"""Device-side failure detection, tested without a GPU fault.

gdn_selftest_wait_timeout runs one CTA whose bounded mbarrier wait (the same
helper every wait of the chunk kernel uses) waits on a barrier nothing arrives
on: the wait gives up after the limit, the CTA records the timeout in the
status word and returns.  The host reads GDN_ERR_DEVICE_TIMEOUT from
gdn_device_status, the read clears the word, and the context keeps working.
"""
import pytest
import torch

import workloads as W
from tests import parity_utils as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import gated_deltanet_chunk_b200 as g
    g.lib()


def test_bounded_wait_expires_and_reports():
    import gated_deltanet_chunk_b200 as g
    assert g.device_status() == 0
    assert g.selftest_wait_timeout(2000) == 0          # 2 ms
    assert g.device_status() == -7                     # GDN_ERR_DEVICE_TIMEOUT
    assert g.device_status() == 0                      # the read cleared it
    # the context is still usable: a small chunked forward matches the oracle
    w = W.make_prefill(lengths=[70, 3], nqk=1, nv=2, d=128, io="bf16", init_state=True, seed=95)
    out, sf = U.run_gpu_prefill(w, 64, "tc")
    ref_o, ref_s = U.run_oracle_prefill(w)
    U.check_prefill(out, sf, ref_o, ref_s, w["cu_seqlens"], U.TOL["bf16"], "after-timeout")
    assert g.device_status() == 0
