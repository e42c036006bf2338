"""Device status path: a bounded wait that gives up is reported by carve_check as
CARVE_ERR_TIMEOUT (then cleared), and the CUDA context stays usable afterwards."""
import pytest

import chunk_gated_delta_b200 as carve
import oracle
from chunk_gated_delta_b200 import inputs as I
from tests.helpers import TOL, host, rel_l2, to_dev

pytestmark = pytest.mark.gpu


def _tiny_fwd(dev):
    w = I.TINY_FP32
    d = I.make_inputs(w)
    dd = to_dev(d, w.io, dev)
    out = carve.carve_fwd(dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"],
                          chunk=w.L, save_for_bwd=False)
    return host(out["o"]), oracle.fwd(d, L=w.L)["o"]


def test_clean_run_reports_ok(cuda_device):
    got, want = _tiny_fwd(cuda_device)
    assert carve.carve_check() == 0
    assert rel_l2(got, want) <= TOL["fp32"]


def test_expired_wait_is_reported_and_context_survives(cuda_device):
    lib = carve.load()
    assert carve.carve_check() == 0
    assert lib.carve_selftest_timeout(1000, None) == 0
    assert carve.carve_check() == 4            # CARVE_ERR_TIMEOUT
    assert carve.carve_check() == 0            # the status word was cleared
    got, want = _tiny_fwd(cuda_device)         # and the context still computes correctly
    assert carve.carve_check() == 0
    assert rel_l2(got, want) <= TOL["fp32"]
