"""Failure detection on the GPU without a fault: the library's bounded waits,
made to run out on purpose (an mbarrier phase nobody completes, a grid barrier
one CTA reaches alone), give up after their limit, report
DSPARK_STATUS_TIMEOUT with the site and the request, and leave the context
usable for the next round."""
import time

import pytest
import torch

from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl
from speculative_decoding_draft_sample_b200.spec_round import SpecRound, to_device

pytestmark = pytest.mark.gpu

SITE_SELFTEST = 30  # wait site the self-test records


def test_bounded_waits_give_up_and_the_context_stays_usable(cuda_ok):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    res = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    bn.selftest_waits(res, ws)  # two waits that run out after the kernels' 2 s limit
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert res.tolist() == [1, 1]  # both waits gave up
    assert 3.9 <= elapsed < 30.0
    assert int(ws[8:12].view(torch.int32).item()) == SITE_SELFTEST  # first site that gave up
    code, first = bn.read_status(ws)
    assert code == bn.STATUS_TIMEOUT and first == 0
    # the context is intact: a round right after runs clean
    w = wl.scaled(wl.DSPARK5, name="after_timeout", B=8, V=2048)
    dev = to_device(wl.generate(w))
    rnd = SpecRound(w.B, w.K, w.V, w.r)
    rnd.run(dev, wl.PHILOX_SEED, 0)
    torch.cuda.synchronize()
    assert rnd.status() == (0, -1)
    assert int(rnd.n_emit.min().item()) >= 1


def test_selftest_argument_checks(cuda_ok):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    res = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(bn.DSparkError, match="invalid argument"):
        bn.selftest_waits(res, ws[:128])
    with pytest.raises(bn.DSparkError, match="result must have shape"):
        bn.selftest_waits(res[:1], ws)
