"""Sequential Temperature Scaling and ECE on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import calibration as cal
from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _gpu_fit(z, y):
    N, K = z.shape
    zt = torch.from_numpy(z).cuda()
    yt = torch.from_numpy(y).cuda()
    T = torch.zeros(K, dtype=torch.float32, device="cuda")
    idx = torch.full((K,), -1, dtype=torch.int32, device="cuda")
    eb = torch.zeros(K, dtype=torch.float32, device="cuda")
    ea = torch.zeros(K, dtype=torch.float32, device="cuda")
    ws = torch.zeros(bn.workspace_bytes(bn.OP_CALIB, N, K, 0, 0, 0), dtype=torch.uint8, device="cuda")
    bn.sts_fit(zt, yt, T, idx, eb, ea, ws)
    torch.cuda.synchronize()
    assert bn.read_status(ws) == (0, -1)
    return T.cpu().numpy(), idx.cpu().numpy(), eb.cpu().numpy(), ea.cpu().numpy()


@pytest.mark.parametrize("N,K", [(300, 5), (20000, 5), (65536, 3), (7, 1)])
def test_sts_fit_matches_oracle(cuda_ok, N, K):
    z, y = wl.calib_inputs(N, K=K, seed=N)
    r = cal.sts_fit(z, y)
    T, idx, eb, ea = _gpu_fit(z, y)
    # the grid index is exact unless the oracle flags a near-tie of losses
    ok = (idx == r["index"]) | r["tie"]
    assert ok.all(), (idx, r["index"])
    grid = cal.temperature_grid()
    np.testing.assert_allclose(T, grid[idx].astype(np.float32), rtol=1e-6)
    # the ECE of a position depends on the fitted temperatures up to it: compare
    # where the fit agrees (all positions unless a flagged tie went the other way)
    np.testing.assert_allclose(eb, r["ece_before"], atol=2e-6, rtol=1e-5)
    agree = np.cumprod(idx == r["index"]).astype(bool)
    np.testing.assert_allclose(ea[agree], r["ece_after"][agree], atol=2e-6, rtol=1e-5)


def test_sts_reduces_the_calibration_error(cuda_ok):
    z, y = wl.calib_inputs(65536, K=5, seed=3)
    T, idx, eb, ea = _gpu_fit(z, y)
    assert np.all(ea < 0.02) and np.all(ea < eb) and eb.max() > 0.03
    np.testing.assert_allclose(T, wl.CALIB_GAMMAS, rtol=0.1)
