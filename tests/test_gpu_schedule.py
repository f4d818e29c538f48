"""dspark_prefix_schedule against the oracle's prefix cut over batch shapes up to
the one-CTA limit (B*K <= 16384): every request's cut bit for bit (a flagged
near-tie may only flip the one decision it flags, see cut_alternatives) and the
survival products within 1e-5.

"DSpark turns speculation into a scheduler", "Confidence is a serving
primitive" (survival product, the scheduler trims under load); "DSpark LLM
inference speedup", "The Real Innovation" (early stopping)."""
import numpy as np
import pytest
import torch

from oracle import dspark as o
from speculative_decoding_draft_sample_b200 import binding as bn

pytestmark = pytest.mark.gpu

SHAPES = [(1, 1), (3, 5), (7, 64), (256, 5), (1000, 8), (1024, 8), (2048, 8), (16384, 1), (4096, 4),
          (129, 3)]


def _case(B, K, kind, seed):
    rng = np.random.default_rng([seed, B, K])
    z = rng.normal(0.8, 1.6, (B, K)).astype(np.float32)
    T = np.linspace(1.0, 1.6, K).astype(np.float32)
    n = B * (K + 1)
    m = np.arange(1, n + 1, dtype=np.float64)
    if kind == "flat":
        cost = np.ones(n, np.float32)
    elif kind == "step":
        cost = np.where(m <= max(B, int(1.6 * B)), 1.0, 1.5).astype(np.float32)
    else:
        cost = (0.5 + m / n).astype(np.float32)
    return z, T, cost, float(B)


@pytest.mark.parametrize("B,K", SHAPES)
@pytest.mark.parametrize("kind", ["flat", "step", "linear"])
def test_schedule_matches_oracle(cuda_ok, B, K, kind):
    z, T, cost, fixed = _case(B, K, kind, 0)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    cut = torch.empty(B, dtype=torch.int32, device="cuda")
    surv = torch.empty((B, K), device="cuda")
    ws = torch.zeros(bn.workspace_bytes(bn.OP_SCHEDULE, B, K, 8, 1, bn.F32), dtype=torch.uint8,
                     device="cuda")
    bn.prefix_schedule(dev(z), dev(T), dev(cost), fixed, bn.CUT_COST, 0.0, cut, surv, ws)
    assert bn.read_status(ws) == (0, -1)
    _, S = o.survival(z.astype(np.float64), T.astype(np.float64))
    L, flag = o.prefix_cut(S, cost.astype(np.float64), fixed)
    g = cut.cpu().numpy().astype(np.int64)
    if flag:
        L, _ = o.adopt_cut(L, o.cut_alternatives(S, cost.astype(np.float64), fixed), g)
    assert np.array_equal(g, L), (int((g != L).sum()), int(g.sum()), int(L.sum()))
    np.testing.assert_allclose(surv.cpu().numpy(), S, rtol=1e-5, atol=0.0)
    # a second call on the same workspace gives the same cut
    bn.prefix_schedule(dev(z), dev(T), dev(cost), fixed, bn.CUT_COST, 0.0, cut, surv, ws)
    assert np.array_equal(cut.cpu().numpy(), g)
