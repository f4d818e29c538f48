"""dspark_draft_sample_static, the entry point for callers that cannot allocate
device memory (an inference server or framework whose allocator owns the
device, a plug-in host that passes only inputs and outputs, a latency-critical
path that cannot take cudaMalloc's synchronisation): it must give exactly what
dspark_draft_sample gives with a workspace, call after call, although every
call reuses the library's one fixed scratch array.

This file is collected last on purpose (if it fails, every other test has
already run), and it passes both alone in a fresh process and after the rest."""
import pytest
import torch

from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl
from speculative_decoding_draft_sample_b200.spec_round import to_device

pytestmark = pytest.mark.gpu

CASES = [
    wl.scaled(wl.DSPARK5, name="noalloc_bf16", B=64, K=3, V=16384),      # tensor-core path
    wl.scaled(wl.TINY, name="noalloc_f32", B=8, K=4, V=2048),            # fp32 CUDA-core path
]


def _outputs(w, dtype):
    i32 = dict(dtype=torch.int32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    return dict(x=torch.full((w.B, w.K), -7, **i32),
                d=torch.zeros((w.B, w.K, w.V), dtype=dtype, device="cuda"),
                q_lse=torch.zeros((w.B, w.K), **f32), q_tok=torch.zeros((w.B, w.K), **f32))


def _with_workspace(w, dev, seed, rnd_id):
    o = _outputs(w, dev["base"].dtype)
    code = bn.BF16 if w.dtype == wl.BF16 else bn.F32
    ws = torch.zeros(bn.workspace_bytes(bn.OP_DRAFT, w.B, w.K, w.V, w.r, code),
                     dtype=torch.uint8, device="cuda")
    bn.draft_sample(dev["base"], dev["U"], dev["W"], dev["bias_scale"], dev["last_tok"],
                    dev["temp"], seed, rnd_id, o["x"], o["d"], o["q_lse"], o["q_tok"], ws)
    assert bn.read_status(ws) == (0, -1)
    return o


def _static(w, dev, seed, rnd_id, status):
    o = _outputs(w, dev["base"].dtype)
    bn.draft_sample_static(dev["base"], dev["U"], dev["W"], dev["bias_scale"], dev["last_tok"],
                           dev["temp"], seed, rnd_id, o["x"], o["d"], o["q_lse"], o["q_tok"],
                           status)
    return o


def _same(a, b):
    assert torch.equal(a["x"], b["x"])
    assert torch.equal(a["d"], b["d"])
    torch.testing.assert_close(a["q_lse"], b["q_lse"], rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(a["q_tok"], b["q_tok"], rtol=1e-5, atol=0.0)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_static_scratch_matches_workspace_twice(cuda_ok, w):
    dev = to_device(wl.generate(w))
    status = torch.full((2,), 99, dtype=torch.int32, device="cuda")
    # two calls in a row on the shared array: different rounds, then the first again
    for rnd_id in (0, 1, 0):
        ref = _with_workspace(w, dev, wl.PHILOX_SEED, rnd_id)
        got = _static(w, dev, wl.PHILOX_SEED, rnd_id, status)
        torch.cuda.synchronize()
        _same(got, ref)
        assert status.tolist() == [0, -1]


def test_static_scratch_reports_and_then_clears_status(cuda_ok):
    w = CASES[0]
    dev = to_device(wl.generate(w))
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    bad = dict(dev, last_tok=dev["last_tok"].clone())
    bad["last_tok"][5] = w.V + 1
    _static(w, bad, wl.PHILOX_SEED, 0, status)
    torch.cuda.synchronize()
    assert status.tolist() == [bn.STATUS_BAD_TOKEN, 5]
    _static(w, dev, wl.PHILOX_SEED, 0, status)  # the next call starts from a clear status
    torch.cuda.synchronize()
    assert status.tolist() == [0, -1]


def test_static_scratch_size_limit(cuda_ok):
    # 256 + 8 * B * ceil(V / 256) bytes must fit in the fixed 8 MiB
    B, K, V, r = 4096, 1, 65536, 16
    base = torch.zeros((B, K, V), dtype=torch.bfloat16, device="cuda")
    U = torch.zeros((V, r), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((r, V), dtype=torch.bfloat16, device="cuda")
    o = dict(x=torch.empty((B, K), dtype=torch.int32, device="cuda"), d=torch.empty_like(base),
             q=torch.empty((B, K), device="cuda"))
    with pytest.raises(bn.DSparkError, match="workspace"):
        bn.draft_sample_static(base, U, W, None, torch.zeros(B, dtype=torch.int32, device="cuda"),
                               torch.ones(B, device="cuda"), 1, 0, o["x"], o["d"], o["q"], o["q"])
