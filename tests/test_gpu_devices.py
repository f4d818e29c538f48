"""The binding runs every call on the device that holds the call's tensors.

The library launches on the current device and keeps per-device state (the
fixed scratch of dspark_draft_sample_static), so a call whose tensors sit on
another GPU than the current one must switch to that GPU, and a stream of
another device must be refused. Needs two GPUs; skipped otherwise."""
import pytest
import torch

from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl
from speculative_decoding_draft_sample_b200.spec_round import SpecRound, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture
def two_gpus(cuda_ok):
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")


def test_round_on_the_second_gpu_matches_the_first(two_gpus):
    w = wl.scaled(wl.DSPARK5, name="two_gpus", B=16, K=3, V=4096)
    inp = wl.generate(w)
    outs = []
    for dev in ("cuda:0", "cuda:1"):
        torch.cuda.set_device(0)  # cuda:0 stays current for both rounds
        d = to_device(inp, device=dev)
        rnd = SpecRound(w.B, w.K, w.V, w.r, torch.bfloat16, device=dev)
        rnd.run(d, wl.PHILOX_SEED, 0)
        torch.cuda.synchronize(dev)
        assert rnd.status() == (0, -1)
        outs.append((rnd.x.cpu(), rnd.out.cpu(), rnd.d.cpu()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    # the fixed-scratch entry point uses the scratch of the tensors' device
    torch.cuda.set_device(0)
    d1 = to_device(inp, device="cuda:1")
    x = torch.empty((w.B, w.K), dtype=torch.int32, device="cuda:1")
    dd = torch.empty((w.B, w.K, w.V), dtype=torch.bfloat16, device="cuda:1")
    q = torch.empty((w.B, w.K), device="cuda:1")
    q2 = torch.empty((w.B, w.K), device="cuda:1")
    bn.draft_sample_static(d1["base"], d1["U"], d1["W"], d1["bias_scale"], d1["last_tok"],
                           d1["temp"], wl.PHILOX_SEED, 0, x, dd, q, q2)
    torch.cuda.synchronize("cuda:1")
    assert torch.equal(x.cpu(), outs[0][0])


def test_stream_of_another_device_is_refused(two_gpus):
    w = wl.scaled(wl.DSPARK5, name="two_gpus_stream", B=8, K=2, V=1024)
    d = to_device(wl.generate(w), device="cuda:1")
    rnd = SpecRound(w.B, w.K, w.V, w.r, torch.bfloat16, device="cuda:1")
    s0 = torch.cuda.Stream(device="cuda:0")
    with pytest.raises(bn.DSparkError, match="stream is on cuda:0"):
        rnd.run(d, wl.PHILOX_SEED, 0, stream=s0)
