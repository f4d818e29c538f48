"""dspark_draft_sample_beside: the one-launch draft leaving SMs to other streams.

The number of SMs left free changes only the grid (how many vocabulary tiles
each CTA streams), never the arithmetic of a tile or the order of a row's
chunks, so every output must equal dspark_draft_sample's (Markov head) or
dspark_draft_sample_recurrent's (recurrent head) bit for bit, for every count
from 0 to more than the GPU has (clamped so each group of 128 requests keeps
one SM). The shape has three groups of requests and 300 vocabulary tiles, so
the counts below give 1 to 300 tiles per CTA and a ragged last tile."""
import pytest
import torch

from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import workloads as wl
from speculative_decoding_draft_sample_b200.spec_round import to_device

pytestmark = pytest.mark.gpu

SEED = 4242
W = wl.scaled(wl.DSPARK5, name="beside", B=300, K=3, V=76800 - 40)
FREE = (0, 2, 20, 61, 140, 10000)


def _outputs(w, with_h):
    dev = "cuda"
    B, K, V, r = w.B, w.K, w.V, w.r
    o = dict(x=torch.empty((B, K), dtype=torch.int32, device=dev),
             d=torch.empty((B, K, V), dtype=torch.bfloat16, device=dev),
             q_lse=torch.empty((B, K), dtype=torch.float32, device=dev),
             q_tok=torch.empty((B, K), dtype=torch.float32, device=dev),
             q_norm=torch.empty((B, K, 2), dtype=torch.float32, device=dev))
    o["h"] = torch.empty((B, K, r), dtype=torch.bfloat16, device=dev) if with_h else None
    nbytes = bn.workspace_bytes(bn.OP_DRAFT, B, K, V, r, bn.BF16)
    o["ws"] = torch.zeros((nbytes,), dtype=torch.uint8, device=dev)
    return o


@pytest.mark.parametrize("head", ["markov", "recurrent"])
def test_beside_matches_the_full_width_draft(cuda_ok, head):
    w = W
    inp = wl.generate(w)
    dev = to_device(inp)
    R = wl.recurrent_factor(w, 1.0).to("cuda") if head == "recurrent" else None
    ref = _outputs(w, R is not None)
    if R is None:
        bn.draft_sample(dev["base"], dev["U"], dev["W"], dev["bias_scale"], dev["last_tok"],
                        dev["temp"], SEED, 3, ref["x"], ref["d"], ref["q_lse"], ref["q_tok"],
                        ref["ws"], q_norm=ref["q_norm"])
    else:
        bn.draft_sample_recurrent(dev["base"], dev["U"], dev["W"], R, dev["bias_scale"],
                                  dev["last_tok"], dev["temp"], SEED, 3, ref["x"], ref["d"],
                                  ref["q_lse"], ref["q_tok"], ref["h"], ref["ws"],
                                  q_norm=ref["q_norm"])
    torch.cuda.synchronize()
    assert bn.read_status(ref["ws"]) == (0, -1)
    for free in FREE:
        got = _outputs(w, R is not None)
        bn.draft_sample_beside(dev["base"], dev["U"], dev["W"], R, dev["bias_scale"],
                               dev["last_tok"], dev["temp"], SEED, 3, got["x"], got["d"],
                               got["q_lse"], got["q_tok"], got["h"], free, got["ws"],
                               q_norm=got["q_norm"])
        torch.cuda.synchronize()
        assert bn.read_status(got["ws"]) == (0, -1), free
        for k in ("x", "d", "q_lse", "q_tok", "q_norm") + (("h",) if R is not None else ()):
            assert torch.equal(got[k], ref[k]), (free, k)


def test_negative_free_count_is_an_argument_error(cuda_ok):
    w = wl.scaled(wl.DSPARK5, name="beside_neg", B=8, K=2, V=4096)
    dev = to_device(wl.generate(w))
    o = _outputs(w, False)
    with pytest.raises(bn.DSparkError):
        bn.draft_sample_beside(dev["base"], dev["U"], dev["W"], None, dev["bias_scale"],
                               dev["last_tok"], dev["temp"], SEED, 0, o["x"], o["d"], o["q_lse"],
                               o["q_tok"], None, -1, o["ws"], q_norm=o["q_norm"])
