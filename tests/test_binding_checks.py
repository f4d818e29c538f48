"""The binding checks every tensor against the sizes it passes to the library.

The C entry points see only pointers and B, K, V, r, so a tensor smaller than
those sizes imply would be read or written past its end on the device. These
checks run before anything reaches the library and need no GPU: the shapes,
dtypes and devices are checked first, the device type last.
"""
import pytest
import torch

from speculative_decoding_draft_sample_b200 import binding as bn

B, K, V, r = 4, 3, 64, 16
bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def draft_args(**over):
    a = dict(base=torch.zeros(B, K, V, dtype=bf), U=torch.zeros(V, r, dtype=bf),
             W=torch.zeros(r, V, dtype=bf), bias_scale=None, last_tok=torch.zeros(B, dtype=i32),
             temp=torch.ones(B), seed=1, round_id=0, x=torch.zeros(B, K, dtype=i32),
             d=torch.zeros(B, K, V, dtype=bf), q_lse=torch.zeros(B, K), q_tok=torch.zeros(B, K),
             ws=torch.zeros(1 << 16, dtype=torch.uint8))
    a.update(over)
    return a


def verify_args(**over):
    a = dict(target=torch.zeros(B, K + 1, V, dtype=bf), d=torch.zeros(B, K, V, dtype=bf),
             x=torch.zeros(B, K, dtype=i32), q_tok=torch.ones(B, K), cut=None, temp=torch.ones(B),
             seed=1, round_id=0, accepted=torch.zeros(B, dtype=i32),
             out=torch.zeros(B, K + 1, dtype=i32), n_emit=torch.zeros(B, dtype=i32),
             ws=torch.zeros(1 << 16, dtype=torch.uint8))
    a.update(over)
    return a


@pytest.mark.parametrize("over,msg", [
    (dict(x=torch.zeros(B, K + 1, dtype=i32)), "x must have shape"),
    (dict(d=torch.zeros(B, K, V - 8, dtype=bf)), "d must have shape"),
    (dict(U=torch.zeros(V, r + 1, dtype=bf)), "W must have shape"),  # r is taken from U
    (dict(W=torch.zeros(r, V, dtype=f32)), "W must be"),
    (dict(q_tok=torch.zeros(B * K)), "q_tok must have shape"),
    (dict(last_tok=torch.zeros(B, dtype=torch.int64)), "last_tok must be"),
    (dict(bias_scale=torch.ones(B + 1)), "bias_scale must have shape"),
    (dict(q_norm=torch.zeros(B, K)), "q_norm must have shape"),
    (dict(x=torch.zeros(K, B, dtype=i32).t()), "x must be contiguous"),  # shape (B, K), strided
    (dict(d=torch.zeros(B, V, K, dtype=bf).transpose(1, 2)), "d must be contiguous"),
    (dict(temp=torch.ones(B, device="meta")), "temp is on meta"),
    ({}, "must be CUDA tensors"),
])
def test_draft_sample_checks(over, msg):
    with pytest.raises(bn.DSparkError, match=msg):
        bn.draft_sample(**draft_args(**over))


@pytest.mark.parametrize("over,msg", [
    (dict(out=torch.zeros(B, K, dtype=i32)), "out must have shape"),
    (dict(d=torch.zeros(B, K + 1, V, dtype=bf)), "d must have shape"),
    (dict(cut=torch.zeros(B + 1, dtype=i32)), "cut must have shape"),
    (dict(accepted=torch.zeros(B, dtype=torch.int64)), "accepted must be"),
    (dict(d=torch.zeros(B, K, V, dtype=f32)), "d must be"),
    (dict(q_norm=torch.zeros(B, K, 2, dtype=torch.float64)), "q_norm must be"),
    ({}, "must be CUDA tensors"),
])
def test_verify_checks(over, msg):
    with pytest.raises(bn.DSparkError, match=msg):
        bn.verify(**verify_args(**over))


def test_pick_logits_schedule_and_calibration_checks():
    a = draft_args()
    with pytest.raises(bn.DSparkError, match="x must have shape"):
        bn.draft_pick(a["d"], a["last_tok"], a["temp"], 1, 0, 1, torch.zeros(B, dtype=i32),
                      a["q_lse"], a["q_tok"], a["ws"])
    with pytest.raises(bn.DSparkError, match="x must have shape"):
        bn.draft_logits(a["base"], a["U"], a["W"], None, a["last_tok"], torch.zeros(B, K + 2, dtype=i32),
                        a["temp"], 1, a["d"], a["ws"])
    with pytest.raises(bn.DSparkError, match="step_cost must have shape"):
        bn.prefix_schedule(torch.zeros(B, K), torch.ones(K), torch.ones(B * K), 0.0, bn.CUT_COST,
                           0.0, torch.zeros(B, dtype=i32), torch.zeros(B, K), a["ws"])
    with pytest.raises(bn.DSparkError, match="pos_temp must have shape"):
        bn.prefix_schedule(torch.zeros(B, K), torch.ones(K + 1), torch.ones(B * (K + 1)), 0.0,
                           bn.CUT_COST, 0.0, torch.zeros(B, dtype=i32), torch.zeros(B, K), a["ws"])
    with pytest.raises(bn.DSparkError, match="survived must have shape"):
        bn.sts_fit(torch.zeros(10, K), torch.zeros(10, K + 1, dtype=torch.uint8), torch.zeros(K),
                   None, None, None, a["ws"])
    with pytest.raises(bn.DSparkError, match="status_out must have shape"):
        bn.draft_sample_static(a["base"], a["U"], a["W"], None, a["last_tok"], a["temp"], 1, 0,
                               a["x"], a["d"], a["q_lse"], a["q_tok"],
                               status_out=torch.zeros(1, dtype=i32))
    with pytest.raises(bn.DSparkError, match="must be a CUDA tensor"):
        bn.read_status(a["ws"])
