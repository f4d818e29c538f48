"""One speculative round on the device: draft_sample -> prefix_schedule -> verify.

``SpecRound`` owns the round's output buffers and one workspace (PyTorch
allocations: device memory is PyTorch's job here) and issues the three C-ABI
calls on one stream. ``run_host`` is the end-to-end form: inputs in pinned host
memory are copied in, the round runs, and the emitted tokens come back.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Optional

import torch

from . import binding as bn
from . import replicas

# Most SMs a round's draft leaves to the side stream, and how much longer the
# draft may get for it (the ratio of the most vocabulary tiles per CTA to the
# most with the library's default of 2 free SMs).
MAX_FREE_SMS = 32
FREE_SMS_SLACK = 8.0 / 7.0
DEFAULT_FREE_SMS = 2


def draft_tiles_per_cta(num_sms: int, B: int, V: int, free_sms: int) -> int:
    """The most 128 x 256 (requests x vocabulary) tiles one CTA of the one-launch
    draft streams per position when free_sms SMs are left free: each group of
    128 requests gets (SMs - free) / groups CTAs, which split the vocabulary's
    256-entry tiles among them."""
    m = (B + 127) // 128
    n = (V + 255) // 256
    free = min(max(free_sms, 0), num_sms - m)
    per_m = max(1, (num_sms - free) // m)
    return -(-n // per_m)


def beside_free_sms(num_sms: int, B: int, V: int) -> int:
    """SMs a round's draft leaves to the target rows' statistics on the side
    stream: the largest count up to MAX_FREE_SMS whose most tiles per CTA stays
    within FREE_SMS_SLACK of the default's. At B = 256, V = 129280 on 148 SMs
    that is 20 (eight tiles per CTA instead of seven); for one group of requests
    over V = 151936 it is 29 (five tiles per CTA either way)."""
    limit = math.floor(draft_tiles_per_cta(num_sms, B, V, DEFAULT_FREE_SMS) * FREE_SMS_SLACK + 1e-9)
    best = DEFAULT_FREE_SMS
    for f in range(DEFAULT_FREE_SMS, MAX_FREE_SMS + 1):
        if draft_tiles_per_cta(num_sms, B, V, f) <= limit:
            best = f
    return best


class GlobalSchedule:
    """One prefix schedule over the requests of every rank, in place of one
    per engine: the confidence logits of all ranks are gathered (the only
    data-path collective), every rank runs the same schedule on the combined
    batch against the combined batch's cost table, so all ranks compute the
    same cut, and each keeps the slice of its own requests (rank r holds
    requests r * B .. r * B + B - 1 of the combined batch).

    step_cost has (B * world) * (K + 1) entries (workloads.cost_table of the
    combined batch); gather (default replicas.all_gather_rows) stacks every
    rank's [B, K] confidence logits in rank order.
    """

    def __init__(self, B: int, K: int, step_cost, fixed_cost: float, rank: int, world: int,
                 device: str = "cuda", gather: Optional[Callable] = None):
        if not 0 <= rank < world:
            raise bn.DSparkError(f"rank {rank} outside a world of {world}")
        self.B, self.K, self.rank, self.world = B, K, rank, world
        bg = B * world
        dev = torch.device(device)
        self.step_cost = torch.as_tensor(step_cost, dtype=torch.float32).to(dev).contiguous()
        if self.step_cost.numel() != bg * (K + 1):
            raise bn.DSparkError(f"step_cost needs {bg * (K + 1)} entries for {world} ranks of "
                                 f"{B} requests, got {self.step_cost.numel()}")
        self.fixed_cost = float(fixed_cost)
        self.cut = torch.empty((bg,), dtype=torch.int32, device=dev)
        self.survival = torch.empty((bg, K), dtype=torch.float32, device=dev)
        self.gather = gather if gather is not None else replicas.all_gather_rows

    def run(self, conf_logit, pos_temp, mode: int, threshold: float, cut, survival, ws,
            stream) -> None:
        """This rank's cut [B] and survival [B, K] from the combined batch's
        schedule, on `stream` (the schedule kernel's status lands in ws)."""
        with torch.cuda.stream(stream):
            conf_all = self.gather(conf_logit)
            bn.prefix_schedule(conf_all, pos_temp, self.step_cost, self.fixed_cost, mode,
                               threshold, self.cut, self.survival, ws, stream)
            lo = self.rank * self.B
            cut.copy_(self.cut[lo:lo + self.B])
            survival.copy_(self.survival[lo:lo + self.B])


class SpecRound:
    def __init__(self, B: int, K: int, V: int, r: int, dtype: torch.dtype = torch.bfloat16,
                 device: str = "cuda"):
        self.B, self.K, self.V, self.r = B, K, V, r
        self.dtype = dtype
        dev = torch.device(device)
        code = bn.F32 if dtype == torch.float32 else bn.BF16
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.x = torch.empty((B, K), **i32)
        self.d = torch.empty((B, K, V), dtype=dtype, device=dev)
        self.q_lse = torch.empty((B, K), **f32)
        self.q_tok = torch.empty((B, K), **f32)
        self.q_norm = torch.empty((B, K, 2), **f32)  # the draws' normalisers, for verify
        self.h = None  # the recurrent head's states [B, K, r], when a round uses it
        self.cut = torch.empty((B,), **i32)
        self.survival = torch.empty((B, K), **f32)
        self.accepted = torch.empty((B,), **i32)
        self.out = torch.empty((B, K + 1), **i32)
        self.n_emit = torch.empty((B,), **i32)
        nbytes = max(bn.workspace_bytes(op, B, K, V, r, code)
                     for op in (bn.OP_DRAFT, bn.OP_SCHEDULE, bn.OP_VERIFY))  # verify's holds the draft's
        if nbytes == 0:
            raise bn.DSparkError(f"unsupported round shape B={B} K={K} V={V} r={r}")
        self.ws = torch.zeros((nbytes,), dtype=torch.uint8, device=dev)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count if dev.type == "cuda" else 148
        # SMs the draft leaves to the side stream's statistics when a round has one
        self.free_sms = beside_free_sms(sms, B, V)

    def run(self, inp: Dict[str, torch.Tensor], seed: int, round_id: int,
            mode: int = bn.CUT_COST, threshold: float = 0.0, stream=None,
            side_stream=None, global_schedule: Optional[GlobalSchedule] = None) -> None:
        """Issues the round on ``stream`` (no host synchronisation).

        The prefix schedule needs only the confidence logits, and the target
        rows' statistics only the target logits and the cut, so with a
        ``side_stream`` both run there, concurrently with the draft, which then
        leaves ``self.free_sms`` SMs free for them (dspark_draft_sample_beside;
        the same results as dspark_draft_sample); the rest of verification
        waits for both. The calls share the workspace: the draft's
        partials and the statistics occupy different regions of it, and they
        meet only in its status block, which every call updates atomically.
        """
        main = stream if stream is not None else torch.cuda.current_stream(self.x.device)

        def schedule_and_stats(s):
            if global_schedule is not None:  # one cut over every rank's requests
                global_schedule.run(inp["conf_logit"], inp["pos_temp"], mode, threshold, self.cut,
                                    self.survival, self.ws, s)
            else:
                bn.prefix_schedule(inp["conf_logit"], inp["pos_temp"], inp["step_cost"],
                                   float(inp["fixed_cost"]), mode, threshold, self.cut,
                                   self.survival, self.ws, s)
            bn.verify_target_stats(inp["target"], self.cut, inp["temp"], self.ws, s)

        if side_stream is not None:
            if side_stream.device != self.x.device or main.device != self.x.device:
                raise bn.DSparkError(f"the round's streams must be on {self.x.device}")
            fork, join = torch.cuda.Event(), torch.cuda.Event()
            fork.record(main)
            side_stream.wait_event(fork)
            schedule_and_stats(side_stream)
            join.record(side_stream)
        R = inp.get("R")
        if R is not None and self.h is None:  # the recurrent head; its states land in self.h
            self.h = torch.empty((self.B, self.K, self.r), dtype=self.dtype, device=self.x.device)
        if side_stream is not None:
            bn.draft_sample_beside(inp["base"], inp["U"], inp["W"], R, inp.get("bias_scale"),
                                   inp["last_tok"], inp["temp"], seed, round_id, self.x, self.d,
                                   self.q_lse, self.q_tok, self.h, self.free_sms, self.ws, main,
                                   q_norm=self.q_norm)
        elif R is not None:
            bn.draft_sample_recurrent(inp["base"], inp["U"], inp["W"], R,
                                      inp.get("bias_scale"), inp["last_tok"], inp["temp"], seed,
                                      round_id, self.x, self.d, self.q_lse, self.q_tok, self.h,
                                      self.ws, main, q_norm=self.q_norm)
        else:
            bn.draft_sample(inp["base"], inp["U"], inp["W"], inp.get("bias_scale"), inp["last_tok"],
                            inp["temp"], seed, round_id, self.x, self.d, self.q_lse, self.q_tok,
                            self.ws, main, q_norm=self.q_norm)
        if side_stream is None:
            schedule_and_stats(main)
        else:
            main.wait_event(join)
        bn.verify_from_stats(inp["target"], self.d, self.x, self.q_tok, self.cut, inp["temp"],
                             seed, round_id, self.accepted, self.out, self.n_emit, self.ws, main,
                             q_norm=self.q_norm)

    def status(self, stream=None):
        return bn.read_status(self.ws, stream)


DEVICE_KEYS = ("base", "target", "U", "W", "bias_scale", "last_tok", "temp", "conf_logit",
               "pos_temp", "step_cost")
OPTIONAL_KEYS = ("R",)  # the recurrent head's state matrix


def to_device(inp: Dict[str, object], device: str = "cuda", pin: bool = False) -> Dict[str, object]:
    """Device (or pinned host) copies of a workload's tensors (numpy arrays become tensors)."""
    out: Dict[str, object] = {}
    for k in DEVICE_KEYS:
        v = inp[k]
        t = v if isinstance(v, torch.Tensor) else torch.from_numpy(v)
        if k == "last_tok":
            t = t.to(torch.int32)
        elif t.dtype == torch.float64:
            t = t.float()
        t = t.contiguous()
        out[k] = t.pin_memory() if pin else t.to(device, non_blocking=False)
    for k in OPTIONAL_KEYS:
        v = inp.get(k)
        if v is not None:
            t = v if isinstance(v, torch.Tensor) else torch.from_numpy(v)
            out[k] = t.contiguous().pin_memory() if pin else t.contiguous().to(device)
    out["fixed_cost"] = float(inp["fixed_cost"])
    return out


def run_host(rnd: SpecRound, host: Dict[str, object], dev: Dict[str, object], seed: int,
             round_id: int, out_host: torch.Tensor, n_emit_host: torch.Tensor,
             mode: int = bn.CUT_COST, stream=None, side_stream=None,
             threshold: float = 0.0, global_schedule: Optional[GlobalSchedule] = None) -> None:
    """End to end from pinned host buffers: H2D copies, the round, D2H of the tokens."""
    for k in DEVICE_KEYS:
        dev[k].copy_(host[k], non_blocking=True)
    rnd.run(dev, seed, round_id, mode, threshold, stream=stream, side_stream=side_stream,
            global_schedule=global_schedule)
    out_host.copy_(rnd.out, non_blocking=True)
    n_emit_host.copy_(rnd.n_emit, non_blocking=True)
