"""Batched decode with multi-level padding over a pool of per-request states.

Section 3 of "MiniMax-01技術報告解讀以及與DeepSeek-V3對比" (m.futurefh.com)
lists, among the inference optimisations, separate prefill and decode and
padding in several levels so that little work is spent on padding.  Here a
decode step serves n live requests, each owning one slot of a state pool.
The batch is padded up to the smallest of a few fixed sizes (the levels);
padding rows carry slot -1, which the kernels treat as "no work": zero output
and no state traffic (``la_decode_step_slots`` / ``la_decode_step_q8``).  The
step of each level is captured once as a CUDA graph and replayed, so the host
cost of a step is a few small copies and one graph launch whatever n is.

The state pool is either fp32 (``[num_slots, H, d, d]``) or the 8-bit form
(int8 codes ``[num_slots, H, d, d]`` plus fp32 scales ``[num_slots, H, d]``)
that the yuliangy.com digest's 8-bit quantisation is read as.

Only argument marshalling and bookkeeping live here; the step itself is one
launch of the library's decode kernel.
"""
from __future__ import annotations

from typing import Iterable, Sequence

import linear_attention_13_b200 as la

DEFAULT_LEVELS = (1, 2, 4, 8, 16, 32, 64, 128, 256)


def pick_level(n: int, levels: Sequence[int] = DEFAULT_LEVELS) -> int:
    """Smallest level >= n (n >= 1).  Raises ValueError when n exceeds them all."""
    if n < 1:
        raise ValueError("a decode batch needs at least one live row")
    for lv in sorted(levels):
        if lv >= n:
            return int(lv)
    raise ValueError(f"batch of {n} rows exceeds the largest padding level {max(levels)}")


def padded_slots(slots: Iterable[int], level: int, num_slots: int) -> list:
    """The live slots followed by -1 up to ``level`` entries.

    Checks what the kernels cannot: every slot in [0, num_slots) and no slot
    twice (two rows updating one state in the same step would race)."""
    live = [int(s) for s in slots]
    if len(live) > level:
        raise ValueError("more live rows than the padding level")
    if any(s < 0 or s >= num_slots for s in live):
        raise ValueError("slot id out of range")
    if len(set(live)) != len(live):
        raise ValueError("a slot may appear once per step")
    return live + [-1] * (level - len(live))


def validate_levels(levels: Sequence[int]) -> tuple:
    lv = tuple(sorted(int(x) for x in levels))
    if not lv or lv[0] < 1 or len(set(lv)) != len(lv):
        raise ValueError("levels must be distinct positive sizes")
    return lv


class PaddedDecoder:
    """Decode steps for up to ``max(levels)`` live requests over ``num_slots`` states.

    ``state`` is "fp32" or "q8".  ``step(q, k, v, slots)`` takes [n, H, d]
    CUDA tensors and a host list of n distinct slots and returns the [n, H, d]
    output, a view into the level's output buffer that stays valid until the
    next step at the same level.
    """

    def __init__(self, num_slots: int, H: int, d: int, dtype=None, state: str = "fp32",
                 levels: Sequence[int] = DEFAULT_LEVELS, device="cuda", use_graphs: bool = True):
        import torch
        if state not in ("fp32", "q8"):
            raise ValueError("state must be 'fp32' or 'q8'")
        self.torch = torch
        self.num_slots, self.H, self.d = int(num_slots), int(H), int(d)
        self.dtype = dtype if dtype is not None else torch.bfloat16
        self.state_kind = state
        self.levels = validate_levels(levels)
        self.device = torch.device(device)
        self.use_graphs = use_graphs
        if state == "fp32":
            self.pool = torch.zeros((num_slots, H, d, d), dtype=torch.float32, device=self.device)
        else:
            self.codes = torch.zeros((num_slots, H, d, d), dtype=torch.int8, device=self.device)
            self.scales = torch.zeros((num_slots, H, d), dtype=torch.float32, device=self.device)
        self._bufs = {}
        self._graphs = {}

    # ------------------------------------------------------------ state slots
    def load_state(self, slot: int, state_fp32) -> None:
        """Set a slot from an fp32 state [H, d, d] (e.g. a prefill's final state)."""
        if self.state_kind == "fp32":
            self.pool[slot].copy_(state_fp32)
        else:
            la.state_quantize_q8(state_fp32.contiguous(), codes=self.codes[slot], scales=self.scales[slot])

    def read_state(self, slot: int):
        """A slot's state as fp32 [H, d, d] (dequantised for the 8-bit pool)."""
        if self.state_kind == "fp32":
            return self.pool[slot].clone()
        return la.state_dequantize_q8(self.codes[slot], self.scales[slot])

    def reset(self, slot: int) -> None:
        if self.state_kind == "fp32":
            self.pool[slot].zero_()
        else:
            self.codes[slot].zero_()
            self.scales[slot].zero_()

    # ------------------------------------------------------------ one step
    def _buffers(self, level: int):
        b = self._bufs.get(level)
        if b is None:
            torch = self.torch
            shape = (level, self.H, self.d)
            b = {name: torch.zeros(shape, dtype=self.dtype, device=self.device)
                 for name in ("q", "k", "v", "o")}
            b["slots"] = torch.full((level,), -1, dtype=torch.int32, device=self.device)
            b["slots_host"] = torch.full((level,), -1, dtype=torch.int32).pin_memory()
            # the asynchronous upload of slots_host must have run before the host
            # overwrites it for the next step of this level
            b["uploaded"] = torch.cuda.Event()
            b["pending"] = False
            self._bufs[level] = b
        return b

    def _launch(self, b) -> None:
        if self.state_kind == "fp32":
            la.decode_step_slots(b["q"], b["k"], b["v"], self.pool, b["slots"], out=b["o"])
        else:
            la.decode_step_q8(b["q"], b["k"], b["v"], self.codes, self.scales, b["slots"], out=b["o"])

    def _graph(self, level: int, b):
        g = self._graphs.get(level)
        if g is None:
            torch = self.torch
            # capture with every row padding: the capture run touches no state
            saved = b["slots"].clone()
            b["slots"].fill_(-1)
            side = torch.cuda.Stream(device=self.device)
            side.wait_stream(torch.cuda.current_stream(self.device))
            with torch.cuda.stream(side):
                self._launch(b)                      # warm-up outside the graph
            torch.cuda.current_stream(self.device).wait_stream(side)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._launch(b)
            b["slots"].copy_(saved)
            self._graphs[level] = g
        return g

    def captured_levels(self) -> tuple:
        return tuple(sorted(self._graphs))

    def step(self, q, k, v, slots: Sequence[int]):
        n = len(slots)
        if q.shape != (n, self.H, self.d) or k.shape != q.shape or v.shape != q.shape:
            raise ValueError("q, k, v must be [len(slots), H, d]")
        level = pick_level(n, self.levels)
        padded = padded_slots(slots, level, self.num_slots)
        b = self._buffers(level)
        b["q"][:n].copy_(q)
        b["k"][:n].copy_(k)
        b["v"][:n].copy_(v)
        if b["pending"]:
            b["uploaded"].synchronize()
        b["slots_host"].copy_(self.torch.tensor(padded, dtype=self.torch.int32))
        b["slots"].copy_(b["slots_host"], non_blocking=True)
        b["uploaded"].record()
        b["pending"] = True
        if self.use_graphs:
            self._graph(level, b).replay()
        else:
            self._launch(b)
        return b["o"][:n]
