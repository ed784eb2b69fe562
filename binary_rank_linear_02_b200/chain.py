"""Decode chain: the factorised linear layers of a stack of decoder blocks, run back to
back on one stream.

A decoder runs its quantised linears one after the other (hardwired.dev, "NanoQuant
jednoduse: 70B model na herni grafice", section "Cisla": decode tokens/s of a whole
quantised model).  The pages print no model around the layers, so the wiring here is the
library's reading of a decoder's linear chain:

  * each block's input h (batch x d bfloat16, unit root-mean-square) feeds q, k, v, gate
    and up;
  * o reads bf16(v's output), down reads bf16(up's output);
  * the next block's input is bf16(down's output / rms(down's output)).

Per block this issues two libnq calls (``nq_lowrank_linear_fwd_grouped_ex``): the
five layers that read h, with v and up also writing their bf16 copies (the inputs of o
and down), then o and down, with down also writing its RMS-normalised bf16 copy (the next
block's h).  On the decode path each call is two kernels, so a block is four.  This module
only lays out buffers and passes pointers; every step runs in libnq's kernels.
"""
from __future__ import annotations

import ctypes

from . import nq

FIRST = ("q", "k", "v", "gate", "up")
SECOND = ("o", "down")
LAYERS = FIRST + SECOND


class DecodeChain:
    """blocks: one dict per block, {name: (Upk, Vpk, s1, s2, m, n, r)} for q, k, v, o,
    gate, up and down, every tensor on the same CUDA device (packed words as int32,
    scales as int16 fp16 patterns).  batch: tokens per step (1 .. 8 runs the decode path).

    After ``run``, ``h[i]`` holds block i's input (``h[0]`` the chain's input, ``h[-1]``
    its output) and ``y[name][i]`` every layer's fp32 output; ``x_o[i]`` and ``x_down[i]``
    the bf16 inputs of o and down.
    """

    def __init__(self, blocks, batch: int):
        import torch

        if not blocks:
            raise ValueError("a chain needs at least one block")
        self.batch = batch
        self.nblocks = len(blocks)
        d = blocks[0]["q"][5]
        f = blocks[0]["up"][4]
        want = {"q": (d, d), "k": (d, d), "v": (d, d), "o": (d, d), "gate": (f, d), "up": (f, d), "down": (d, f)}
        for i, w in enumerate(blocks):
            for name in LAYERS:
                if tuple(w[name][4:6]) != want[name]:
                    raise ValueError(f"block {i} layer {name}: (m, n) = {tuple(w[name][4:6])}, want {want[name]}")
        self.d, self.f = d, f
        dev = blocks[0]["q"][0].device
        nb = self.nblocks
        self.h = torch.zeros((nb + 1, batch, d), dtype=torch.int16, device=dev)
        self.y = {name: torch.empty((nb, batch, want[name][0]), dtype=torch.float32, device=dev)
                  for name in ("q", "k", "gate", "o", "down")}
        # v's and up's outputs side by side (and their bf16 copies)
        self._y_vu = torch.empty((nb, batch * (d + f)), dtype=torch.float32, device=dev)
        self._x_vu = torch.empty((nb, batch * (d + f)), dtype=torch.int16, device=dev)
        self.y["v"] = self._y_vu[:, : batch * d].view(nb, batch, d)
        self.y["up"] = self._y_vu[:, batch * d:].view(nb, batch, f)
        self.x_o = self._x_vu[:, : batch * d].view(nb, batch, d)
        self.x_down = self._x_vu[:, batch * d:].view(nb, batch, f)
        self._first, self._second = [], []
        bf16_out = {"v": self.x_o, "up": self.x_down}
        for i, w in enumerate(blocks):
            first = [(self.h[i], *w[name][:4], self.y[name][i], *w[name][4:],
                      bf16_out[name][i] if name in bf16_out else None, None) for name in FIRST]
            second = [(self.x_o[i], *w["o"][:4], self.y["o"][i], *w["o"][4:], None, None),
                      (self.x_down[i], *w["down"][:4], self.y["down"][i], *w["down"][4:], None, self.h[i + 1])]
            self._first.append(nq.make_descs_ex(first))
            self._second.append(nq.make_descs_ex(second))
        self._keep = blocks
        for name in LAYERS:
            m, n, r = blocks[0][name][4:]
            nq.workspace_reserve(m, n, r, batch)

    def packed_bytes(self) -> int:
        """Bytes of packed signs one pass of the chain reads."""
        return sum(r * (m + n) // 8 for w in self._keep for (_, _, _, _, m, n, r) in (w[k] for k in LAYERS))

    def run(self, h0=None, stream=None):
        """One decode step through every block; returns the last block's output (bf16 patterns)."""
        import torch

        if h0 is not None:
            self.h[0].copy_(h0.view(self.batch, self.d))
        s = int(stream) if stream is not None else torch.cuda.current_stream(self.h.device).cuda_stream
        L = nq.lib()
        b = self.batch
        for i in range(self.nblocks):
            nq._check(L.nq_lowrank_linear_fwd_grouped_ex(ctypes.addressof(self._first[i]), len(FIRST), b, s),
                      "nq_lowrank_linear_fwd_grouped_ex")
            nq._check(L.nq_lowrank_linear_fwd_grouped_ex(ctypes.addressof(self._second[i]), len(SECOND), b, s),
                      "nq_lowrank_linear_fwd_grouped_ex")
        return self.h[self.nblocks]

    launches_per_step_per_block = 4  # two grouped calls of two kernels each (decode path)
