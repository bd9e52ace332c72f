"""Run one of the five workloads through the C ABI exactly as a caller would.

One ``step()`` is the whole workload once from a zero state: for the
single-block configurations one ``la_full_forward``; for the streaming
configurations ``la_state_init`` and then ``la_block_forward`` for every
block and every denoising pass (the last pass of a block commits).  Inputs
for every call are drawn once on the device and stay resident in HBM; every
call writes its own output buffer.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import torch

from . import la, synth


class Runner:
    def __init__(self, w: synth.Workload, device="cuda", blocks: Optional[int] = None, e4m3: bool = False,
                 nvfp4: bool = False):
        self.w = w
        self.e4m3 = e4m3
        self.nvfp4 = nvfp4
        if e4m3 and nvfp4:
            raise ValueError("one input format")
        self.device = torch.device(device)
        self.calls: List[tuple] = []          # (block, pass, q, k, v) in call order
        if w.mode == "full":
            q, k, v = synth.full_sequence(w, device=self.device)
            self.calls.append((0, 0, q, k, v))
            L = 0 if w.n_blocks == 1 else w.n_blk
            self.ws = la.alloc_workspace(w.B, w.n_total, w.H, w.d, L, device=self.device)
            self.tokens_per_block = L
        else:
            for c in synth.stream(w, device=self.device, blocks=blocks):
                self.calls.append(c)
            self.ws = la.alloc_workspace(w.B, w.n_blk, w.H, w.d, w.n_blk, device=self.device)
            self.tokens_per_block = w.n_blk
        self.outs = [torch.empty_like(c[2]) for c in self.calls]
        self.scales = None
        if e4m3:
            # FP8 inputs: each call's q, k, v as E4M3 codes with per-tensor scales
            self.scales = []
            for i, c in enumerate(self.calls):
                qk = [synth.to_e4m3(t) for t in c[2:5]]
                self.calls[i] = (c[0], c[1], *[x for x, _ in qk])
                self.scales.append([s_ for _, s_ in qk])
        self.fp4 = None
        if nvfp4:
            # NVFP4 inputs: each call's q, k, v as (E2M1 codes, E4M3 block scales, per-tensor scale)
            self.fp4 = []
            for i, c in enumerate(self.calls):
                self.fp4.append([synth.to_nvfp4(t) for t in c[2:5]])
                self.calls[i] = (c[0], c[1], *[x[0] for x in self.fp4[-1]])
        self.inputs = [c[2:5] for c in self.calls]        # device inputs of each call
        if nvfp4:
            self.inputs = [tuple(x[0] for x in f) + tuple(x[1] for x in f) for f in self.fp4]
        self.out_call = list(range(len(self.calls)))      # the call that writes each out
        self.state = la.State(w.B, w.H, w.d, device=self.device) if w.mode == "stream" else None
        self.rope = None
        if w.rope:
            # t_offset < 0: each streaming call takes its frames from the state's t_next
            self.rope = la.make_rope(Hg=w.Hg, Wg=w.Wg, T=w.frames,
                                     t_offset=-1 if w.mode == "stream" else 0,
                                     dims=w.rope_dims, base=w.rope_base)

    @property
    def launches_per_step(self) -> int:
        return self._launches

    def step(self, after_call: Optional[Callable[[int], None]] = None, stream=None) -> None:
        w = self.w
        n = 0
        if w.mode == "full":
            _, _, q, k, v = self.calls[0]
            if self.nvfp4:
                la.full_forward_nvfp4(*self.fp4[0], self.tokens_per_block, eps=w.eps, ws=self.ws,
                                      out=self.outs[0], stream=stream, rope=self.rope)
            elif self.e4m3:
                la.full_forward_e4m3(q, k, v, self.scales[0], self.tokens_per_block, eps=w.eps, ws=self.ws,
                                     out=self.outs[0], stream=stream, rope=self.rope)
            else:
                la.full_forward(q, k, v, self.tokens_per_block, rope=self.rope, eps=w.eps, ws=self.ws,
                                out=self.outs[0], stream=stream)
            n += la.la_last_launch_count()
            if after_call:
                after_call(0)
        else:
            st = self.state
            rc = la.la_state_init(st.c, st.S.data_ptr(), st.Z.data_ptr(), w.B, w.H, w.d,
                                  la._stream_ptr(stream))
            if rc != la.LA_OK:
                raise la.LAError(rc, "la_state_init")
            for i, (blk, p, q, k, v) in enumerate(self.calls):
                if self.nvfp4:
                    la.block_forward_nvfp4(*self.fp4[i], st, commit=(p == w.passes - 1), eps=w.eps,
                                           ws=self.ws, out=self.outs[i], stream=stream, rope=self.rope)
                elif self.e4m3:
                    la.block_forward_e4m3(q, k, v, self.scales[i], st, commit=(p == w.passes - 1), eps=w.eps,
                                          ws=self.ws, out=self.outs[i], stream=stream, rope=self.rope)
                else:
                    la.block_forward(q, k, v, st, commit=(p == w.passes - 1), rope=self.rope, eps=w.eps,
                                     ws=self.ws, out=self.outs[i], stream=stream)
                n += la.la_last_launch_count()
                if after_call:
                    after_call(i)
        self._launches = n

    def tokens_per_call(self, i: int) -> int:
        return self.calls[i][2].shape[1]


def host_heads(t: torch.Tensor, heads: Sequence[int]) -> torch.Tensor:
    """Copy the listed heads of a [B, N, H, d] device tensor to the host."""
    idx = torch.as_tensor(list(heads), device=t.device)
    return t.index_select(2, idx).contiguous().cpu()


class BackwardRunner:
    """One training backward pass (``la_full_backward``) over a workload's
    whole sequence: its blocks concatenated (one pass per block), the same
    block length and RoPE, a seeded upstream gradient dout; writes dq, dk, dv.
    The same interface as Runner for the benchmark."""

    def __init__(self, w: synth.Workload, device="cuda"):
        self.w = w.shrink(passes=1)
        w = self.w
        self.device = torch.device(device)
        q, k, v = synth.full_sequence(w, device=self.device)
        dout = synth.upstream_grad(w, device=self.device)
        self.calls = [(0, 0, q, k, v)]
        self.inputs = [(q, k, v, dout)]
        self.outs = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
        self.out_call = [0, 0, 0]
        self.tokens_per_block = 0 if w.n_blocks == 1 else w.n_blk
        self.ws = la.alloc_backward_workspace(w.B, w.n_total, w.H, w.d, self.tokens_per_block, device=self.device)
        self.rope = (la.make_rope(Hg=w.Hg, Wg=w.Wg, T=w.frames, t_offset=0, dims=w.rope_dims, base=w.rope_base)
                     if w.rope else None)
        self._launches = 0

    @property
    def launches_per_step(self) -> int:
        return self._launches

    def step(self, after_call: Optional[Callable[[int], None]] = None, stream=None) -> None:
        q, k, v, dout = self.inputs[0]
        la.full_backward(q, k, v, dout, self.tokens_per_block, rope=self.rope, eps=self.w.eps, ws=self.ws,
                         grads=tuple(self.outs), stream=stream)
        self._launches = la.la_last_launch_count()
        if after_call:
            after_call(0)

    def tokens_per_call(self, i: int) -> int:
        return self.calls[i][2].shape[1]
