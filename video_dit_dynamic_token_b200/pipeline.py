"""Host-to-host sparse attention with the transfers overlapped.

Heads are independent through the whole path: each head has its own plan,
Q/K block scales, V channel scales and attention.  A batch held in pinned host
memory can therefore be processed in chunks of heads, so that the host->device
copy of chunk c+1, the plan and forward kernels of chunk c and the
device->host copy of chunk c-1's output run at the same time (two copy engines
and the SMs).  Nothing is computed here: the chunks go through
`lx_sparse_attn_plan` and `lx_sparse_attn_fwd` like any other call, and the
class only owns the device buffers, streams and events.
"""
from __future__ import annotations

import torch

from . import empty_plan, lx_sparse_attn, lx_sparse_attn_ws_size


class HostPipeline:
    """Plan + forward over pinned host tensors [B, H, L, D] (bf16), in chunks of
    `heads_per_chunk` heads, with two device slots per buffer.

    Slot reuse is ordered by events: the copy of chunk c+2 into a slot waits for
    chunk c's kernels (which read Q/K/V), and chunk c+2's kernels wait for chunk
    c's output copy (which reads O)."""

    def __init__(self, B, H, L, D, keep, mode="int8fp8", heads_per_chunk=8, device="cuda"):
        self.B, self.H, self.L, self.D = B, H, L, D
        self.keep, self.mode = keep, mode
        self.hc = max(1, min(heads_per_chunk, H))
        self.dev = torch.device(device)
        self.chunks = [(h0, min(H, h0 + self.hc)) for h0 in range(0, H, self.hc)]
        shape = (B, self.hc, L, D)
        self.slots = []
        for _ in range(2):
            q, k, v, o = (torch.empty(shape, dtype=torch.bfloat16, device=self.dev) for _ in range(4))
            ws = torch.empty(max(lx_sparse_attn_ws_size(q, keep, mode), 256), dtype=torch.uint8, device=self.dev)
            # one plan per distinct chunk width (the last chunk may be narrower)
            plans = {n: empty_plan(B, n, L, D, keep, self.dev) for n in {h1 - h0 for h0, h1 in self.chunks}}
            self.slots.append(dict(q=q, k=k, v=v, o=o, ws=ws, plans=plans))
        self.s_h2d = torch.cuda.Stream(self.dev)
        self.s_cmp = torch.cuda.Stream(self.dev)
        self.s_d2h = torch.cuda.Stream(self.dev)

    def run(self, hQ, hK, hV, hO, stream=None):
        """Enqueue the whole batch; work starts after everything already queued on
        `stream` (default: the current stream), and `stream` waits for the last
        output copy, so events recorded on it bracket the transfers and kernels."""
        caller = stream if stream is not None else torch.cuda.current_stream(self.dev)
        start = torch.cuda.Event()
        start.record(caller)
        ev_h2d, ev_cmp, ev_d2h = [], [], []
        for c, (h0, h1) in enumerate(self.chunks):
            n = h1 - h0
            sl = self.slots[c % 2]
            dq, dk, dv, do = (sl[x][:, :n] for x in ("q", "k", "v", "o"))
            e_h2d, e_cmp, e_d2h = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
            self.s_h2d.wait_event(start)
            if c >= 2:
                self.s_h2d.wait_event(ev_cmp[c - 2])
            with torch.cuda.stream(self.s_h2d):
                dq.copy_(hQ[:, h0:h1], non_blocking=True)
                dk.copy_(hK[:, h0:h1], non_blocking=True)
                dv.copy_(hV[:, h0:h1], non_blocking=True)
                e_h2d.record(self.s_h2d)
            self.s_cmp.wait_event(e_h2d)
            if c >= 2:
                self.s_cmp.wait_event(ev_d2h[c - 2])
            with torch.cuda.stream(self.s_cmp):
                lx_sparse_attn(dq, dk, dv, self.keep, self.mode, plan=sl["plans"][n], out=do, ws=sl["ws"],
                               stream=self.s_cmp)
                e_cmp.record(self.s_cmp)
            self.s_d2h.wait_event(e_cmp)
            with torch.cuda.stream(self.s_d2h):
                hO[:, h0:h1].copy_(do, non_blocking=True)
                e_d2h.record(self.s_d2h)
            ev_h2d.append(e_h2d)
            ev_cmp.append(e_cmp)
            ev_d2h.append(e_d2h)
        caller.wait_event(ev_d2h[-1])
        return hO
