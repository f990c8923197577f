"""Host-memory inputs and outputs, with copies overlapped with the attention kernel.

For callers whose q, k, v live in (pinned) host memory, e.g. one forward per request.
A ``HostPipeline`` keeps two sets of device buffers.  Step i's host-to-device copies
run on one stream while step i-1's kernel runs on another, and a third stream copies
step i-1's result back.  The PCIe or C2C link traffic then hides behind the
tensor-core work instead of adding to it.  Events order the streams:

    h2d(i)  waits  kernel(i-2)  (buffer set i % 2 free again)
    kernel(i) waits h2d(i)
    d2h(i)  waits  kernel(i)
    kernel(i) waits d2h(i-2)   (output set i % 2 read out)

Every step runs the same public entry point as a device-memory caller
(``attn_prefix_fwd``).
"""
from __future__ import annotations

import torch

from . import _binding


class HostPipeline:
    """Double-buffered host -> device -> host forward for one fixed problem shape.

    shape: (B, H, Tq, Tk, D).  submit() enqueues one step and returns at once; the
    host output tensors of a step may be read after synchronize() (or after the
    event returned by submit() has completed).
    """

    def __init__(self, shape, device=None, scale=None):
        B, H, Tq, Tk, D = (int(x) for x in shape)
        self.shape = (B, H, Tq, Tk, D)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.scale = scale
        bf = torch.bfloat16
        mk = lambda *s, dt=bf: [torch.empty(s, dtype=dt, device=self.device) for _ in range(2)]  # noqa: E731
        self.q, self.k, self.v = mk(B, H, Tq, D), mk(B, H, Tk, D), mk(B, H, Tk, D)
        self.kv = mk(B, dt=torch.int32)
        self.out, self.lse = mk(B, H, Tq, D), mk(B, H, Tq, dt=torch.float32)
        self.s_h2d = torch.cuda.Stream(self.device)
        self.s_run = torch.cuda.Stream(self.device)
        self.s_d2h = torch.cuda.Stream(self.device)
        self.ev_run = [None, None]   # kernel of the step that last used buffer set i
        self.ev_d2h = [None, None]   # read-out of the step that last used output set i
        self.step = 0

    def submit(self, q, k, v, kv_len, out, lse=None):
        """Enqueue one step: host q, k, v [B,H,T,D] bf16 and kv_len [B] int32 in; host
        out [B,H,Tq,D] bf16 (and lse [B,H,Tq] fp32, optional) written.  Host tensors
        should be pinned for the copies to run asynchronously."""
        i = self.step & 1
        with torch.cuda.device(self.device):
            with torch.cuda.stream(self.s_h2d):
                if self.ev_run[i] is not None:
                    self.s_h2d.wait_event(self.ev_run[i])
                for d, h in ((self.q[i], q), (self.k[i], k), (self.v[i], v), (self.kv[i], kv_len)):
                    d.copy_(h, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(self.s_h2d)
            with torch.cuda.stream(self.s_run):
                self.s_run.wait_event(ev_in)
                if self.ev_d2h[i] is not None:
                    self.s_run.wait_event(self.ev_d2h[i])
                _binding.fwd(self.q[i], self.k[i], self.v[i], self.kv[i], self.scale, out=self.out[i],
                             lse=self.lse[i])
                self.ev_run[i] = torch.cuda.Event()
                self.ev_run[i].record(self.s_run)
            with torch.cuda.stream(self.s_d2h):
                self.s_d2h.wait_event(self.ev_run[i])
                out.copy_(self.out[i], non_blocking=True)
                if lse is not None:
                    lse.copy_(self.lse[i], non_blocking=True)
                self.ev_d2h[i] = torch.cuda.Event()
                self.ev_d2h[i].record(self.s_d2h)
        self.step += 1
        return self.ev_d2h[i]

    def synchronize(self):
        for s in (self.s_h2d, self.s_run, self.s_d2h):
            s.synchronize()
