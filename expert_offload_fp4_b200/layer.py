"""One decode MoE layer through the C ABI: route -> slot lookup -> miss
streaming (copy stream) -> expert FFN with the combine fused in (compute stream).

This is the public call a user makes per (token batch, layer); it owns only the
per-call device buffers.  The copy of missed experts runs on its own stream and
the FFN kernel starts at once: CTAs on resident experts compute while the copy
engine streams the misses, whose CTAs wait for the slot's ready ticket.
"""
from __future__ import annotations

import torch

from . import api


class DecodeLayer:
    def __init__(self, pool: api.Pool, T: int, device="cuda", renormalize=1, overlap=True):
        if T > pool.max_tokens:
            raise ValueError("T exceeds the pool's max_tokens")
        # overlap=False issues the miss copies before the FFN launch (the host waits
        # for the lookup first): slower, but safe under tools that serialise kernels
        self.pool, self.T, self.renormalize, self.overlap = pool, T, renormalize, overlap
        k, H, E = pool.k, pool.H, pool.E
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.w = torch.empty((T, k), dtype=torch.float32, device=device)
        self.slot_of = torch.empty((T, k), dtype=torch.int32, device=device)
        self.y_part = torch.empty((T, k, H), dtype=torch.float32, device=device)
        self.y = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.ws = torch.zeros(api.route_workspace_bytes(T, E), dtype=torch.uint8, device=device)
        self.lookup = api.Lookup(min(T * k, E))
        self.copy_stream = torch.cuda.Stream(device=device)
        # optional timing hooks: lists that receive (start, end) CUDA events recorded
        # around the miss copies (copy stream) and around the FFN launch (compute
        # stream; setting this one issues the layer call by call from Python)
        self.ffn_events = None
        self.copy_events = None
        self._spare_events = []

    def reserve_copy_events(self, n):
        """Create n (start, end) event pairs for the copy_events hook ahead of time
        (torch creates a CUDA event at its first record, so each is recorded once)."""
        for _ in range(n):
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for e in ev:
                e.record(self.copy_stream)
            self._spare_events.append(ev)

    def __call__(self, layer, x, wr, bias, stream=None):
        """x [T, H] bf16, wr [E, H] bf16, bias [E] fp32 (or None), all on the device.
        Returns y [T, H] bf16 (a buffer reused by the next call).

        Order: route, lookup, FFN and combine are enqueued back to back on the
        compute stream; then the host collects the lookup's miss list and drives
        the copy engine.  The FFN's CTAs on resident experts run at once; those on
        missed experts wait (bounded) for the slot's ready ticket that the copy
        stream writes after each expert's block lands."""
        p = self.pool
        if self.ffn_events is None:
            # the whole layer in one native call
            ev = None
            if self.copy_events is not None:
                if not self._spare_events:
                    self.reserve_copy_events(1)
                ev = self._spare_events[-1]
            api.decode_layer(p, layer, x, wr, bias, self.renormalize, self.idx, self.w, self.slot_of,
                             self.y_part, self.y, self.status, self.ws, lookup=self.lookup,
                             copy_events=ev, overlap=self.overlap, stream=stream,
                             copy_stream=self.copy_stream)
            if ev is not None and self.lookup.n_miss:
                self.copy_events.append((self._spare_events.pop(), self.lookup.n_miss))
            return self.y
        # step by step, with events around the FFN launch
        api.route(x, wr, bias, p.k, self.renormalize, self.idx, self.w, self.ws, stream)
        if not self.overlap:
            api.slot_lookup(p, layer, self.idx, self.slot_of, self.lookup, stream)
            if self.lookup.n_miss:
                api.stream_misses(p, layer, self.lookup, self.copy_stream)
            api.expert_ffn(p, layer, x, self.idx, self.w, self.slot_of, self.y_part, self.status, self.y,
                           stream)
            return self.y
        api.slot_lookup_launch(p, layer, self.idx, self.slot_of, stream)
        if self.ffn_events is not None:
            cur = stream if stream is not None else torch.cuda.current_stream()
            fe = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            fe[0].record(cur)
        api.expert_ffn(p, layer, x, self.idx, self.w, self.slot_of, self.y_part, self.status, self.y, stream)
        if self.ffn_events is not None:
            fe[1].record(cur)
        # nothing that can wait for the device between the FFN launch and the copies
        api.slot_lookup_result(p, self.lookup)
        if self.lookup.n_miss:
            if self.copy_events is not None:
                ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                ev[0].record(self.copy_stream)
            api.stream_misses(p, layer, self.lookup, self.copy_stream)
            if self.copy_events is not None:
                ev[1].record(self.copy_stream)
                self.copy_events.append((ev, self.lookup.n_miss))
        if self.ffn_events is not None:
            self.ffn_events.append((fe, self.lookup.n_uniq, self.lookup.n_miss))
        return self.y
