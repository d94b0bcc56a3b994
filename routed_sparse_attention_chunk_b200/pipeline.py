"""Three-stream schedule of the query path over a sequence of query batches.

"MSA: Memory Sparse Attention" README, "Inference Pipeline": K̄r stays on the
GPU for routing, the pooled K̄ / V̄ may stay in host memory, and only the
selected documents' rows are fetched, asynchronously, when they are selected.
With the bank's K̄ / V̄ in page-locked host memory the gather of a batch is
bound by the host link, while routing and attention are bound by HBM and the
tensor cores.  This schedule overlaps them across consecutive batches:

    stream R:  msa_route_topk(i+1)
    stream G:  msa_gather(i)        (after route(i); reads topk_idx of batch i)
    stream A:  msa_sparse_attn(i-1) (after gather(i-1))

The gathered rows are double-buffered; events order each buffer's reuse
(gather(i) waits for attention(i-2), which read the same buffer; route(i)
waits for gather(i-2), which read the same topk_idx slot when the caller
reuses two index tensors).  It only orders library calls: every step runs in
the library's kernels, and the results are those of the sequential calls.
"""
from __future__ import annotations

import torch

from . import gather, route_topk, route_topk_workspace_size, sparse_attn, sparse_attn_workspace_size


class QueryPipeline:
    """Buffers, streams and events of the schedule for one bank and one batch shape.

    bank: dict with Krbar, kr_rnorm, doc_chunk_off (device) and Kbar, Vbar (device or
    page-locked host memory).  Every batch passed to run() has the shapes given here.
    """

    def __init__(self, bank: dict, k: int, Mmax: int, B: int, Tq: int, Lloc: int, Hq: int, Hkv: int, d: int,
                 Hr: int, dtype, device, err_flag=None):
        self.bank, self.k, self.Mmax = bank, k, Mmax
        D = bank["doc_chunk_off"].numel() - 1
        C = bank["Krbar"].shape[0]
        self.rws = torch.empty(max(256, route_topk_workspace_size(B, Tq, Hr, D, C, k)), dtype=torch.uint8,
                               device=device)
        self.aws = torch.empty(max(256, sparse_attn_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Mmax)),
                               dtype=torch.uint8, device=device)
        self.Km = [torch.zeros((B, Mmax, Hkv, d), dtype=dtype, device=device) for _ in range(2)]
        self.Vm = [torch.zeros((B, Mmax, Hkv, d), dtype=dtype, device=device) for _ in range(2)]
        self.ml = [torch.zeros(B, dtype=torch.int32, device=device) for _ in range(2)]
        self.flag = err_flag if err_flag is not None else torch.zeros(1, dtype=torch.int32, device=device)
        self.sR, self.sG, self.sA = (torch.cuda.Stream(device=device) for _ in range(3))
        self.ev_r = [torch.cuda.Event() for _ in range(2)]   # route(i) done
        self.ev_g = [torch.cuda.Event() for _ in range(2)]   # gather(i) done
        self.ev_a = [torch.cuda.Event() for _ in range(2)]   # attention(i) done
        self.n = 0  # batches enqueued so far (the event rings continue across run() calls)

    def run(self, batches, marks=None) -> None:
        """Enqueue batches (dicts with Qr, Q, Kloc, Vloc, O, topk_idx and optionally lse).

        The three streams start after the caller's current stream and the caller's stream waits
        for all of them at the end.  marks, if given, receives (stage, start, end) CUDA events
        recorded on the stage's own stream around every call.
        """
        caller = torch.cuda.current_stream()
        for s in (self.sR, self.sG, self.sA):
            s.wait_stream(caller)
        bank = self.bank

        def timed(stage, stream, fn):
            if marks is None:
                fn()
                return
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            marks.append((stage, e0, e1))

        for bt in batches:
            i, slot = self.n, self.n % 2
            with torch.cuda.stream(self.sR):
                if i >= 2:
                    self.sR.wait_event(self.ev_g[slot])
                timed("route_topk", self.sR, lambda: route_topk(
                    bt["Qr"], bank["Krbar"], bank["kr_rnorm"], bank["doc_chunk_off"], self.k, bt["topk_idx"],
                    self.rws, err_flag=self.flag))
                self.ev_r[slot].record(self.sR)
            with torch.cuda.stream(self.sG):
                self.sG.wait_event(self.ev_r[slot])
                if i >= 2:
                    self.sG.wait_event(self.ev_a[slot])
                timed("gather", self.sG, lambda: gather(
                    bt["topk_idx"], bank["doc_chunk_off"], bank["Kbar"], bank["Vbar"], self.Km[slot], self.Vm[slot],
                    self.ml[slot], self.flag))
                self.ev_g[slot].record(self.sG)
            with torch.cuda.stream(self.sA):
                self.sA.wait_event(self.ev_g[slot])
                timed("sparse_attn", self.sA, lambda: sparse_attn(
                    bt["Q"], bt["Kloc"], bt["Vloc"], self.Km[slot], self.Vm[slot], self.ml[slot], bt["O"],
                    bt.get("lse"), ws=self.aws, err_flag=self.flag))
                self.ev_a[slot].record(self.sA)
            self.n += 1
        for s in (self.sR, self.sG, self.sA):
            caller.wait_stream(s)
