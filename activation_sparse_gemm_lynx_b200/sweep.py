"""A DiT block sweep: many Lynx linear layers back to back, replayed from one
CUDA graph.

Each layer is one ``lynx_linear`` call (``skip_sparsify`` for the layers that
selective layer skipping leaves dense: qingkeai.online article section 03.3),
or ``lynx_linear_act`` for a layer whose output takes an activation (the MLP
up-projection's GELU) in the GEMM epilogue.

Two schedules:

* ``run()``: the calls in order on one stream, sharing one workspace (safe
  because they run in order).  Inside a call the GEMM's launch already
  overlaps the sparsify pass's tail (programmatic launch).
* ``run_overlapped(chunks)``: every layer, or each of its ``chunks`` row blocks,
  is a work item split at the layer's internal hand-off
  (``lynx_linear_begin`` / ``lynx_linear_finish``): the sparsify passes run on
  a side stream and the GEMMs on the caller's stream, each GEMM after its own
  pass (an event), with two workspaces in turn (a pass waits for the GEMM that
  last read its workspace).  So the next item's pass can take the SMs that a
  GEMM's last, partly filled round of tiles leaves idle, and with row chunks
  each chunk's compressed operand is smaller (the hand-off from pass to GEMM
  stays in L2).  The layers' inputs must not depend on each other's outputs,
  as in this sweep (no attention or normalisation between the linears).

Capturing a schedule once and replaying it removes the host launch work
(argument checks, tensor-map encoding, launches) from every step; the kernels'
launch parameters, tensor maps included, are fixed at capture.
"""
import numpy as np

from . import lynx


class LinearSweep:
    """Device-resident inputs, weights and outputs of a list of layers.

    ``layers`` holds dicts with the bf16-bit numpy arrays ``X``, ``W``, ``bias``,
    ``A``, ``B`` (as made by ``workloads.make_linear_inputs``), ``skip`` and
    optionally ``act`` (a ``lynx.LYNX_ACT_*`` value, default none).
    """

    def __init__(self, layers, device="cuda"):
        import torch

        self.device = torch.device(device)
        self.layers = []
        ws_bytes = 0
        for layer in layers:
            t = {k: self._dev(layer[k]) for k in ("X", "W", "bias", "A", "B")}
            M, K = t["X"].shape
            N = t["W"].shape[0]
            t["Y"] = torch.empty((M, N), dtype=torch.bfloat16, device=self.device)
            t["skip"] = bool(layer["skip"])
            t["act"] = int(layer.get("act", lynx.LYNX_ACT_NONE))
            t["shape"] = (M, K, N)
            t["r"] = t["A"].shape[0] if t["A"] is not None else lynx.lynx_lora_rank()
            self.layers.append(t)
            ws_bytes = max(ws_bytes, lynx.lynx_workspace_bytes(M, N, K, t["r"]))
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=self.device)
        self.graph = None
        self._overlap = {}  # chunks -> (side stream, workspaces, events)

    def _dev(self, bits):
        import torch

        if bits is None:
            return None
        host = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
        return host.to(self.device)

    @property
    def dense_flops(self):
        """Dense-equivalent work 2*M*N*K summed over the layers."""
        return sum(2 * M * N * K for (M, K, N) in (t["shape"] for t in self.layers))

    def run(self):
        """Enqueue every layer on the current stream."""
        for t in self.layers:
            if t["act"] == lynx.LYNX_ACT_NONE:
                lynx.lynx_linear(t["X"], t["W"], t["bias"], t["A"], t["B"], skip_sparsify=t["skip"],
                                 Y=t["Y"], workspace=self.workspace)
            else:
                lynx.lynx_linear_act(t["X"], t["W"], t["bias"], t["A"], t["B"], skip_sparsify=t["skip"],
                                     act=t["act"], Y=t["Y"], workspace=self.workspace)

    def work_items(self, chunks=1):
        """(layer, first row, last row) of every work item, in order: each
        layer in `chunks` blocks of rows (multiples of 256, the CTA-pair tile)."""
        items = []
        for t in self.layers:
            M = t["shape"][0]
            per = -(-M // chunks)
            per = -(-per // 256) * 256
            for r0 in range(0, M, per):
                items.append((t, r0, min(M, r0 + per)))
        return items

    def _overlap_state(self, chunks):
        import torch

        st = self._overlap.get(chunks)
        if st is None:
            items = self.work_items(chunks)
            ws_bytes = max(lynx.lynx_workspace_bytes(r1 - r0, t["shape"][2], t["shape"][1], t["r"])
                           for (t, r0, r1) in items)
            wss = [torch.empty(ws_bytes, dtype=torch.uint8, device=self.device) for _ in range(2)]
            events = [(torch.cuda.Event(), torch.cuda.Event()) for _ in items]
            st = (torch.cuda.Stream(device=self.device), wss, events, torch.cuda.Event())
            self._overlap[chunks] = st
        return st

    def run_overlapped(self, chunks=1):
        """Enqueue every work item: its sparsify pass on a side stream, its GEMM
        on the current stream after that pass, two workspaces in turn."""
        import torch

        side, wss, events, fork = self._overlap_state(chunks)
        main = torch.cuda.current_stream(self.device)
        fork.record(main)
        side.wait_event(fork)  # nothing before this schedule is overtaken
        for k, (t, r0, r1) in enumerate(self.work_items(chunks)):
            began, done = events[k]
            ws = wss[k % 2]
            X = t["X"][r0:r1]
            Y = t["Y"][r0:r1]
            args = (X, t["W"], t["bias"], t["A"], t["B"])
            kw = dict(skip_sparsify=t["skip"], act=t["act"], Y=Y, workspace=ws)
            with torch.cuda.stream(side):
                if k >= 2:
                    side.wait_event(events[k - 2][1])  # the GEMM that last read this workspace
                lynx.lynx_linear_begin(*args, **kw, stream=side)
                began.record(side)
            main.wait_event(began)
            lynx.lynx_linear_finish(*args, **kw, stream=main)
            done.record(main)

    def side_streams(self):
        """The side streams the overlapped schedules have used (their sparsify
        passes report device errors in these streams' status words)."""
        return [st[0] for st in self._overlap.values()]

    def capture(self, overlapped=False, chunks=1):
        """Record one pass into a CUDA graph.  Run the same schedule once first
        (the library's one-time per-device set-up must not happen inside
        capture)."""
        import torch

        torch.cuda.synchronize(self.device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            if overlapped:
                self.run_overlapped(chunks)
            else:
                self.run()
        torch.cuda.synchronize(self.device)
        self.graph = graph
        return graph

    def replay(self):
        if self.graph is None:
            raise RuntimeError("capture() first")
        self.graph.replay()
