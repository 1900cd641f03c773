"""A DiT block sweep: many Lynx linear layers back to back on one stream,
replayed from one CUDA graph.

Each layer is one ``lynx_linear`` call (``skip_sparsify`` for the layers that
selective layer skipping leaves dense: qingkeai.online article section 03.3),
or ``lynx_linear_act`` for a layer whose output takes an activation (the MLP
up-projection's GELU) in the GEMM epilogue.
The calls share one workspace, which is safe because they run in order on one
stream.  Capturing the whole sequence once and replaying it removes the host
launch work (argument checks, tensor-map encoding, launches) from every step;
the kernels' launch parameters, tensor maps included, are fixed at capture.
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
            self.layers.append(t)
            ws_bytes = max(ws_bytes, lynx.lynx_workspace_bytes(M, N, K, 64))
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=self.device)
        self.graph = None

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

    def capture(self):
        """Record one pass into a CUDA graph.  Run the sweep once first (the
        library's one-time per-device set-up must not happen inside capture)."""
        import torch

        torch.cuda.synchronize(self.device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.run()
        torch.cuda.synchronize(self.device)
        self.graph = graph
        return graph

    def replay(self):
        if self.graph is None:
            raise RuntimeError("capture() first")
        self.graph.replay()
