"""Block-diffusion decoding with the bidirectional mixer: a per-layer cache of
forward states and a whole block (its denoising steps over every layer, then
the commit) captured once as a CUDA graph and replayed per block.

"Training Hybrid Block Diffusion Language Models with Partial
Bidirectionality", Abstract and Methodology: the reverse scan is confined to
the active block, so each layer's mixer caches the forward state of the
prefix and reuses it exactly; a step never changes the cache, and the
finished block is appended to it. "DiffuMamba: High-Throughput Diffusion LMs
with Mamba Backbone", 2. Methodology, Training & Inference Strategy: block-
wise denoising with that cache.

Every computation runs in the library's kernels (ssd_prefix_state_layers,
ssd_block_step, ssd_prefix_state); this module holds buffers and records and
replays the graph.
"""
from __future__ import annotations

import torch

from . import (SSD_PATH_AUTO, Workspace, ssd_block_step, ssd_prefix_state, ssd_prefix_state_layers)


class BlockDiffusionCache:
    """The cached forward states of `layers` mixer layers, (layers, batch, H,
    P, N) fp32, one allocation."""

    def __init__(self, layers: int, batch: int, nheads: int, headdim: int, dstate: int, device=None):
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.state = torch.zeros(layers, batch, nheads, headdim, dstate, dtype=torch.float32, device=self.device)
        self.ws_prefill = Workspace(self.device)

    @property
    def layers(self) -> int:
        return self.state.shape[0]

    def prefill(self, x, dt, A, B, chunk: int = 256):
        """Every layer's state after its prefix, in one call: x (layers, batch,
        L, H, P), dt (layers, batch, L, H) and B (layers, batch, L, G, N) the
        forward direction's, A (layers, H)."""
        ssd_prefix_state_layers(x, dt, A, B, out=self.state, chunk=chunk, workspace=self.ws_prefill)
        return self.state

    def commit(self, x, dt, A, B, chunk: int = 256):
        """Append a finished block to every layer's state, in place, in one call
        (stacked forward-direction inputs as for prefill)."""
        ssd_prefix_state_layers(x, dt, A, B, init=self.state, out=self.state, chunk=chunk,
                                workspace=self.ws_prefill)
        return self.state


class BlockGraph:
    """One block of `steps` denoising steps over every layer of a cache, then
    the commit of the block, captured as one CUDA graph.

    The graph reads its inputs from static buffers this object owns, laid out
    per step and layer as ssd_block_step takes them:
      x  (steps, layers, batch, T, H, P)       io
      dt (steps, layers, 2, batch, T, H)       io
      B, C (steps, layers, 2, batch, T, G, N)  io
    and A, D (layers, 2, H) fp32. Step s of layer l writes out[s, l]
    (batch, T, H, P). After the last step every layer's state takes the block
    through its forward direction with the last step's inputs (one
    ssd_prefix_state per layer: the block step's direction-stacked layout
    keeps each layer's forward slices contiguous). Fill the buffers, then
    replay(); the outputs and the cache are ready when the stream reaches the
    replay's end."""

    def __init__(self, cache: BlockDiffusionCache, steps: int, block: int, nheads: int, headdim: int, dstate: int,
                 ngroups: int, dtype=torch.bfloat16, path: int = SSD_PATH_AUTO):
        self.cache, self.steps, self.path = cache, steps, path
        L, b = cache.layers, cache.state.shape[1]
        dev = cache.device
        self.x = torch.zeros(steps, L, b, block, nheads, headdim, dtype=dtype, device=dev)
        self.dt = torch.zeros(steps, L, 2, b, block, nheads, dtype=dtype, device=dev)
        self.B = torch.zeros(steps, L, 2, b, block, ngroups, dstate, dtype=dtype, device=dev)
        self.C = torch.zeros_like(self.B)
        self.A = torch.zeros(L, 2, nheads, dtype=torch.float32, device=dev)
        self.D = torch.zeros(L, 2, nheads, dtype=torch.float32, device=dev)
        self.out = torch.zeros_like(self.x)
        self.ws_step = [Workspace(dev) for _ in range(L)]
        self.ws_commit = [Workspace(dev) for _ in range(L)]
        self.graph = None

    def _block(self):
        st = self.cache.state
        for s in range(self.steps):
            for layer in range(self.cache.layers):
                ssd_block_step(self.x[s, layer], self.dt[s, layer], self.A[layer], self.B[s, layer], self.C[s, layer],
                               self.D[layer], st[layer], out=self.out[s, layer], path=self.path,
                               workspace=self.ws_step[layer])
        last = self.steps - 1
        for layer in range(self.cache.layers):
            ssd_prefix_state(self.x[last, layer], self.dt[last, layer, 0], self.A[layer, 0], self.B[last, layer, 0],
                             init=st[layer], out=st[layer], workspace=self.ws_commit[layer])

    def capture(self):
        """Record the block. Runs it once first, outside the capture, to size the
        workspaces (so that run commits a block into the cache: capture on a
        scratch state, or save and restore the cache around it)."""
        saved = self.cache.state.clone()
        dev = self.cache.device
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self._block()
            self.cache.state.copy_(saved)
            torch.cuda.synchronize(dev)
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph, stream=side):
                self._block()
        torch.cuda.current_stream(dev).wait_stream(side)
        self.cache.state.copy_(saved)
        return self

    def replay(self):
        if self.graph is None:
            raise RuntimeError("BlockGraph.replay before capture")
        self.graph.replay()
