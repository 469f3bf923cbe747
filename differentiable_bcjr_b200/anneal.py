"""Annealing-sweep driver: the forward and backward calls of one temperature
schedule, captured once as a CUDA graph and replayed.

"BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization",
technical summary: training anneals the temperature towards zero, where the
soft codeword becomes the hard Viterbi code.  One sweep here is, for every T
of the schedule in order, w_hat_T = soft codeword of w at T and
(grad_w_T, grad_codebook_T) = its vector-Jacobian product with the upstream
gradient g.

The calls of the library allocate nothing and are asynchronous on the
current stream, so after one warm-up sweep (which sizes the workspaces and
caches the launch geometry) the whole sweep is captured in one graph; a
replay reads the current contents of the static input buffers `w`, `g` and
`codebook` and overwrites the static outputs.
"""
from __future__ import annotations

import torch

from . import Workspace, bcjr_backward, bcjr_forward


class AnnealSweep:
    """A captured sweep over `temperatures` for fixed shapes.

    Inputs live in the static tensors `self.w` [N][n], `self.g` [N][n] and
    `self.codebook` [S]; `run(w, g)` copies into them and replays.  Outputs:
    `self.w_hat` and `self.grad_w` [len(T)][N][n], `self.grad_codebook`
    [len(T)][S] (each temperature's own gradient, not accumulated).
    """

    def __init__(self, codebook: torch.Tensor, temperatures, state_bits: int, k: int, n_seq: int, seq_len: int,
                 checkpoint_interval: int = 0):
        if not codebook.is_cuda:
            raise ValueError("AnnealSweep runs on a CUDA device")
        dev = codebook.device
        self.temperatures = [float(t) for t in temperatures]
        self.state_bits, self.k, self.C = int(state_bits), int(k), int(checkpoint_interval)
        S = 1 << self.state_bits
        if codebook.shape != (S,):
            raise ValueError(f"codebook must have {S} entries")
        nT = len(self.temperatures)
        self.codebook = codebook.detach().contiguous().clone()
        self.w = torch.zeros((n_seq, seq_len), dtype=torch.float32, device=dev)
        self.g = torch.zeros_like(self.w)
        self.w_hat = torch.empty((nT, n_seq, seq_len), dtype=torch.float32, device=dev)
        self.grad_w = torch.empty_like(self.w_hat)
        self.grad_codebook = torch.empty((nT, S), dtype=torch.float32, device=dev)
        self._ws_f = Workspace(dev)
        self._ws_b = Workspace(dev)
        self.graph = None

    def _sweep(self):
        for i, T in enumerate(self.temperatures):
            bcjr_forward(self.w, self.codebook, T, self.state_bits, self.k, checkpoint_interval=self.C,
                         ws=self._ws_f, out=self.w_hat[i])
            bcjr_backward(self.g, self.w, self.codebook, self.w_hat[i], T, self.state_bits, self.k,
                          checkpoint_interval=self.C, ws=self._ws_b, grad_codebook=self.grad_codebook[i],
                          accumulate_codebook=False, grad_w_out=self.grad_w[i])

    def capture(self):
        """Warm up once on a side stream, then capture one sweep."""
        side = torch.cuda.Stream(device=self.w.device)
        side.wait_stream(torch.cuda.current_stream(self.w.device))
        with torch.cuda.stream(side):
            self._sweep()
        torch.cuda.current_stream(self.w.device).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._sweep()

    def run(self, w: torch.Tensor, g: torch.Tensor):
        """One sweep on (w, g); returns (w_hat, grad_w, grad_codebook) (the static outputs)."""
        self.w.copy_(w)
        self.g.copy_(g)
        if self.graph is None:
            self.capture()
        self.graph.replay()
        return self.w_hat, self.grad_w, self.grad_codebook
