"""The MLP block of a 12B hybrid Mamba-Transformer layer (up-projection ->
squared ReLU -> down-projection), forward and backward, as a sequence of the
library's C-ABI calls.

Every operand of the six GEMMs is NVFP4 (aisight.pl, section "Architektura
NVFP4 kontra ograniczenia mikroskalowania"); the Wgrad operands carry the
16-point random Hadamard transform, and the gradient operand stochastic
rounding (same page, section "Technologie stabilizujace proces
treningowy").  This module only orders the calls and holds the buffers:
argument marshalling through `binding`, all arithmetic in the CUDA library.

A step, with X [M x H], W1 [F x H], W2 [H x F], dY2 [M x H] (bf16):
  forward   X_r = rowwise(X); a1 = amax(W1); W1_r = rowwise(W1, a1); W1_c = colwise(W1, a1)
            Y1 = X_r . W1_r^T and h = relu(Y1)^2 from one GEMM (the epilogue also
            returns max|h| and max|RHT(h)|)
            h_r = rowwise(h, amax supplied); a2 = amax(W2); W2_r = rowwise(W2, a2);
            W2_c = colwise(W2, a2); Y2 = h_r . W2_r^T
  backward  dY2_r = rowwise(dY2)
            dY1 = (dY2_r . W2_c^T) * 2 relu(Y1) from one GEMM (the epilogue applies the
            derivative to the bf16 dh, which is never stored, and returns max|dY1| and
            max|RHT(dY1)|)
            dY2_c = colwise(dY2, RHT, SR); h_c = colwise(h, RHT, amax supplied); dW2 = dY2_c . h_c^T
            dY1_r = rowwise(dY1, amax supplied); dX = dY1_r . W1_c^T
            dY1_c = colwise(dY1, RHT, SR, amax supplied); X_c = colwise(X, RHT); dW1 = dY1_c . X_c^T
With fused=False the two squared-ReLU steps run as their own kernels after
plain GEMMs (dh stored), with the same results bit for bit.
"""
import torch

from . import binding

SEED = 1234


class MlpStep:
    """Device buffers and the call sequence of one MLP block step (bf16 in and
    out, dW in float32).  `inputs` maps X, W1, W2, dY2 to device tensors.
    `lib` is the module whose calls run the step (the binding of the CUDA
    library; tests substitute a CPU stand-in with the same call names)."""

    def __init__(self, inputs, seed=SEED, lib=binding, fused=True):
        self.B = B = lib
        self.seed = seed
        self.fused = fused
        self.d = inputs
        X, W1 = inputs["X"], inputs["W1"]
        M, H = X.shape
        F = W1.shape[0]
        self.M, self.H, self.F = M, H, F
        device = X.device
        bf = dict(dtype=torch.bfloat16, device=device)
        self.Y1 = torch.empty((M, F), **bf)
        self.h = torch.empty_like(self.Y1)
        self.Y2 = torch.empty((M, H), **bf)
        self.dh = None if fused else torch.empty_like(self.Y1)  # the fused Dgrad epilogue never stores dh
        self.dY1 = torch.empty_like(self.Y1)
        self.dX = torch.empty((M, H), **bf)
        self.dW1 = torch.empty((F, H), dtype=torch.float32, device=device)
        self.dW2 = torch.empty((H, F), dtype=torch.float32, device=device)
        self.ws = B.workspace(256, device)      # GEMM status word
        self.qws = B.workspace(B.nvfp4_quantize_dual_workspace_size(), device)
        self.amax = torch.zeros(16, dtype=torch.float32, device=device)  # h, RHT(h), dY1, RHT(dY1) at 0, 4, 8, 12
        self.wamax = torch.zeros(8, dtype=torch.float32, device=device)  # W1, W2 at 0, 4
        mk = B.empty_nvfp4
        self.q = {
            "X_r": mk(M, H, device), "W1_r": mk(F, H, device), "W1_c": mk(H, F, device),
            "h_r": mk(M, F, device), "W2_r": mk(H, F, device), "W2_c": mk(F, H, device),
            "dY2_r": mk(M, H, device), "dY2_c": mk(H, M, device), "h_c": mk(F, M, device),
            "dY1_r": mk(M, F, device), "dY1_c": mk(F, M, device), "X_c": mk(H, M, device),
        }
        self.launches = 0

    # Each call appends (kind, algorithmic work, end event) to `ev` when given.
    def _mark(self, ev, kind, work):
        self.launches += self.B.nvfp4_last_launch_count()
        if ev is not None:
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            ev.append((kind, work, e))

    def _quant(self, x, key, colwise=False, sr=False, rht=False, amax_in=None, ev=None, bytes_per_elem=None):
        B = self.B
        B.nvfp4_quantize(x, orientation=B.NVFP4_COLWISE if colwise else B.NVFP4_ROWWISE,
                         rounding=B.NVFP4_SR if sr else B.NVFP4_RTN, rht=rht, seed=self.seed, amax_in=amax_in,
                         out=self.q[key], ws=self.qws)
        self._mark(ev, "quant", x.numel() * bytes_per_elem(amax_in is not None) if bytes_per_elem else 0)

    def _weight(self, w, key_r, key_c, amax, ev=None, bytes_per_elem=None):
        """A weight's two RTN operands from one amax pass: the amax does not depend on the
        orientation (no transform), so both quantisations take it as supplied."""
        self.B.nvfp4_amax(w, out=amax, ws=self.qws)
        self._mark(ev, "quant", w.numel() * bytes_per_elem("amax") if bytes_per_elem else 0)
        self._quant(w, key_r, amax_in=amax, ev=ev, bytes_per_elem=bytes_per_elem)
        self._quant(w, key_c, colwise=True, amax_in=amax, ev=ev, bytes_per_elem=bytes_per_elem)

    def _gemm(self, a, b, out, ev=None):
        self.B.nvfp4_gemm(self.q[a], self.q[b], out=out, ws=self.ws)
        self._mark(ev, "gemm", 2 * self.q[a].rows * self.q[b].rows * self.q[a].k)

    def forward(self, X=None, Y2=None, ev=None, bytes_per_elem=None):
        d, X = self.d, (self.d["X"] if X is None else X)
        Y2 = self.Y2 if Y2 is None else Y2
        kw = dict(ev=ev, bytes_per_elem=bytes_per_elem)
        self._quant(X, "X_r", **kw)
        self._weight(d["W1"], "W1_r", "W1_c", self.wamax[0:1], **kw)
        # relu^2 also returns max|h| and max|RHT(h)|: both quantisations of h skip their amax pass
        if self.fused:
            self.B.nvfp4_gemm_relu2_fwd(self.q["X_r"], self.q["W1_r"], seed=self.seed, y=self.Y1, h=self.h,
                                        amax_out=self.amax[0:1], amax_rht_out=self.amax[4:5], ws=self.qws)
            self._mark(ev, "gemm", 2 * self.M * self.F * self.H)
        else:
            self._gemm("X_r", "W1_r", self.Y1, ev)
            self.B.nvfp4_relu2_fwd_amax_rht(self.Y1, seed=self.seed, out=self.h, amax_out=self.amax[0:1],
                                            amax_rht_out=self.amax[4:5], ws=self.qws)
            self._mark(ev, "relu2", self.Y1.numel())
        self._quant(self.h, "h_r", amax_in=self.amax[0:1], **kw)
        self._weight(d["W2"], "W2_r", "W2_c", self.wamax[4:5], **kw)
        self._gemm("h_r", "W2_r", Y2, ev)

    def backward(self, X=None, dY2=None, ev=None, bytes_per_elem=None, grad_ready=None):
        """grad_ready(name, tensor), if given, is called as soon as the GEMM producing
        a weight gradient is queued: dW2 first, then dW1."""
        d = self.d
        X = d["X"] if X is None else X
        dY2 = d["dY2"] if dY2 is None else dY2
        kw = dict(ev=ev, bytes_per_elem=bytes_per_elem)
        self._quant(dY2, "dY2_r", **kw)
        # dY1 = dh * 2 relu(Y1), with max|dY1| and max|RHT(dY1)| for its two quantisations
        if self.fused:
            self.B.nvfp4_gemm_relu2_bwd(self.q["dY2_r"], self.q["W2_c"], self.Y1, seed=self.seed, out=self.dY1,
                                        amax_out=self.amax[8:9], amax_rht_out=self.amax[12:13], ws=self.qws)
            self._mark(ev, "gemm", 2 * self.M * self.F * self.H)
        else:
            self._gemm("dY2_r", "W2_c", self.dh, ev)
        self._quant(dY2, "dY2_c", colwise=True, sr=True, rht=True, **kw)
        self._quant(self.h, "h_c", colwise=True, rht=True, amax_in=self.amax[4:5], **kw)
        self._gemm("dY2_c", "h_c", self.dW2, ev)
        if grad_ready:
            grad_ready("dW2", self.dW2)
        if not self.fused:
            self.B.nvfp4_relu2_bwd_amax_rht(self.dh, self.Y1, seed=self.seed, out=self.dY1, amax_out=self.amax[8:9],
                                            amax_rht_out=self.amax[12:13], ws=self.qws)
            self._mark(ev, "relu2", self.Y1.numel())
        self._quant(self.dY1, "dY1_r", amax_in=self.amax[8:9], **kw)
        self._gemm("dY1_r", "W1_c", self.dX, ev)
        self._quant(self.dY1, "dY1_c", colwise=True, sr=True, rht=True, amax_in=self.amax[12:13], **kw)
        self._quant(X, "X_c", colwise=True, rht=True, **kw)
        self._gemm("dY1_c", "X_c", self.dW1, ev)
        if grad_ready:
            grad_ready("dW1", self.dW1)

    def step(self, X=None, dY2=None, Y2=None, ev=None, bytes_per_elem=None, grad_ready=None):
        """Forward and backward; X, dY2 and the output Y2 default to the step's own buffers."""
        self.forward(X, Y2, ev=ev, bytes_per_elem=bytes_per_elem)
        self.backward(X, dY2, ev=ev, bytes_per_elem=bytes_per_elem, grad_ready=grad_ready)

    def capture(self, stream=None):
        """The step on its own buffers (inputs["X"], inputs["dY2"], self.Y2 ...) captured once in
        a CUDA graph; returns the graph, whose replay() runs the same 24 kernels with the same
        arguments.  A loop copies each step's inputs into those buffers and replays.  The
        step is run once eagerly first (the library's per-device set-up happens outside the
        capture).  The gradient exchange is not captured: call it after replay()."""
        s = stream if stream is not None else torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            self.step()
        torch.cuda.current_stream().wait_stream(s)
        return g
