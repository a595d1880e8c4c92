"""PoetxLinear: device buffers of one POET-X layer and thin wrappers around
the C calls (allocation with torch, arithmetic in libpoetx.so).

State of a layer (POET-X write-up, sections 2-3 and the merge step of its API
snippet): the frozen weight stored in the frame of the current permutations
(W[j'][i'] = W0[permR[i']][permP[j']], [n][m]), the permutations, the packed
triangles qR, qP (the trainable parameters) and the G blocks built from them.
"""
from __future__ import annotations

from typing import NamedTuple, Optional, Tuple

import torch

from . import (POETX_BF16, POETX_FOLD_ALL, POETX_FP32, make_layer, poetx_backward, poetx_backward_dG,
               poetx_backward_recompute_workspace_bytes, poetx_backward_workspace_bytes, poetx_cnp_backward,
               poetx_cnp_workspace_bytes,
               poetx_forward, poetx_forward_workspace_bytes, poetx_frame_export, poetx_frame_import,
               poetx_layer_cnp_build, poetx_layer_cnp_workspace_bytes, poetx_layers_cnp_build,
               poetx_layers_cnp_workspace_bytes, poetx_merge, poetx_merge_workspace_bytes, poetx_weight_dequantize,
               poetx_weight_quantize, poetx_adamw_step)

_TORCH_DTYPE = {POETX_BF16: torch.bfloat16, POETX_FP32: torch.float32}


def _need(t, shape, dtype, device: torch.device, name: str) -> None:
    """Host-side check of a tensor handed to the library.  The C calls take
    raw device pointers and trust the layer's sizes, so a tensor of another
    shape, dtype, device or stride must be refused here, before any launch."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device.type != device.type or (device.index is not None and t.device.index != device.index):
        raise ValueError(f"{name}: tensor on {t.device}, the layer is on {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


class Saved(NamedTuple):
    """Activations the forward keeps for the backward: Y ([T][n], the P-side
    input in the Psi_P frame) and optionally Xg ([T][m], x in the Psi_R frame)."""
    y: Optional[torch.Tensor]
    xg: Optional[torch.Tensor]


class PoetxLinear:
    """One layer z = x R W0 P (x: [T][m], z: [T][n]).

    `fold` (POETX_FOLD_* bits, default 0) lets a bf16 layer apply a block
    product to the weight instead of the token rows where that moves fewer
    bytes; 0 keeps the write-up's input-centric evaluation everywhere."""

    def __init__(self, m: int, n: int, b: int, dtype: int, device="cuda", fold: int = 0):
        if dtype not in _TORCH_DTYPE:
            raise ValueError("dtype must be POETX_BF16 or POETX_FP32")
        if fold & ~POETX_FOLD_ALL:
            raise ValueError("fold: unknown POETX_FOLD bits")
        self.fold = fold
        self.m, self.n, self.b, self.dtype = m, n, b, dtype
        self.device = torch.device(device)
        td = _TORCH_DTYPE[dtype]
        tri = b * (b - 1) // 2
        self.W = torch.empty((n, m), dtype=td, device=self.device)
        self.permR = torch.empty(m, dtype=torch.int32, device=self.device)
        self.permP = torch.empty(n, dtype=torch.int32, device=self.device)
        self.qR = torch.zeros((m // b, tri), dtype=torch.float32, device=self.device)
        self.qP = torch.zeros((n // b, tri), dtype=torch.float32, device=self.device)
        self.GR = torch.empty((m // b, b, b), dtype=td, device=self.device)
        self.GP = torch.empty((n // b, b, b), dtype=td, device=self.device)
        self._ws = {}
        self.Wq = None      # POET-XQ: int8 codes of W and per-row scales
        self.Wscale = None
        self._wscratch = None

    # -------------------------------------------------------------- POET-XQ
    def quantize_weight(self, scratch: Optional[torch.Tensor] = None, stream=None) -> None:
        """Keep W as int8 codes + per-row scales (POET-XQ) and drop the bf16
        copy; every forward / backward dequantizes it into `scratch` (a flat
        tensor of at least n*m elements of the layer dtype, which several
        layers may share) right before use."""
        self.Wq = torch.empty((self.n, self.m), dtype=torch.int8, device=self.device)
        self.Wscale = torch.empty(self.n, dtype=torch.float32, device=self.device)
        poetx_weight_quantize(self.n, self.m, self.W, self.dtype, self.Wq, self.Wscale, stream)
        if scratch is None:
            scratch = torch.empty(self.n * self.m, dtype=self.torch_dtype, device=self.device)
        if scratch.numel() < self.n * self.m:
            raise ValueError(f"scratch: {scratch.numel()} elements, the layer needs {self.n * self.m}")
        _need(scratch, (scratch.numel(),), self.torch_dtype, self.device, "scratch")
        self._wscratch = scratch
        self.W = scratch[: self.n * self.m].view(self.n, self.m)

    def _dequantize(self, stream=None) -> None:
        if self.Wq is not None:
            self.W = self._wscratch[: self.n * self.m].view(self.n, self.m)
            poetx_weight_dequantize(self.n, self.m, self.Wq, self.Wscale, self.dtype, self.W, stream)

    @property
    def torch_dtype(self) -> torch.dtype:
        return _TORCH_DTYPE[self.dtype]

    def abi(self):
        return make_layer(self.m, self.n, self.b, self.dtype, self.W, self.permR, self.permP, self.qR, self.qP,
                          self.GR, self.GP, self.fold)

    def workspace(self, kind: str, nbytes: int) -> torch.Tensor:
        ws = self._ws.get(kind)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=self.device)
            self._ws[kind] = ws
        return ws

    # -------------------------------------------------------------- state
    def load(self, W0lin: torch.Tensor, permR: torch.Tensor, permP: torch.Tensor, qR: torch.Tensor,
             qP: torch.Tensor, stream=None) -> None:
        """Set the permutations and triangles, import the natural nn.Linear
        weight W0^T ([n][m]) into the frame, and build G."""
        W0lin = W0lin.contiguous()
        _need(W0lin, (self.n, self.m), self.torch_dtype, self.device, "W0lin")
        for name, t, shape in (("permR", permR, self.permR.shape), ("permP", permP, self.permP.shape),
                               ("qR", qR, self.qR.shape), ("qP", qP, self.qP.shape)):
            if tuple(t.shape) != tuple(shape):
                raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
        self.permR.copy_(permR)
        self.permP.copy_(permP)
        self.qR.copy_(qR)
        self.qP.copy_(qP)
        poetx_frame_import(self.abi(), W0lin, stream)
        self.build(stream)

    def export_weight(self, stream=None) -> torch.Tensor:
        out = torch.empty((self.n, self.m), dtype=self.torch_dtype, device=self.device)
        poetx_frame_export(self.abi(), out, stream)
        return out

    def build(self, stream=None) -> None:
        """G_R, G_P from qR, qP (Cayley-Neumann), both sides in one batch."""
        L = self.abi()
        nb = poetx_layer_cnp_workspace_bytes(L)
        ws = self.workspace("cnp", nb)
        poetx_layer_cnp_build(L, ws, nb, stream)

    # -------------------------------------------------------------- layer
    def forward(self, x: torch.Tensor, save: bool = True, save_xg: bool = False, z: Optional[torch.Tensor] = None,
                y: Optional[torch.Tensor] = None, xg: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, Optional["Saved"]]:
        """z = x R W0 P.  With `save`, also returns what the backward needs:
        Y (the P-side input) and, with `save_xg`, Xg = x[:, permR]."""
        T = x.shape[0]
        td = self.torch_dtype
        _need(x, (T, self.m), td, self.device, "x")
        if z is None:
            z = torch.empty((T, self.n), dtype=td, device=self.device)
        _need(z, (T, self.n), td, self.device, "z")
        if save and y is None:
            y = torch.empty((T, self.n), dtype=td, device=self.device)
        if save:
            _need(y, (T, self.n), td, self.device, "y")
        if save and save_xg and xg is None:
            xg = torch.empty((T, self.m), dtype=td, device=self.device)
        if not (save and save_xg):
            xg = None
        if xg is not None:
            _need(xg, (T, self.m), td, self.device, "xg")
        self._dequantize(stream)
        L = self.abi()
        nb = poetx_forward_workspace_bytes(L, T)
        ws = self.workspace("fwd", nb)
        poetx_forward(L, T, x, z, y if save else None, xg, ws, nb, stream)
        return z, (Saved(y, xg) if save else None)

    def backward(self, x: torch.Tensor, saved, dz: torch.Tensor, need_dx: bool = True,
                 dx: Optional[torch.Tensor] = None, dqR: Optional[torch.Tensor] = None,
                 dqP: Optional[torch.Tensor] = None, accumulate: bool = False, stream=None):
        """dx, dqR, dqP of L = <dz, z>.  `saved` is what forward returned (or
        just the saved Y tensor); None recomputes Y from x (the "mem" variant,
        which keeps no [T][n] activation between forward and backward)."""
        if saved is None:
            saved = Saved(None, None)
        elif isinstance(saved, torch.Tensor):
            saved = Saved(saved, None)
        T = dz.shape[0]
        if need_dx and dx is None:
            dx = torch.empty((T, self.m), dtype=self.torch_dtype, device=self.device)
        if dqR is None:
            dqR = torch.empty_like(self.qR)
        if dqP is None:
            dqP = torch.empty_like(self.qP)
        self._check_backward(T, x, saved, dz, dx if need_dx else None)
        _need(dqR, tuple(self.qR.shape), torch.float32, self.device, "dqR")
        _need(dqP, tuple(self.qP.shape), torch.float32, self.device, "dqP")
        self._dequantize(stream)
        L = self.abi()
        nb = (poetx_backward_workspace_bytes if saved.y is not None else poetx_backward_recompute_workspace_bytes)(L, T)
        ws = self.workspace("bwd", nb)
        poetx_backward(L, T, x, saved.y, saved.xg, dz, dx if need_dx else None, dqR, dqP, int(accumulate), ws, nb,
                       stream)
        return (dx if need_dx else None), dqR, dqP

    def backward_dG(self, x: torch.Tensor, saved, dz: torch.Tensor, dGR: torch.Tensor, dGP: torch.Tensor,
                    need_dx: bool = True, dx: Optional[torch.Tensor] = None, accumulate: bool = False,
                    stream=None) -> Optional[torch.Tensor]:
        """backward() up to the token sums dGR [m/b][b][b], dGP [n/b][b][b]
        (fp32), without the CNP backward; LayerGroup.cnp_backward turns the dG
        of all layers into dq in one batch."""
        if saved is None:
            saved = Saved(None, None)
        elif isinstance(saved, torch.Tensor):
            saved = Saved(saved, None)
        T = dz.shape[0]
        if need_dx and dx is None:
            dx = torch.empty((T, self.m), dtype=self.torch_dtype, device=self.device)
        self._check_backward(T, x, saved, dz, dx if need_dx else None)
        _need(dGR, (self.m // self.b, self.b, self.b), torch.float32, self.device, "dGR")
        _need(dGP, (self.n // self.b, self.b, self.b), torch.float32, self.device, "dGP")
        self._dequantize(stream)
        L = self.abi()
        nb = (poetx_backward_workspace_bytes if saved.y is not None else poetx_backward_recompute_workspace_bytes)(L, T)
        ws = self.workspace("bwd", nb)
        poetx_backward_dG(L, T, x, saved.y, saved.xg, dz, dx if need_dx else None, dGR, dGP, int(accumulate), ws, nb,
                          stream)
        return dx if need_dx else None

    def _check_backward(self, T: int, x, saved: "Saved", dz, dx) -> None:
        td = self.torch_dtype
        _need(dz, (T, self.n), td, self.device, "dz")
        if x is not None:
            _need(x, (T, self.m), td, self.device, "x")
        elif saved.xg is None:
            raise ValueError("x: needed unless the forward saved Xg")
        if saved.y is not None:
            _need(saved.y, (T, self.n), td, self.device, "saved y")
        if saved.xg is not None:
            _need(saved.xg, (T, self.m), td, self.device, "saved xg")
        if dx is not None:
            _need(dx, (T, self.m), td, self.device, "dx")

    def merge(self, new_permR: torch.Tensor, new_permP: torch.Tensor, stream=None) -> None:
        """W0 <- R W0 P, re-expressed in the frame of the new permutations;
        q = 0 and G = I afterwards."""
        L = self.abi()
        nb = poetx_merge_workspace_bytes(L)
        ws = self.workspace("merge", nb)
        W_out = torch.empty_like(self.W)
        newR = new_permR.to(device=self.device, dtype=torch.int32).contiguous()
        newP = new_permP.to(device=self.device, dtype=torch.int32).contiguous()
        _need(newR, (self.m,), torch.int32, self.device, "new_permR")
        _need(newP, (self.n,), torch.int32, self.device, "new_permP")
        poetx_merge(L, newR, newP, W_out, ws, nb, stream)
        self.W = W_out
        self.permR.copy_(newR)
        self.permP.copy_(newP)


class LayerGroup:
    """Several layers with the same b and dtype whose G blocks are rebuilt
    together (one batched CNP build for all of them), optionally with their
    packed triangles in one flat buffer (qR then qP of each layer, in order)
    so one optimizer launch updates all of them."""

    def __init__(self, layers):
        self.layers = list(layers)
        self._ws = None
        self._bws = None
        self.q = None
        self.m1 = None
        self.m2 = None
        self.steps = 0

    def flatten_params(self) -> torch.Tensor:
        """Move every layer's qR, qP into one flat fp32 buffer (the layers keep
        views into it) and allocate the optimizer moments; returns the buffer."""
        total = sum(L.qR.numel() + L.qP.numel() for L in self.layers)
        dev = self.layers[0].device
        self.q = torch.empty(total, dtype=torch.float32, device=dev)
        off = 0
        for L in self.layers:
            for name in ("qR", "qP"):
                t = getattr(L, name)
                view = self.q[off:off + t.numel()].view_as(t)
                view.copy_(t)
                setattr(L, name, view)
                off += t.numel()
        self.m1 = torch.zeros_like(self.q)
        self.m2 = torch.zeros_like(self.q)
        return self.q

    def optimizer_step(self, grad: torch.Tensor, lr: float, beta1: float = 0.9, beta2: float = 0.95,
                       eps: float = 1e-8, weight_decay: float = 0.0, stream=None) -> None:
        """AdamW on the flat packed triangles with the flat gradient `grad`
        (same layout), then the batched CNP rebuild of every G."""
        if self.q is None:
            raise RuntimeError("flatten_params() first")
        _need(grad, tuple(self.q.shape), torch.float32, self.q.device, "grad")
        self.steps += 1
        poetx_adamw_step(self.q.numel(), self.q, grad, self.m1, self.m2, lr, beta1, beta2, eps, weight_decay,
                         self.steps, stream)
        self.build(stream)

    def dG_buffer(self) -> torch.Tensor:
        """A flat fp32 buffer [sum of blocks][b][b] for the dG of every layer,
        blocks in the order of the packed triangles (R then P of each layer)."""
        b = self.layers[0].b
        nblk = sum(L.m // b + L.n // b for L in self.layers)
        return torch.empty((nblk, b, b), dtype=torch.float32, device=self.layers[0].device)

    def dG_views(self, dG: torch.Tensor):
        """(dGR, dGP) views of each layer into a dG_buffer()."""
        out, off = [], 0
        for L in self.layers:
            nR, nP = L.m // L.b, L.n // L.b
            out.append((dG[off:off + nR], dG[off + nR:off + nR + nP]))
            off += nR + nP
        return out

    def cnp_backward(self, dG: torch.Tensor, dq: torch.Tensor, accumulate: bool = False, stream=None) -> None:
        """dq (flat, the layout of flatten_params) from the dG of every layer
        (dG_buffer layout): one batched CNP backward over all blocks."""
        if self.q is None:
            raise RuntimeError("flatten_params() first")
        L0 = self.layers[0]
        nblk = sum(L.m // L.b + L.n // L.b for L in self.layers)
        _need(dG, (nblk, L0.b, L0.b), torch.float32, self.q.device, "dG")
        _need(dq, tuple(self.q.shape), torch.float32, self.q.device, "dq")
        nb = poetx_cnp_workspace_bytes(nblk, L0.b, L0.dtype)
        if self._bws is None or self._bws.numel() < nb:
            self._bws = torch.empty(max(nb, 1), dtype=torch.uint8, device=L0.device)
        poetx_cnp_backward(nblk, L0.b, self.q, dG, dq, int(accumulate), L0.dtype, self._bws, nb, stream)

    def build(self, stream=None) -> None:
        abis = [L.abi() for L in self.layers]
        nb = poetx_layers_cnp_workspace_bytes(abis)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=self.layers[0].device)
        poetx_layers_cnp_build(abis, self._ws, nb, stream)
