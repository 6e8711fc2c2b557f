"""The MoE layer and the batch-1 decode stack, chained through libzmoe's C entry points.

Buffers are allocated once (torch is used for device memory only); every step runs in
libzmoe's kernels.  A layer is one call of ``zmoe_moe_layer`` (one cooperative launch for a few
tokens and at decode sizes); ``MoELayerRunner.run_steps`` chains the separate entry points instead:

    zmoe_route -> zmoe_permute -> zmoe_grouped_swiglu -> zmoe_combine

ZONOS2 Technical Report digest, "method overview and architecture", item 5: 24 MoE layers
of 16 experts with top-1 routing and top-2 in the last one, fed by the RMSNorm of the
summed codebook embeddings.  Per-layer wiring of the stack (the pages leave it open):
pre-norm residual, h <- h + MoE_l(RMSNorm_l(h)), with h kept in fp32 and the layer input
rounded to the weights' dtype.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch

from . import zmoe as Z


@dataclass
class MoEWeights:
    """One layer's device weights.  Shapes: W_r [E, d], W_gate/W_up [E, f, d], W_down [E, d, f].

    A dense FFN layer is the E = 1 case; its router may be None (the gate is 1)."""

    w_router: Optional[torch.Tensor]
    w_gate: torch.Tensor
    w_up: torch.Tensor
    w_down: torch.Tensor
    sel_bias: Optional[torch.Tensor] = None     # f32 [E]
    logit_bias: Optional[torch.Tensor] = None   # f32 [E]
    gamma: Optional[torch.Tensor] = None        # f32 [d], pre-norm gain (stack only)
    k: int = 1
    w_down_f16: Optional[torch.Tensor] = None   # f16 [E, d, f], prepared by prepare_f16()
    down_scale: Optional[torch.Tensor] = None   # f32 [E]

    def prepare_f16(self) -> "MoEWeights":
        """The prefill path's f16 copy of W_down (zmoe_prepare_w_down_f16), made once."""
        if self.w_down_f16 is None:
            self.w_down_f16, self.down_scale = Z.zmoe_prepare_w_down_f16(self.w_down)
        return self

    @property
    def E(self) -> int:
        return self.w_gate.shape[0]

    @property
    def d(self) -> int:
        return self.w_gate.shape[2]

    @property
    def f(self) -> int:
        return self.w_gate.shape[1]

    @property
    def dtype(self) -> torch.dtype:
        return self.w_gate.dtype

    @staticmethod
    def from_host(L, device="cuda", dtype: Optional[torch.dtype] = None) -> "MoEWeights":
        """From a ``moe_inputs.MoELayerInputs`` (float32 arrays, bf16-exact for bf16 layers)."""
        dt = dtype or (torch.bfloat16 if L.dtype == "bf16" else torch.float32)

        def dev(a, t=dt):
            return None if a is None else torch.from_numpy(a).to(device=device, dtype=t).contiguous()

        return MoEWeights(dev(L.w_router), dev(L.w_gate), dev(L.w_up), dev(L.w_down),
                          dev(L.sel_bias, torch.float32), dev(L.logit_bias, torch.float32),
                          dev(L.gamma, torch.float32), L.k)


class MoELayerRunner:
    """Preallocated buffers for T tokens through one MoE layer shape."""

    def __init__(self, T: int, E: int, d: int, f: int, k: int, dtype: torch.dtype, device="cuda"):
        self.T, self.E, self.d, self.f, self.k, self.dtype = T, E, d, f, k, dtype
        dev = torch.device(device)
        M = T * k
        self.idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.gates = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.margin = torch.empty((T,), dtype=torch.float32, device=dev)
        self.perm_outs = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
                              offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                              perm=torch.empty(M, dtype=torch.int32, device=dev),
                              inv_perm=torch.empty((T, k), dtype=torch.int32, device=dev),
                              x_perm=torch.empty((M, d), dtype=dtype, device=dev))
        self.perm_ws = torch.empty(max(Z.zmoe_permute_workspace_size(T, E, k), 16), dtype=torch.uint8, device=dev)
        self.h = torch.empty((M, Z.hidden_cols(f, dtype)), dtype=dtype, device=dev)
        self.y_perm = torch.empty((M, d), dtype=torch.float32, device=dev)
        self.ffn_ws = torch.empty(max(Z.zmoe_grouped_swiglu_workspace_size(M, E, d, f, dtype), 16),
                                  dtype=torch.uint8, device=dev)
        self.y = torch.empty((T, d), dtype=torch.float32, device=dev)
        self.h16 = torch.empty((M, f), dtype=torch.float16, device=dev) if dtype == torch.bfloat16 else None
        self.layer_ws = torch.empty(max(Z.zmoe_moe_layer_workspace_size(T, d, f, E, k, dtype), 16), dtype=torch.uint8,
                                    device=dev)

    def run(self, x: Optional[torch.Tensor], W: MoEWeights, residual: Optional[torch.Tensor] = None,
            out: Optional[torch.Tensor] = None, stream=None, gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
            x_norm: Optional[torch.Tensor] = None) -> torch.Tensor:
        """y = residual + sum_i gate_i * FFN_{e_i}(x), f32 [T, d], in one zmoe_moe_layer call.

        With ``gamma`` the layer input is RMSNorm(residual) * gamma (written to ``x_norm`` if given)."""
        outs = dict(expert_idx=self.idx, gates=self.gates, margin=self.margin)
        if x_norm is not None:
            outs["x_norm"] = x_norm
        return Z.zmoe_moe_layer(W.w_router, W.w_gate, W.w_up, W.w_down, W.k, x=x, h=residual, gamma=gamma, eps=eps,
                                logit_bias=W.logit_bias, sel_bias=W.sel_bias,
                                out=self.y if out is None else out, outs=outs, workspace=self.layer_ws,
                                stream=stream)

    def run_f16h(self, x: Optional[torch.Tensor], W: MoEWeights, residual: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, stream=None, gamma: Optional[torch.Tensor] = None,
                 eps: float = 1e-6) -> torch.Tensor:
        """The layer in one zmoe_moe_layer_f16h call (prefill sizes; W needs prepare_f16())."""
        outs = dict(expert_idx=self.idx, gates=self.gates, margin=self.margin)
        return Z.zmoe_moe_layer_f16h(W.w_router, W.w_gate, W.w_up, W.w_down_f16, W.down_scale, W.k, x=x, h=residual,
                                     gamma=gamma, eps=eps, logit_bias=W.logit_bias, sel_bias=W.sel_bias,
                                     out=self.y if out is None else out, outs=outs, workspace=self.layer_ws16,
                                     stream=stream)

    @property
    def layer_ws16(self) -> torch.Tensor:
        if not hasattr(self, "_layer_ws16"):
            n = int(Z.lib().zmoe_moe_layer_f16h_workspace_size(self.T, self.d, self.f, self.E, self.k))
            self._layer_ws16 = torch.empty(max(n, 16), dtype=torch.uint8, device=self.y.device)
        return self._layer_ws16

    def run_steps_f16h(self, x: torch.Tensor, W: MoEWeights, residual: Optional[torch.Tensor] = None,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """route -> permute -> grouped SwiGLU (f16 h) -> combine through the separate entry points."""
        Z.zmoe_route(x, W.w_router, W.k, W.logit_bias, W.sel_bias, outs=(self.idx, self.gates, self.margin),
                     stream=stream)
        Z.zmoe_permute(self.idx, x, W.E, outs=self.perm_outs, workspace=self.perm_ws, stream=stream)
        Z.zmoe_grouped_swiglu_f16h(self.perm_outs["x_perm"], self.perm_outs["offsets"], W.w_gate, W.w_up,
                                   W.w_down_f16, W.down_scale, h=self.h16, y_perm=self.y_perm, stream=stream)
        return Z.zmoe_combine(self.y_perm, self.perm_outs["inv_perm"], self.gates, residual,
                              out=self.y if out is None else out, stream=stream)

    def run_steps(self, x: torch.Tensor, W: MoEWeights, residual: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """The same layer through the four separate entry points (intermediates kept in this runner)."""
        Z.zmoe_route(x, W.w_router, W.k, W.logit_bias, W.sel_bias, outs=(self.idx, self.gates, self.margin),
                     stream=stream)
        Z.zmoe_permute(self.idx, x, W.E, outs=self.perm_outs, workspace=self.perm_ws, stream=stream)
        Z.zmoe_grouped_swiglu(self.perm_outs["x_perm"], self.perm_outs["offsets"], W.w_gate, W.w_up, W.w_down,
                              h=self.h, y_perm=self.y_perm, workspace=self.ffn_ws, stream=stream)
        return Z.zmoe_combine(self.y_perm, self.perm_outs["inv_perm"], self.gates, residual,
                              out=self.y if out is None else out, stream=stream)


class DecodeStack:
    """Embedding sum + RMSNorm, then L pre-norm residual MoE layers, for T tokens per step; with head
    weights, also the codebook heads and the greedy next frame (``next_ids``)."""

    def __init__(self, tables: torch.Tensor, gamma0: torch.Tensor, layers: List[MoEWeights], eps: float = 1e-6,
                 T: int = 1, w_heads: Optional[torch.Tensor] = None, gamma_out: Optional[torch.Tensor] = None,
                 persistent: Optional[bool] = None):
        self.tables, self.gamma0, self.layers, self.eps, self.T = tables, gamma0, layers, eps, T
        L0 = layers[0]
        dev = tables.device
        self.dtype = L0.dtype
        self.runners = {(L.E, L.k): MoELayerRunner(T, L.E, L.d, L.f, L.k, L.dtype, dev) for L in layers}
        self.ids = torch.empty((T, tables.shape[0]), dtype=torch.int32, device=dev)
        self.h = torch.empty((T, L0.d), dtype=torch.float32, device=dev)
        self.x = torch.empty((T, L0.d), dtype=L0.dtype, device=dev)
        self.w_heads, self.gamma_out = w_heads, gamma_out
        self.next_ids = torch.empty((T, tables.shape[0]), dtype=torch.int32, device=dev)
        self.head_x = torch.empty((T, L0.d), dtype=L0.dtype, device=dev)
        self.head_ws = torch.empty(max(int(Z.lib().zmoe_output_heads_workspace_size(T, tables.shape[0])), 16),
                                   dtype=torch.uint8, device=dev) if w_heads is not None else None
        self.record_inputs = False
        self.layer_inputs: List[torch.Tensor] = []
        self.layer_h: List[torch.Tensor] = []
        self.layer_idx: List[torch.Tensor] = []
        # One token per step: the whole stack (embedding included) is one zmoe_decode_stack call when
        # its sizes are supported; otherwise (or with persistent=False) one zmoe_moe_layer call per layer.
        nL, d, f = len(layers), L0.d, L0.f
        ws = Z.zmoe_decode_stack_workspace_size(nL, d, f, max(L.E for L in layers)) if T == 1 else 0
        if persistent and ws == 0:
            raise ValueError("zmoe_decode_stack does not support these sizes")
        self.persistent = ws > 0 and persistent is not False and L0.dtype == torch.bfloat16
        if self.persistent:
            self.stack_ws = torch.empty(ws, dtype=torch.uint8, device=dev)
            self.stack_arr = Z.stack_layers(layers)
            self.rec = dict(layer_idx=torch.empty((nL, 2), dtype=torch.int32, device=dev),
                            layer_gates=torch.empty((nL, 2), dtype=torch.float32, device=dev),
                            layer_h=torch.empty((nL, d), dtype=torch.float32, device=dev),
                            layer_x=torch.empty((nL, d), dtype=L0.dtype, device=dev))

    def step(self, ids: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """One decode step; returns the final fp32 residual stream h [T, d]."""
        if ids is not None:
            self.ids.copy_(ids)
        if self.persistent:
            Z.zmoe_decode_stack(self.layers, self.h, self.eps, ids=self.ids, tables=self.tables, gamma0=self.gamma0,
                                outs=self.rec if self.record_inputs else None, workspace=self.stack_ws, stream=stream,
                                layer_array=self.stack_arr)
            if self.record_inputs:
                r = self.rec
                self.layer_h = [r["layer_h"][l:l + 1] for l in range(len(self.layers))]
                self.layer_inputs = [r["layer_x"][l:l + 1] for l in range(len(self.layers))]
                self.layer_idx = [r["layer_idx"][l:l + 1, :L.k] for l, L in enumerate(self.layers)]
            self._heads(stream)
            return self.h
        Z.zmoe_embed_sum_rmsnorm(self.ids, self.tables, self.gamma0, self.eps, out=self.h, stream=stream)
        if self.record_inputs:
            self.layer_inputs, self.layer_h, self.layer_idx = [], [], []
        for L in self.layers:
            R = self.runners[(L.E, L.k)]
            if self.record_inputs:
                self.layer_h.append(self.h.clone())
            # h <- h + MoE(RMSNorm(h) * gamma): one zmoe_moe_layer call, in place
            R.run(None, L, residual=self.h, out=self.h, stream=stream, gamma=L.gamma, eps=self.eps,
                  x_norm=self.x if self.record_inputs else None)
            if self.record_inputs:
                self.layer_inputs.append(self.x.clone())
                self.layer_idx.append(R.idx.clone())
        self._heads(stream)
        return self.h

    def _heads(self, stream=None):
        if self.w_heads is not None:
            outs = dict(ids=self.next_ids, x=self.head_x) if self.record_inputs else dict(ids=self.next_ids)
            Z.zmoe_output_heads(self.h, self.w_heads, self.gamma_out, self.eps, outs=outs, workspace=self.head_ws,
                                stream=stream)


def stack_from_bits(tables_bits, gamma0, layer_small, expert_bits, n_layers: int, E: int, d: int, f: int,
                    k_of, eps: float = 1e-6, T: int = 1, device="cuda", E_of=None, heads_bits=None,
                    gamma_out=None, persistent: Optional[bool] = None) -> DecodeStack:
    """Builds a DecodeStack on the device from host arrays.

    tables_bits: uint16 [N, V, d] bf16 bit patterns; gamma0: f32 [d]; layer_small(l) -> (W_r f32 [E, d]
    bf16-exact, sel_bias f32 [E], gamma f32 [d]), W_r and sel_bias None for a dense layer; expert_bits:
    iterable of (l, e, (wg, wu, wd) uint16 bit arrays); k_of(l) -> experts per token in layer l;
    E_of(l) -> experts of layer l (default E; 1 for a dense FFN layer); heads_bits: uint16 [N, V, d] bf16
    bit patterns of the codebook heads (with gamma_out f32 [d], the final norm's gain), or None.
    """
    import numpy as np

    def bits_to_dev(b):
        return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(device).view(torch.bfloat16)

    layers = []
    for l in range(n_layers):
        wr, sb, gm = layer_small(l)
        El = E_of(l) if E_of is not None else E
        layers.append(MoEWeights(None if wr is None else torch.from_numpy(wr).to(device=device, dtype=torch.bfloat16),
                                 torch.empty((El, f, d), dtype=torch.bfloat16, device=device),
                                 torch.empty((El, f, d), dtype=torch.bfloat16, device=device),
                                 torch.empty((El, d, f), dtype=torch.bfloat16, device=device),
                                 None if sb is None else torch.from_numpy(sb).to(device), None,
                                 torch.from_numpy(gm).to(device), k_of(l)))
    for l, e, (wg, wu, wd) in expert_bits:
        layers[l].w_gate[e].copy_(bits_to_dev(wg))
        layers[l].w_up[e].copy_(bits_to_dev(wu))
        layers[l].w_down[e].copy_(bits_to_dev(wd))
    tables = bits_to_dev(tables_bits)
    heads = bits_to_dev(heads_bits) if heads_bits is not None else None
    g_out = torch.from_numpy(gamma_out).to(device) if gamma_out is not None else None
    return DecodeStack(tables, torch.from_numpy(gamma0).to(device), layers, eps, T, heads, g_out, persistent)
