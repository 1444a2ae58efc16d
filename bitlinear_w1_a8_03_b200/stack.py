"""A stack of decoder-layer BitLinears on the device, driven through the C ABI.

Every BitLinear input is quantised on entry and the residual addition stays in
float ("1.58-bit 大模型极限量化实战", chenxutan.com/d/5049.html §6.1: Q/K/V, the
output projection and the MLP linears become BitLinear; norms and residual
additions stay in floating point).  The pages give no wiring between the seven
linears of a layer; the stack uses this one: q, k, v, gate and up consume
quant(h); o consumes quant(y_v); down consumes quant(y_up); the next layer's
input is h' = y_o + y_down (binary32), summed inside the next quantisation.

Per layer this is two bitlinear_linear_block calls (four kernels chained by
programmatic dependent launch); a final call materialises the last h'.  This
module only marshals arguments: every step runs in libbitlinear.so.
"""
from __future__ import annotations

import bitlinear_w1_a8_03_b200 as bl

MATRICES = ("q", "k", "v", "o", "gate", "up", "down")


def shapes(hidden: int, ffn: int) -> dict:
    """(N, K) of each linear of one layer."""
    return {"q": (hidden, hidden), "k": (hidden, hidden), "v": (hidden, hidden), "o": (hidden, hidden),
            "gate": (ffn, hidden), "up": (ffn, hidden), "down": (hidden, ffn)}


class LinearStack:
    """Buffers and prebuilt call arguments of one stack at a fixed token count.

    layers: one dict per layer mapping each name in MATRICES to
    (W_packed uint8 tensor, alpha float32 tensor) on the device.
    keep_all: give every layer its own output buffers (and store each layer's
    input h) so that all of them can be inspected afterwards; otherwise the
    per-layer outputs are overwritten layer after layer.
    """

    def __init__(self, layers: list, hidden: int, ffn: int, M: int, device, keep_all: bool = False):
        import torch
        self.hidden, self.ffn, self.M, self.L = hidden, ffn, M, len(layers)
        f32 = dict(dtype=torch.float32, device=device)
        self.h0 = torch.empty((M, hidden), **f32)
        self.h_final = torch.empty((M, hidden), **f32)
        sh = shapes(hidden, ffn)
        n_sets = self.L if keep_all else 1
        self.y = [{n: torch.empty((M, sh[n][0]), **f32) for n in MATRICES} for _ in range(n_sets)]
        self.h_in = [torch.empty((M, hidden), **f32) for _ in range(self.L)] if keep_all else None
        i8 = dict(dtype=torch.int8, device=device)
        self.xq = {"h": torch.empty((M, hidden), **i8), "v": torch.empty((M, hidden), **i8),
                   "up": torch.empty((M, ffn), **i8)}
        self.beta = {k: torch.empty(M, **f32) for k in self.xq}
        self.calls = []
        for l, layer in enumerate(layers):
            y = self.y[l if keep_all else 0]
            if l == 0:
                act_h = dict(a=self.h0, x_q=self.xq["h"], beta=self.beta["h"])
            else:
                yp = self.y[l - 1 if keep_all else 0]
                act_h = dict(a=yp["o"], b=yp["down"], x_q=self.xq["h"], beta=self.beta["h"])
            if keep_all:
                act_h["x_sum"] = self.h_in[l]
            fwd1 = [self._fwd(layer, n, "h", y) for n in ("q", "k", "v", "gate", "up")]
            acts2 = [dict(a=y["v"], x_q=self.xq["v"], beta=self.beta["v"]),
                     dict(a=y["up"], x_q=self.xq["up"], beta=self.beta["up"])]
            fwd2 = [self._fwd(layer, "o", "v", y), self._fwd(layer, "down", "up", y)]
            self.calls.append((bl.make_act_sum_problems([act_h]), 1, bl.make_forward_problems(fwd1), 5))
            self.calls.append((bl.make_act_sum_problems(acts2), 2, bl.make_forward_problems(fwd2), 2))
        last = self.y[-1]
        self.calls.append((bl.make_act_sum_problems([dict(a=last["o"], b=last["down"], x_sum=self.h_final,
                                                          x_q=self.xq["h"], beta=self.beta["h"])]), 1, None, 0))
        self.weight_bytes = sum(int(layer[n][0].numel()) for layer in layers for n in MATRICES)

    def _fwd(self, layer, name, src, y):
        W, alpha = layer[name]
        return dict(x_q=self.xq[src], beta=self.beta[src], W_packed=W, alpha=alpha, N=y[name].shape[1], y=y[name])

    def launches(self) -> int:
        """Kernel launches of one run when each call runs its quantisation and
        its products as separate launches (the products of a call always share
        one launch).  For at most four tokens a call may instead run as one
        fused launch, which only lowers this count."""
        return sum((1 if n_a else 0) + (1 if n_f else 0) for _, n_a, _, n_f in self.calls)

    def run(self, stream=None, flags: int = bl.BL_LINEAR_WEIGHTS_STATIC) -> None:
        """One pass of the whole stack from h0 to h_final (asynchronous)."""
        L = bl.lib()
        s = bl._stream(stream)
        for acts, n_a, fwd, n_f in self.calls:
            bl.check(L.bitlinear_linear_block(acts, n_a, fwd, n_f, flags, s), "bitlinear_linear_block")
