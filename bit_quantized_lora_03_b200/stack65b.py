"""The 65B-shaped linear stack, resident on one GPU: 80 layers x 7 NF4 linears (h = 8192,
FFN 22016; 64.76 G weights, 33.4 GB packed), LoRA r = 64 on every linear, 2048 tokens.

Only the linear path is run: attention and norms are identity, and every layer's linears read
the same seeded inputs and upstream gradients (``inputs.stack65b_activations``). A chained
residual stream through identity attention would multiply the activations by about 6 per
layer with N(0, 0.02) weights and overflow bf16 before layer 50; the kernels, sizes and launch
order are the same either way. A step is the forward and backward of all 560 linears, each
through ``qlora_linear_fwd`` / ``qlora_linear_bwd``. Weights are drawn and quantized on the
device one linear at a time, so the fp32 copy never exceeds one linear (721 MB).
"""

from __future__ import annotations

import torch

from . import binding as B
from . import inputs


class Stack65B:
    def __init__(self, device, layers: int = inputs.STACK65B_LAYERS, t: int = inputs.STACK65B_TOKENS,
                 r: int = inputs.STACK65B_RANK, s: float = inputs.STACK65B_S):
        self.dev, self.t, self.r, self.s, self.layers = device, t, r, s, layers
        X, dY = inputs.stack65b_activations(t)
        self.X = {k: v.to(device) for k, v in X.items()}
        self.dY = {k: v.to(device) for k, v in dY.items()}
        self.lin = []   # per linear: (layer, i, h, o, packed W, L1, L2, sT, dL1, dL2)
        wsf = wsb = 0
        for layer in range(layers):
            for i, (_, h, o) in enumerate(inputs.LLAMA65B_LINEARS):
                Wt = inputs.stack65b_weight(layer, i, device)
                p = B.nf4_quantize(Wt)
                del Wt
                L1, L2 = inputs.stack65b_adapters(layer, i, device, r)
                sT = torch.empty(t, r, dtype=torch.bfloat16, device=device)
                dL1 = torch.empty(h, r, dtype=torch.float32, device=device)
                dL2 = torch.empty(r, o, dtype=torch.float32, device=device)
                self.lin.append((layer, i, h, o, p, L1, L2, sT, dL1, dL2))
                wsf = max(wsf, B.fwd_workspace_bytes(t, h, o, r))
                wsb = max(wsb, B.bwd_workspace_bytes(t, h, o, r))
        # outputs nothing reads back are written to per-shape scratch buffers
        self.Y = {n: torch.empty(t, n, dtype=torch.bfloat16, device=device) for n in (8192, 22016)}
        self.dX = {n: torch.empty(t, n, dtype=torch.bfloat16, device=device) for n in (8192, 22016)}
        self.wsf = torch.empty(wsf, dtype=torch.uint8, device=device)
        self.wsb = torch.empty(wsb, dtype=torch.uint8, device=device)
        torch.cuda.synchronize(device)

    @property
    def packed_bytes(self) -> int:
        return sum(e[4].nbytes for e in self.lin)

    def flops_per_step(self) -> int:
        """Algorithmic flops of one fwd+bwd: 4 t h o + 6 t r (h + o) per linear (no dW)."""
        return sum(4 * self.t * h * o + 6 * self.t * self.r * (h + o) for _, _, h, o, *_ in self.lin)

    def step(self, keep=None):
        """Forward and backward of every linear. `keep` (a set of (layer, i)) returns copies
        of those linears' Y and dX, taken right after each is written."""
        kept = {}
        for layer, i, h, o, p, L1, L2, sT, dL1, dL2 in self.lin:
            X, dY, Y, dX = self.X[h], self.dY[o], self.Y[o], self.dX[h]
            B.qlora_linear_fwd(X, p, L1, L2, self.s, Y=Y, sT=sT, ws=self.wsf)
            if keep and (layer, i) in keep:
                kept[(layer, i, "Y")] = Y.clone()
            B.qlora_linear_bwd(dY, X, p, L1, L2, self.s, sT=sT, dX=dX, dL1=dL1, dL2=dL2,
                               ws=self.wsb)
            if keep and (layer, i) in keep:
                kept[(layer, i, "dX")] = dX.clone()
        return kept

    def linear(self, layer: int, i: int):
        return self.lin[layer * len(inputs.LLAMA65B_LINEARS) + i]
