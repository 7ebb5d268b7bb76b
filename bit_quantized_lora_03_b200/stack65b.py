"""The 65B-shaped linear stack, resident on one GPU: 80 layers x 7 NF4 linears (h = 8192,
FFN 22016; 64.76 G weights, 33.4 GB packed), LoRA r = 64 on every linear, 2048 tokens.

Only the linear path is run: attention and norms are identity, and every layer's linears read
the same seeded inputs and upstream gradients (``inputs.stack65b_activations``). A chained
residual stream through identity attention would multiply the activations by about 6 per
layer with N(0, 0.02) weights and overflow bf16 before layer 50; the kernels, sizes and launch
order are the same either way. A step is the forward and backward of all 560 linears, each
through ``qlora_linear_fwd`` / ``qlora_linear_bwd``, the independent linears spread
round-robin over two streams. Weights are drawn and quantized on the device one linear at a
time, so the fp32 copy never exceeds one linear (721 MB).
"""

from __future__ import annotations

import torch

from . import binding as B
from . import inputs


class Stack65B:
    def __init__(self, device, layers: int = inputs.STACK65B_LAYERS, t: int = inputs.STACK65B_TOKENS,
                 r: int = inputs.STACK65B_RANK, s: float = inputs.STACK65B_S, streams: int = 2):
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
        # outputs nothing reads back go to per-shape scratch buffers, one set per stream
        self.streams = [torch.cuda.Stream(device) for _ in range(streams)] if streams > 1 else []
        self.scratch = []
        for _ in range(max(1, streams)):
            self.scratch.append({
                "Y": {n: torch.empty(t, n, dtype=torch.bfloat16, device=device) for n in (8192, 22016)},
                "dX": {n: torch.empty(t, n, dtype=torch.bfloat16, device=device) for n in (8192, 22016)},
                "wsf": torch.empty(wsf, dtype=torch.uint8, device=device),
                "wsb": torch.empty(wsb, dtype=torch.uint8, device=device)})
        torch.cuda.synchronize(device)

    @property
    def packed_bytes(self) -> int:
        return sum(e[4].nbytes for e in self.lin)

    def flops_per_step(self) -> int:
        """Algorithmic flops of one fwd+bwd: 4 t h o + 6 t r (h + o) per linear (no dW)."""
        return sum(4 * self.t * h * o + 6 * self.t * self.r * (h + o) for _, _, h, o, *_ in self.lin)

    def step(self, keep=None):
        """Forward and backward of every linear, round-robin over the streams (the linears are
        independent; each stream has its own scratch outputs and workspaces). `keep` (a set of
        (layer, i)) returns copies of those linears' Y and dX, taken right after each is
        written."""
        kept = {}
        cur = torch.cuda.current_stream(self.dev)
        if self.streams:
            go = torch.cuda.Event()
            go.record(cur)
            for st in self.streams:
                st.wait_event(go)
        for n, (layer, i, h, o, p, L1, L2, sT, dL1, dL2) in enumerate(self.lin):
            k = n % len(self.streams) if self.streams else 0
            sc = self.scratch[k]
            with torch.cuda.stream(self.streams[k] if self.streams else cur):
                X, dY, Y, dX = self.X[h], self.dY[o], sc["Y"][o], sc["dX"][h]
                B.qlora_linear_fwd(X, p, L1, L2, self.s, Y=Y, sT=sT, ws=sc["wsf"])
                if keep and (layer, i) in keep:
                    kept[(layer, i, "Y")] = Y.clone()
                B.qlora_linear_bwd(dY, X, p, L1, L2, self.s, sT=sT, dX=dX, dL1=dL1, dL2=dL2,
                                   ws=sc["wsb"])
                if keep and (layer, i) in keep:
                    kept[(layer, i, "dX")] = dX.clone()
        for st in self.streams:
            done = torch.cuda.Event()
            done.record(st)
            cur.wait_event(done)
        return kept

    def linear(self, layer: int, i: int):
        return self.lin[layer * len(inputs.LLAMA65B_LINEARS) + i]
