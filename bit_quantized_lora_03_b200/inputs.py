"""Seeded synthetic inputs for the QLoRA NF4 linear path.

This module only draws random tensors with fixed seeds and shapes. It contains none of the
method's arithmetic (no quantization, no products), so both the CUDA library's tests and
the CPU oracle can be fed from it without sharing any of the computation under test.

All draws use ``torch.Generator('cpu')`` and ``torch.randn``; fp32 values are scaled by one
fp32 multiply; bf16 tensors are the round-to-nearest-even cast of an fp32 draw, so the
same bits go to the oracle and to the GPU.

Workloads (weights are Gaussian stand-ins with LLaMA shapes; there are no real weights
here). W is the method's h x o matrix; it is drawn and stored transposed as Wt (o x h,
"out x in"), which is the layout the library quantizes.
"""

from __future__ import annotations

import dataclasses

import torch

W_SIGMA = 0.02          # N(0, 0.02) weights
ADAPTER_SIGMA = 0.01    # N(0, 0.01) adapters
OUTLIER_FRACTION = 0.01
OUTLIER_SIGMAS = 8.0

# The seven linears of one LLaMA-7B-shaped decoder layer, as (name, h = in, o = out).
LLAMA7B_LINEARS = (
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 4096, 11008), ("up_proj", 4096, 11008),
    ("down_proj", 11008, 4096),
)

# The seven linears of one LLaMA-65B-shaped decoder layer (h = 8192, FFN 22016).
LLAMA65B_LINEARS = (
    ("q_proj", 8192, 8192), ("k_proj", 8192, 8192), ("v_proj", 8192, 8192),
    ("o_proj", 8192, 8192), ("gate_proj", 8192, 22016), ("up_proj", 8192, 22016),
    ("down_proj", 22016, 8192),
)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator("cpu")
    g.manual_seed(int(seed))
    return g


def normal_f32(shape, sigma: float, g: torch.Generator) -> torch.Tensor:
    """N(0, sigma) fp32: a standard normal draw times fp32(sigma)."""
    return torch.randn(*shape, generator=g, dtype=torch.float32) * torch.tensor(
        sigma, dtype=torch.float32)


def normal_bf16(shape, sigma: float, g: torch.Generator) -> torch.Tensor:
    """N(0, sigma) rounded to bf16 (round to nearest even)."""
    return normal_f32(shape, sigma, g).to(torch.bfloat16)


def weight_f32(o: int, h: int, seed: int, outliers: bool = False) -> torch.Tensor:
    """Wt (o x h fp32) ~ N(0, 0.02); optionally exactly 1% of positions set to +-8 sigma.

    Outlier positions come from a seeded ``randperm`` and their signs from a seeded draw,
    both after the Gaussian draw from the same generator.
    """
    g = _gen(seed)
    w = normal_f32((o, h), W_SIGMA, g)
    if outliers:
        n = o * h
        k = int(n * OUTLIER_FRACTION)
        pos = torch.randperm(n, generator=g)[:k]
        sign = torch.randint(0, 2, (k,), generator=g, dtype=torch.int64) * 2 - 1
        mag = torch.tensor(OUTLIER_SIGMAS * W_SIGMA, dtype=torch.float32)
        w.view(-1)[pos] = sign.to(torch.float32) * mag
    return w


@dataclasses.dataclass
class LinearInputs:
    """One adapted linear: Wt (o x h fp32), X (t x h bf16), L1 (h x r), L2 (r x o), s,
    and an upstream gradient dY (t x o bf16) when a backward is part of the workload."""
    name: str
    Wt: torch.Tensor
    X: torch.Tensor
    L1: torch.Tensor
    L2: torch.Tensor
    s: float
    dY: torch.Tensor | None = None

    @property
    def t(self) -> int:
        return self.X.shape[0]

    @property
    def h(self) -> int:
        return self.Wt.shape[1]

    @property
    def o(self) -> int:
        return self.Wt.shape[0]

    @property
    def r(self) -> int:
        return self.L1.shape[1]


def single_linear_1024(seed: int = 0) -> LinearInputs:
    """Single QLoRA linear forward: W 1024 x 1024 N(0,0.02); X 16 x 1024 N(0,1); L1 1024 x 16
    and L2 16 x 1024 N(0,0.01); s = 2. One generator, drawn in the order W, X, L1, L2."""
    g = _gen(seed)
    Wt = normal_f32((1024, 1024), W_SIGMA, g)
    X = normal_bf16((16, 1024), 1.0, g)
    L1 = normal_bf16((1024, 16), ADAPTER_SIGMA, g)
    L2 = normal_bf16((16, 1024), ADAPTER_SIGMA, g)
    return LinearInputs("single_linear_1024", Wt, X, L1, L2, 2.0)


def llama7b_quant_weights(with_outliers: bool = True):
    """The seven fp32 weights of one LLaMA-7B-shaped layer, seeds 200 + i, with 1% outliers
    at +-8 sigma. Yields (name, Wt)."""
    for i, (name, h, o) in enumerate(LLAMA7B_LINEARS):
        yield name, weight_f32(o, h, 200 + i, outliers=with_outliers)


def decode_gemv_weights():
    """The two decode-shape weights: (h, o) = (4096, 11008) seed 300, (8192, 28672) seed 301."""
    return [("w_4096x11008", weight_f32(11008, 4096, 300)),
            ("w_8192x28672", weight_f32(28672, 8192, 301))]


def decode_gemv_activations(h: int, t: int) -> torch.Tensor:
    """X (t x h bf16) ~ N(0,1), seed 310 + t."""
    return normal_bf16((t, h), 1.0, _gen(310 + t))


def decode_gemv_adapters(h: int, o: int, r: int = 16):
    """L1 (h x r), L2 (r x o) bf16 ~ N(0, 0.01), seed 320."""
    g = _gen(320)
    return normal_bf16((h, r), ADAPTER_SIGMA, g), normal_bf16((r, o), ADAPTER_SIGMA, g)


def training_linear(i: int, t: int = 4096, r: int = 64, s: float = 0.25,
                    shapes=LLAMA7B_LINEARS, seed_base: int = 400) -> LinearInputs:
    """Linear i of the training-shape workload: Wt seed base + i (no outliers); X (t x h)
    N(0,1) seed base + 10 + i; dY (t x o) N(0,1) seed base + 20 + i; L1, L2 N(0, 0.01)
    seed base + 30 + i."""
    name, h, o = shapes[i]
    Wt = weight_f32(o, h, seed_base + i)
    X = normal_bf16((t, h), 1.0, _gen(seed_base + 10 + i))
    dY = normal_bf16((t, o), 1.0, _gen(seed_base + 20 + i))
    ga = _gen(seed_base + 30 + i)
    L1 = normal_bf16((h, r), ADAPTER_SIGMA, ga)
    L2 = normal_bf16((r, o), ADAPTER_SIGMA, ga)
    return LinearInputs(name, Wt, X, L1, L2, s, dY)


def random_linear(t: int, h: int, o: int, r: int, s: float, seed: int,
                  with_grad: bool = True) -> LinearInputs:
    """A generic seeded linear of any shape (test cases with ragged sizes)."""
    g = _gen(seed)
    Wt = normal_f32((o, h), W_SIGMA, g)
    X = normal_bf16((t, h), 1.0, g)
    L1 = normal_bf16((h, r), ADAPTER_SIGMA, g)
    L2 = normal_bf16((r, o), ADAPTER_SIGMA, g)
    dY = normal_bf16((t, o), 1.0, g) if with_grad else None
    return LinearInputs(f"random_t{t}_h{h}_o{o}_r{r}", Wt, X, L1, L2, s, dY)


# ------------------------------------------------------------------------------------------
# The 65B-shaped stack: 80 layers x the 7 linears of LLAMA65B_LINEARS, 2048 tokens, r = 64,
# s = 0.25. Its 64.76 G weights are drawn on the device (a CPU draw of that size is too slow):
# torch's CUDA generator, seeded 500 + 7 layer + i for the weight of linear i of a layer and
# 100000 + 7 layer + i for its adapters (L1 then L2), N(0,0.02) and N(0,0.01) as elsewhere.
# Every layer's linears read shared seeded inputs and upstream gradients (CPU generator):
# X (t x 8192) seed 510 for the six linears with 8192 inputs, X (t x 22016) seed 511 for
# down_proj; dY (t x 8192) seed 520 for the outputs of width 8192, dY (t x 22016) seed 521.
# ------------------------------------------------------------------------------------------
STACK65B_LAYERS = 80
STACK65B_TOKENS = 2048
STACK65B_RANK = 64
STACK65B_S = 0.25


def _device_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def stack65b_weight(layer: int, i: int, device) -> torch.Tensor:
    """Wt (o x h fp32, on `device`) of linear i of `layer`: N(0, 0.02), seed 500 + 7 layer + i."""
    _, h, o = LLAMA65B_LINEARS[i]
    g = _device_gen(500 + 7 * layer + i, device)
    return torch.randn(o, h, generator=g, dtype=torch.float32, device=device) * torch.tensor(
        W_SIGMA, dtype=torch.float32, device=device)


def stack65b_adapters(layer: int, i: int, device, r: int = STACK65B_RANK):
    """(L1 h x r, L2 r x o) bf16 on `device`: N(0, 0.01), seed 100000 + 7 layer + i."""
    _, h, o = LLAMA65B_LINEARS[i]
    g = _device_gen(100000 + 7 * layer + i, device)
    sig = torch.tensor(ADAPTER_SIGMA, dtype=torch.float32, device=device)
    L1 = (torch.randn(h, r, generator=g, dtype=torch.float32, device=device) * sig).to(torch.bfloat16)
    L2 = (torch.randn(r, o, generator=g, dtype=torch.float32, device=device) * sig).to(torch.bfloat16)
    return L1, L2


def stack65b_activations(t: int = STACK65B_TOKENS):
    """Shared inputs and upstream gradients: {8192: X, 22016: X} and {8192: dY, 22016: dY},
    bf16 N(0,1) on the CPU."""
    X = {8192: normal_bf16((t, 8192), 1.0, _gen(510)), 22016: normal_bf16((t, 22016), 1.0, _gen(511))}
    dY = {8192: normal_bf16((t, 8192), 1.0, _gen(520)), 22016: normal_bf16((t, 22016), 1.0, _gen(521))}
    return X, dY
