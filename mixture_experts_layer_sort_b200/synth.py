"""Seeded synthetic inputs for the fused MoE layer.

Holds none of the layer's arithmetic: it only draws random tensors with the
shapes and distributions of the workloads (decode and prefill shapes of a
large MoE model), so that the CUDA path and the CPU oracle can be fed the very
same numbers. Nothing here routes, permutes, quantises or multiplies.

Recipe (every tensor is drawn in fp32 from its own generator and rounded to
its storage type):
  x       [M, H]   N(0, 1)                       -> bf16, seed = base
  logits  [M, E]   N(0, 1) (+ a per-expert bias)  fp32, seed = base + 1
  W_gate  [E, I, H], W_up [E, I, H], W_down [E, H, I]
          N(0, std) per expert, seed = base * 1_000_003 + 3e + {2, 3, 4} -> bf16
The skewed workload adds bias_e = -s * ln(e + 1) to every token's logits, the
log of a Zipf(s) law over expert ranks (rank = id + 1), so low ids are hot.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    E: int
    k: int
    H: int
    I: int
    Ms: tuple
    w_std: float
    zipf_s: float = 0.0
    dtypes: tuple = ("bf16",)
    description: str = ""


WORKLOADS = {
    "tiny": Workload("tiny", E=8, k=2, H=256, I=512, Ms=(16,), w_std=0.02,
                     description="tiny bf16 layer, E=8 top-2, H=256, I=512, M=16"),
    "decode": Workload("decode", E=128, k=8, H=2048, I=768, Ms=(1, 4, 16, 64), w_std=0.02,
                       description="decode bf16, E=128 top-8, H=2048, I=768 (1.2 GB of expert weights)"),
    "decode_fp8": Workload("decode_fp8", E=128, k=8, H=2048, I=768, Ms=(1, 8, 32, 64), w_std=0.02,
                           dtypes=("fp8",),
                           description="decode e4m3, E=128 top-8, H=2048, I=768, per-tensor scales"),
    "decode_e5m2": Workload("decode_e5m2", E=128, k=8, H=2048, I=768, Ms=(1, 8, 32, 64), w_std=0.02,
                            dtypes=("fp8_e5m2",),
                            description="decode e5m2, E=128 top-8, H=2048, I=768, per-tensor scales"),
    "large_decode": Workload("large_decode", E=256, k=8, H=7168, I=2048, Ms=(1, 32, 64, 128),
                             w_std=0.01, zipf_s=1.1,
                             description="large decode bf16, E=256 top-8, H=7168, I=2048, "
                                         "Zipf(1.1)-skewed router (22.5 GB of expert weights)"),
    "prefill": Workload("prefill", E=256, k=8, H=7168, I=2048, Ms=(4096,), w_std=0.01,
                        dtypes=("bf16", "fp8"),
                        description="prefill, E=256 top-8, H=7168, I=2048, M=4096, bf16 and e4m3"),
    # a supplementary compute-heavier point: the prefill layer at 4x the tokens (~512 per
    # expert, two 256-row token blocks each), where the FLOPs (11.5 TFLOP) outweigh the
    # weight bytes at the measured peaks
    "prefill_m16384": Workload("prefill_m16384", E=256, k=8, H=7168, I=2048, Ms=(16384,), w_std=0.01,
                               description="prefill at M=16384 (compute-bound point), E=256 top-8, H=7168, I=2048"),
    # profiling stand-in for prefill: same H, I and tokens per expert (~128) and the same
    # schedule (no split-K), 3/16 of the experts, so a multi-pass profiler capture holds
    # ~4 GB instead of 23 GB
    "prefill_e48": Workload("prefill_e48", E=48, k=8, H=7168, I=2048, Ms=(768,), w_std=0.01,
                            dtypes=("bf16", "fp8"),
                            description="prefill-shaped profiling case, E=48 top-8, H=7168, I=2048, M=768"),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    return g


def make_tokens(E: int, H: int, M: int, seed: int = 0, device="cpu", zipf_s: float = 0.0):
    """x [M, H] bf16 and router logits [M, E] fp32."""
    x = torch.randn((M, H), generator=_gen(seed, device), device=device,
                    dtype=torch.float32).to(torch.bfloat16)
    logits = torch.randn((M, E), generator=_gen(seed + 1, device), device=device,
                         dtype=torch.float32)
    if zipf_s:
        bias = torch.tensor([-zipf_s * math.log(e + 1.0) for e in range(E)],
                            dtype=torch.float32, device=device)
        logits = logits + bias
    return x, logits


def expert_seed(seed: int, e: int, which: int) -> int:
    return seed * 1_000_003 + 3 * e + 2 + which


def make_expert(E_index: int, H: int, I: int, w_std: float, seed: int = 0, device="cpu"):
    """(W_gate[e] [I,H], W_up[e] [I,H], W_down[e] [H,I]) bf16 of one expert."""
    out = []
    for which, shape in enumerate(((I, H), (I, H), (H, I))):
        g = _gen(expert_seed(seed, E_index, which), device)
        w = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * w_std
        out.append(w.to(torch.bfloat16))
    return tuple(out)


def make_weights(E: int, H: int, I: int, w_std: float, seed: int = 0, device="cpu"):
    """Stacked bf16 weights W_gate [E,I,H], W_up [E,I,H], W_down [E,H,I], drawn per expert."""
    wg = torch.empty((E, I, H), dtype=torch.bfloat16, device=device)
    wu = torch.empty((E, I, H), dtype=torch.bfloat16, device=device)
    wd = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
    for e in range(E):
        g, u, d = make_expert(e, H, I, w_std, seed, device)
        wg[e].copy_(g)
        wu[e].copy_(u)
        wd[e].copy_(d)
    return wg, wu, wd


def bf16_to_f32_numpy(t: torch.Tensor):
    """Exact widening of a bf16 tensor to a float32 numpy array (host copy)."""
    return t.detach().to("cpu").to(torch.float32).numpy()
