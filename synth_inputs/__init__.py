"""Seeded synthetic inputs for the LiteLinear forward.

This module is shared by the CUDA path's tests/benchmarks and by the CPU
oracle's tests.  It holds no arithmetic of the method itself: it only draws
random tensors with the shapes, dtypes and value distributions of the
workloads, and rounds them to the storage formats the layer consumes
(bf16 activations and factors, e4m3fn residual codes, fp32 scale).

Storage formats follow the LiteLinear README ("Features": A, B in bf16 and
Q_fp8 in e4m3fn; "Usage": bf16 activations in and out).  Shapes follow the
formula in the README introduction and the sibling SVDLinearLayer
(tt_compressor page, class SVDLinearLayer: A is (out, r), B is (r, in)):

    x [M, K] bf16,  B [r, K] bf16,  A [N, r] bf16,  Q [N, K] e4m3fn codes,
    scale [N] (per output row) or [1] (per tensor) fp32,  bias [N] bf16.

Distributions (the variance reading of N(0, s^2)):
    x ~ N(0, 1);  B ~ N(0, 1/K);  A ~ N(0, 1/r) * 0.1;
    Q = e4m3fn round-to-nearest-even of N(0, 1), clipped to +-448;
    scale = 2e-3 (or U(1e-3, 3e-3) for the attention projection);
    bias ~ N(0, 0.01), i.e. standard deviation 0.1.

Every tensor draws from its own torch.Generator, seeded from (seed, name),
so a tensor's values do not depend on which other tensors were drawn.
The encodings to bf16 and e4m3fn are torch's own dtype conversions.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import torch

SCALE_PER_TENSOR = 0
SCALE_PER_ROW = 1

_E4M3_MAX = 448.0


def _gen(seed: int, name: str) -> torch.Generator:
    h = hashlib.sha256(f"{seed}:{name}".encode()).digest()
    g = torch.Generator(device="cpu")
    g.manual_seed(int.from_bytes(h[:8], "little") & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal(shape, std: float, seed: int, name: str) -> torch.Tensor:
    t = torch.randn(*shape, generator=_gen(seed, name), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def e4m3_codes_from_float(v: torch.Tensor) -> torch.Tensor:
    """Round float values to e4m3fn (nearest even, saturating at +-448) and
    return the raw byte codes as uint8."""
    v = v.clamp(-_E4M3_MAX, _E4M3_MAX)
    return v.to(torch.float8_e4m3fn).view(torch.uint8)


@dataclasses.dataclass
class LayerInputs:
    M: int
    K: int
    N: int
    r: int
    scale_mode: int
    x: torch.Tensor            # bf16 [M, K]
    B: Optional[torch.Tensor]  # bf16 [r, K] (None when r == 0)
    A: Optional[torch.Tensor]  # bf16 [N, r] (None when r == 0)
    Q: torch.Tensor            # uint8 e4m3fn codes [N, K]
    scale: torch.Tensor        # fp32 [N] or [1]
    bias: Optional[torch.Tensor]  # bf16 [N] or None


def make_weights(K: int, N: int, r: int, *, scale_mode: int = SCALE_PER_ROW,
                 scale_value: float = 2e-3, scale_range=None, bias: bool = True,
                 seed: int = 0, q_zero: bool = False):
    """Draw (B, A, Q, scale, bias) for one layer."""
    if r > 0:
        B = _normal((r, K), 1.0 / max(K, 1) ** 0.5, seed, "B").to(torch.bfloat16)
        A = _normal((N, r), 0.1 / r ** 0.5, seed, "A").to(torch.bfloat16)
    else:
        B = A = None
    if q_zero:
        Q = torch.zeros(N, K, dtype=torch.uint8)
    else:
        Q = e4m3_codes_from_float(_normal((N, K), 1.0, seed, "Q"))
    n_scale = N if scale_mode == SCALE_PER_ROW else 1
    if scale_range is not None:
        lo, hi = scale_range
        u = torch.rand(n_scale, generator=_gen(seed, "scale"), dtype=torch.float64)
        scale = (lo + (hi - lo) * u).to(torch.float32)
    else:
        scale = torch.full((n_scale,), scale_value, dtype=torch.float32)
    b = _normal((N,), 0.1, seed, "bias").to(torch.bfloat16) if bias else None
    return B, A, Q, scale, b


def make_x(M: int, K: int, *, seed: int = 0, name: str = "x") -> torch.Tensor:
    return _normal((M, K), 1.0, seed, name).to(torch.bfloat16)


def make_inputs(M: int, K: int, N: int, r: int, **kw) -> LayerInputs:
    seed = kw.get("seed", 0)
    B, A, Q, scale, b = make_weights(K, N, r, **kw)
    x = make_x(M, K, seed=seed)
    return LayerInputs(M, K, N, r, kw.get("scale_mode", SCALE_PER_ROW),
                       x, B, A, Q, scale, b)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One named layer shape with its value distributions."""
    name: str
    M: int
    K: int
    N: int
    r: int
    scale_mode: int = SCALE_PER_ROW
    scale_value: float = 2e-3
    scale_range: Optional[tuple] = None

    def inputs(self, seed: int = 0, M: Optional[int] = None) -> LayerInputs:
        return make_inputs(self.M if M is None else M, self.K, self.N, self.r,
                           scale_mode=self.scale_mode, scale_value=self.scale_value,
                           scale_range=self.scale_range, seed=seed)

    def weights(self, seed: int = 0):
        return make_weights(self.K, self.N, self.r, scale_mode=self.scale_mode,
                            scale_value=self.scale_value,
                            scale_range=self.scale_range, seed=seed)


def _build_workloads():
    w = {}
    w["tiny_m64_k256_n256_r16"] = Workload("tiny_m64_k256_n256_r16", 64, 256, 256, 16)
    # Attention projection of a 480x704x81 video latent (15x22x11 = 3630 tokens).
    w["attn_m3630_k2048_n2048_r32"] = Workload(
        "attn_m3630_k2048_n2048_r32", 3630, 2048, 2048, 32, scale_range=(1e-3, 3e-3))
    w["ffn_up_m3630_k2048_n8192_r64"] = Workload("ffn_up_m3630_k2048_n8192_r64", 3630, 2048, 8192, 64)
    w["ffn_down_m3630_k8192_n2048_r64"] = Workload("ffn_down_m3630_k8192_n2048_r64", 3630, 8192, 2048, 64)
    for m in (1, 16, 64):
        n = f"small_m{m}_k4096_n16384_r512"
        w[n] = Workload(n, m, 4096, 16384, 512, scale_mode=SCALE_PER_TENSOR)
    for (k, n) in ((4096, 4096), (4096, 16384)):
        for m in (1024, 4096, 8192, 16384):
            for r in (32, 64, 512):
                name = f"sweep_m{m}_k{k}_n{n}_r{r}"
                w[name] = Workload(name, m, k, n, r)
    # The FFN shapes captured from LTX-Video that the LiteLinear README's
    # kernel benchmark lists ("Performance Benchmark on shapes captured from
    # LTX-Video"): w1 = up-projection, w2 = down-projection, M = flattened
    # activation rows.  The page states neither K / N nor the rank; the
    # shapes here take the README's own usage example (in_features 4096,
    # out_features 16384) for the up-projection and its transpose for the
    # down-projection, at ranks 32 and 64.
    for cfg, m, _count in PAGE_MICROBENCH:
        k, n = (4096, 16384) if cfg == "w1" else (16384, 4096)
        for r in (32, 64):
            name = f"page_{cfg}_m{m}_k{k}_n{n}_r{r}"
            w[name] = Workload(name, m, k, n, r)
    return w


# (projection, M, call count) of the README's LTX-Video benchmark table, in
# its row order; the count-weighted total over these rows is its TOTAL row.
PAGE_MICROBENCH = (
    ("w2", 1400, 336), ("w1", 1400, 336), ("w2", 2450, 336), ("w1", 2450, 336),
    ("w2", 5600, 480), ("w1", 5600, 480), ("w2", 9800, 144), ("w1", 9800, 144),
    ("w2", 10850, 336), ("w1", 10850, 336), ("w2", 22400, 144), ("w1", 22400, 144),
    ("w2", 43400, 144), ("w1", 43400, 144),
)


def page_workload(cfg: str, m: int, r: int) -> str:
    k, n = (4096, 16384) if cfg == "w1" else (16384, 4096)
    return f"page_{cfg}_m{m}_k{k}_n{n}_r{r}"


WORKLOADS = _build_workloads()

# Groups of workloads that are timed together (the FFN pair is summed).
FFN_PAIR = ("ffn_up_m3630_k2048_n8192_r64", "ffn_down_m3630_k8192_n2048_r64")
SMALL_BATCH = ("small_m1_k4096_n16384_r512", "small_m16_k4096_n16384_r512",
               "small_m64_k4096_n16384_r512")


def to_numpy_bits(t: Optional[torch.Tensor]):
    """Raw storage bits of a CPU tensor as a contiguous numpy array
    (bf16 -> uint16, uint8 -> uint8, fp32 -> float32)."""
    if t is None:
        return None
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()
