"""Seeded synthetic inputs for the OPQ weight-quantization hot path.

This module only draws random tensors with the shapes and value
distributions of diffusion-transformer linear layers. It contains none of
the quantization arithmetic, so both the CPU oracle (``oracle/``) and the
CUDA library can be fed from it without sharing any of the method.

Distributions (all values are rounded once, fp32 -> bf16, round-to-nearest-even):

* ``student_t4``: Student-t with 4 degrees of freedom, t = Z / sqrt(chi2_4 / 4)
  with chi2_4 = -2 ln(U1 U2), rescaled by std / sqrt(2) (the variance of t_4
  is 2), so the weights have standard deviation ``std``.
* ``normal``: N(0, std^2).
* outlier rows: ``round(frac * N)`` rows chosen by the generator each get one
  column set to +-8*std (random sign), the "0.1% of rows holding a +-8 sigma
  outlier" of the attention-projection workload.

Seeds: the tiny case draws W then x from one generator seeded 0; every other
workload seeds each tensor separately with ``1000 * case + tensor_index``;
the whole-model pass seeds layer j of block b with ``5000 + 7 * b + j``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

WEIGHT_STD = 0.02
ALPHA = 0.73


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return (z * std).to(torch.bfloat16)


def student_t4(shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    u1 = torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
    u2 = torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
    # U in (0, 1]: torch.rand draws from [0, 1); flip so log() never sees 0.
    u1 = 1.0 - u1
    u2 = 1.0 - u2
    chi2 = -2.0 * torch.log(u1 * u2)
    t = z / torch.sqrt(chi2 / 4.0)
    return (t * (std / math.sqrt(2.0))).to(torch.bfloat16)


def random_planes(N: int, K: int, seed: int):
    """Packed planes of random bits for an N x K weight, as numpy arrays: codes uint32 [N, K/8]
    (any nibble is a valid level), signs uint32 [N, K/32] and positive fp32 row maxima [N] in
    [0.01, 0.1). Inputs for the linear at sizes where quantizing a weight first would take the
    oracle too long; nothing of the method is computed here."""
    import numpy as np
    rng = np.random.default_rng(int(seed))
    codes = rng.integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint32)
    signs = rng.integers(0, 1 << 32, size=(N, K // 32), dtype=np.uint32)
    scales = (0.01 + 0.09 * rng.random(N)).astype(np.float32)
    return codes, signs, scales


def random_gmax(N: int, groups: int, seed: int):
    """float16 group maxima [N, groups] in [0.01, 0.1), as their uint16 bit patterns (numpy): with
    random_planes, the group-wise format's inputs for the linear at the largest sizes."""
    import numpy as np
    rng = np.random.default_rng(int(seed))
    return (0.01 + 0.09 * rng.random((N, groups))).astype(np.float16).view(np.uint16)


def add_outlier_rows(w: torch.Tensor, frac: float, std: float, gen: torch.Generator) -> torch.Tensor:
    n, k = w.shape
    count = int(round(frac * n))
    if count == 0:
        return w
    dev = w.device
    rows = torch.randperm(n, generator=gen, device=dev)[:count]
    cols = torch.randint(0, k, (count,), generator=gen, device=dev)
    sgn = torch.randint(0, 2, (count,), generator=gen, device=dev).to(torch.float32) * 2.0 - 1.0
    w = w.clone()
    w[rows, cols] = (sgn * 8.0 * std).to(torch.bfloat16)
    return w


@dataclass
class Linear:
    """One x[M,K] @ W[N,K]^T problem with its seeds."""
    name: str
    M: int
    N: int
    K: int
    alpha: float = ALPHA
    w_seed: int = 0
    x_seed: int = 1
    w_dist: str = "student_t4"
    outlier_frac: float = 0.0
    shared_seed: bool = False  # tiny case: W then x from one generator

    def make(self, device="cpu"):
        """Return (x bf16 [M,K], W bf16 [N,K]) on ``device``."""
        if self.shared_seed:
            g = _gen(self.w_seed, device)
            w = self._weights(g, device)
            x = normal((self.M, self.K), 1.0, g, device)
            return x, w
        gw = _gen(self.w_seed, device)
        w = self._weights(gw, device)
        gx = _gen(self.x_seed, device)
        x = normal((self.M, self.K), 1.0, gx, device)
        return x, w

    def make_weights(self, device="cpu"):
        if self.shared_seed:
            return self.make(device)[1]
        return self._weights(_gen(self.w_seed, device), device)

    def make_x(self, device="cpu"):
        if self.shared_seed:
            return self.make(device)[0]
        return normal((self.M, self.K), 1.0, _gen(self.x_seed, device), device)

    def _weights(self, g, device):
        shape = (self.N, self.K)
        if self.w_dist == "normal":
            w = normal(shape, WEIGHT_STD, g, device)
        else:
            w = student_t4(shape, WEIGHT_STD, g, device)
        if self.outlier_frac > 0:
            w = add_outlier_rows(w, self.outlier_frac, WEIGHT_STD, g)
        return w

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


def tiny() -> Linear:
    """W 256x512 N(0, 0.02^2) and x 64x512 N(0,1), one generator seeded 0."""
    return Linear("tiny_256x512_m64", 64, 256, 512, w_dist="normal", w_seed=0, shared_seed=True)


def dit_attn_proj() -> Linear:
    """x 3072x3840 (48x64 latent patches of a 768x1024 image), W 3840x3840 t4 + outlier rows."""
    return Linear("dit_attn_proj_3072x3840x3840", 3072, 3840, 3840, w_seed=2000, x_seed=2001,
                  outlier_frac=0.001)


def dit_ffn_pair(alpha: float = ALPHA):
    """x 4096x3840 through W1 10240x3840; x' 4096x10240 through W2 3840x10240."""
    up = Linear(f"dit_ffn_up_4096x10240x3840_a{alpha}", 4096, 10240, 3840, alpha=alpha,
                w_seed=3000, x_seed=3001)
    down = Linear(f"dit_ffn_down_4096x3840x10240_a{alpha}", 4096, 3840, 10240, alpha=alpha,
                  w_seed=3002, x_seed=3003)
    return up, down


def small_m(M: int) -> Linear:
    """x Mx3840 against the fused-QKV weight 11520x3840 (weight-streaming regime)."""
    return Linear(f"qkv_small_m{M}_11520x3840", M, 11520, 3840, w_seed=4000, x_seed=4001 + M)


SMALL_M_SWEEP = (1, 16, 64, 256)


@dataclass
class WholeModel:
    """30 DiT blocks: 4 attention matrices 3840x3840, W1 and W3 10240x3840, W2 3840x10240.

    The listed "3 x (10240x3840)" FFN matrices are read as a SwiGLU FFN (two
    up-projections plus one down-projection); the parameter count, bytes and
    flops are identical to the literal reading.
    """
    blocks: int = 30
    M: int = 3072
    alpha: float = ALPHA
    layers: list = field(default_factory=list)

    def __post_init__(self):
        if not self.layers:
            shapes = [(3840, 3840)] * 4 + [(10240, 3840), (10240, 3840), (3840, 10240)]
            for b in range(self.blocks):
                for j, (n, k) in enumerate(shapes):
                    self.layers.append(Linear(f"block{b}_layer{j}", self.M, n, k, alpha=self.alpha,
                                              w_seed=5000 + 7 * b + j, x_seed=900000 + 7 * b + j))

    @property
    def weights(self) -> int:
        return sum(l.N * l.K for l in self.layers)
