"""Seeded synthetic activation streams (shared by the CUDA path's tests, the
benchmark and the oracle's tests).

This module holds none of the compression arithmetic: it only draws the
per-step activations a_0, a_1, ... that a parallel diffusion model would
exchange.  No model weights or datasets are used; the shapes and statistics
stand in for the workloads named in "Accelerating Parallel Diffusion Model
Serving with Residual Compression" (experiments: FLUX.1-dev main table,
CogVideoX-2b finding):

* tiny      -- 256 x 64 fp32, a_0 ~ N(0,1), a_t = a_{t-1} + 0.1 N(0,1)
* flux      -- 4608 x 3072 bf16 (4096 image + 512 text tokens), a_0 ~ N(0,1)
               with ceil(1% of cols) outlier channels scaled x20, random walk
               a_t = a_{t-1} + 0.1 s_c N(0,1) (s_c the channel scale, so the
               residual-to-activation ratio is 0.1 in every channel)
* ar1       -- 4096 x 3072 bf16, stationary AR(1) a_t = rho a_{t-1} +
               0.1 N(0,1), rho = sqrt(0.99): sigma_delta / sigma_a = 0.1 with
               an i.i.d. (high-rank) Gaussian innovation
* cogvideox -- 60 tensors (30 layers x 2) of 17550 x 1920 bf16, per-tensor
               residual ratio drawn U[0.05, 0.2]
* lowrank_walk -- a random walk whose innovation is dominated by a fixed
               rank-k structure with a decaying spectrum, plus a small i.i.d.
               part: a residual whose leading subspace is well separated

Rows are tokens, columns are channels (the hidden dimension).  The walk state
is kept in fp32 and cast to the stream dtype each step.
"""
from __future__ import annotations

import math

import torch

__all__ = ["ActivationStream", "LowRankWalk", "tiny", "flux", "ar1", "cogvideox", "lowrank_walk"]


class ActivationStream:
    """A seeded stream of ``batch`` activation tensors of shape (rows, cols).

    ``next()`` returns the next step's activations as one tensor of shape
    (batch, rows, cols) in ``dtype`` on ``device``.
    """

    def __init__(self, rows, cols, *, batch=1, dtype=torch.bfloat16, device="cpu", seed=0,
                 sigma=0.1, rho=1.0, outlier_frac=0.0, outlier_scale=20.0, sigma_per_tensor=None,
                 seed_per_tensor=None):
        self.rows, self.cols, self.batch = int(rows), int(cols), int(batch)
        self.dtype, self.device = dtype, torch.device(device)
        self.rho = float(rho)
        gdev = "cuda" if self.device.type == "cuda" else "cpu"
        if seed_per_tensor is None:
            seed_per_tensor = [seed + 7919 * b for b in range(self.batch)]
        self.gens = [torch.Generator(device=gdev).manual_seed(int(s)) for s in seed_per_tensor]
        # per-channel scale (outlier channels), chosen on the CPU so it is device independent
        col_scale = torch.ones(self.cols, dtype=torch.float32)
        n_out = math.ceil(outlier_frac * self.cols) if outlier_frac > 0 else 0
        if n_out:
            perm = torch.randperm(self.cols, generator=torch.Generator().manual_seed(int(seed)))
            col_scale[perm[:n_out]] = outlier_scale
        self.col_scale = col_scale.to(self.device)
        self.outlier_cols = sorted(int(c) for c in torch.nonzero(col_scale != 1.0).flatten())
        sig = sigma_per_tensor if sigma_per_tensor is not None else [sigma] * self.batch
        self.sigmas = [float(s) for s in sig]
        self.state = torch.empty(self.batch, self.rows, self.cols, dtype=torch.float32, device=self.device)
        self.t = 0

    def _normal(self, b):
        return torch.randn(self.rows, self.cols, generator=self.gens[b], device=self.device,
                           dtype=torch.float32)

    def next(self, out: torch.Tensor | None = None) -> torch.Tensor:
        for b in range(self.batch):
            z = self._normal(b)
            if self.t == 0:
                self.state[b] = z * self.col_scale
            else:
                if self.rho != 1.0:
                    self.state[b].mul_(self.rho)
                self.state[b].add_(z * (self.sigmas[b] * self.col_scale))
        self.t += 1
        if out is None:
            return self.state.to(self.dtype, copy=True)
        out.copy_(self.state)
        return out


class BlockStream(ActivationStream):
    """A random walk whose innovation scale is constant within each b x b block
    of an H x W token grid (rows = H*W, raster order) and log-uniform over
    blocks in [lo, hi]: the changes between steps concentrate in a few regions."""

    def __init__(self, H, W, cols, *, block=8, lo=0.01, hi=0.3, dtype=torch.bfloat16, device="cpu", seed=0):
        super().__init__(H * W, cols, dtype=dtype, device=device, seed=seed, sigma=1.0, seed_per_tensor=[seed])
        g = torch.Generator().manual_seed(int(seed) + 1)
        K = (H // block) * (W // block)
        u = torch.rand(K, generator=g, dtype=torch.float64)
        scale = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).to(torch.float32)
        grid = scale.reshape(H // block, W // block).repeat_interleave(block, 0).repeat_interleave(block, 1)
        self.row_scale = grid.reshape(H * W, 1).to(self.device)

    def next(self, out: torch.Tensor | None = None) -> torch.Tensor:
        z = self._normal(0)
        if self.t == 0:
            self.state[0] = z
        else:
            self.state[0].add_(z * self.row_scale)
        self.t += 1
        if out is None:
            return self.state.to(self.dtype, copy=True)
        out.copy_(self.state)
        return out


def blocksel(device="cpu", H=64, W=64, cols=3072, block=8, seed=4):
    """Token-grid stream for the block-selection mode: 64 x 64 tokens x 3072
    channels bf16, per-8x8-block innovation scales log-uniform in [0.01, 0.3]."""
    return BlockStream(H, W, cols, block=block, device=device, seed=seed)


class LowRankWalk(ActivationStream):
    """a_0 ~ N(0,1); a_t = a_{t-1} + U diag(s z_t) W^T + noise N(0,1), with fixed
    Gaussian factors U (rows x k) and W (cols x k) scaled by 1/sqrt(rows) and
    1/sqrt(cols), per-step random signs z_t in {-1, +1}^k and weights
    s_i = amp decay^i: the innovation's spectrum decays, every direction is
    present at every step, and its leading subspace stays put, unlike the
    i.i.d. innovation of the AR(1) stream."""

    def __init__(self, rows, cols, *, rank=70, amp=20.0, decay=0.96, noise=1e-3, dtype=torch.bfloat16,
                 device="cpu", seed=0):
        super().__init__(rows, cols, dtype=dtype, device=device, seed=seed, sigma=noise, seed_per_tensor=[seed])
        g = torch.Generator().manual_seed(int(seed) + 1)
        self.U = (torch.randn(rows, rank, generator=g) / math.sqrt(rows)).to(self.device)
        self.W = (torch.randn(cols, rank, generator=g) / math.sqrt(cols)).to(self.device)
        self.s = (amp * decay ** torch.arange(rank, dtype=torch.float32)).to(self.device)
        self.zgen = torch.Generator().manual_seed(int(seed) + 2)

    def next(self, out: torch.Tensor | None = None) -> torch.Tensor:
        z = self._normal(0)
        if self.t == 0:
            self.state[0] = z
        else:
            sg = torch.randint(0, 2, (self.U.shape[1],), generator=self.zgen).to(torch.float32) * 2 - 1
            c = sg.to(self.device) * self.s
            self.state[0].add_(z * self.sigmas[0]).add_((self.U * c) @ self.W.T)
        self.t += 1
        if out is None:
            return self.state.to(self.dtype, copy=True)
        out.copy_(self.state)
        return out


def lowrank_walk(device="cpu", rows=1024, cols=768, seed=5, **kw):
    """Random walk with a well-separated low-rank innovation (see LowRankWalk)."""
    return LowRankWalk(rows, cols, device=device, seed=seed, **kw)


def tiny(device="cpu"):
    """256 x 64 fp32 random walk, sigma 0.1, seed 0."""
    return ActivationStream(256, 64, dtype=torch.float32, device=device, seed=0, sigma=0.1,
                            seed_per_tensor=[0])


def flux(device="cpu", rows=4608, cols=3072, seed=1):
    """FLUX.1-dev-shaped stream with 1% outlier channels (x20)."""
    return ActivationStream(rows, cols, dtype=torch.bfloat16, device=device, seed=seed, sigma=0.1,
                            outlier_frac=0.01, seed_per_tensor=[seed])


def ar1(device="cpu", rows=4096, cols=3072, seed=3, dtype=torch.bfloat16):
    """Stationary AR(1) stream for the low-rank mode."""
    return ActivationStream(rows, cols, dtype=dtype, device=device, seed=seed, sigma=0.1,
                            rho=math.sqrt(0.99), seed_per_tensor=[seed])


def cogvideox_sigmas(n_tensors=60, seed=2):
    g = torch.Generator().manual_seed(seed)
    return (0.05 + 0.15 * torch.rand(n_tensors, generator=g, dtype=torch.float64)).tolist()


def cogvideox(device="cpu", rows=17550, cols=1920, n_tensors=60, seed=2):
    """CogVideoX-2b-shaped step: 30 layers x 2 tensors, per-tensor sigma ~ U[0.05, 0.2]."""
    return ActivationStream(rows, cols, batch=n_tensors, dtype=torch.bfloat16, device=device, seed=seed,
                            sigma_per_tensor=cogvideox_sigmas(n_tensors, seed),
                            seed_per_tensor=[1000 + b for b in range(n_tensors)])
