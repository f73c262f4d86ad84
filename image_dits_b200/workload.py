"""Seeded synthetic Q/K/V shaped like the DiT attention inputs the RainFusion2.0
paper evaluates on (Wan2.2 / HunyuanVideo1.5 video, Qwen-image-edit image).

This module holds only the input recipe and the workload table; none of the
method's arithmetic (permutation, pooling, selection, attention) is here, so
both the CUDA path's tests and the oracle's may consume what it makes.

Recipe (per tensor X in {Q, K, V}, shape [B, heads, N, d], N = T*H*W in the
model's [F, H, W] raster order):

* a smooth field shared by Q, K, V and by every token: for each (head,
  channel) integer frequencies (f_t, f_h, f_w) drawn uniformly from {0,1,2}^3
  and a phase phi ~ U[0, 2*pi); F = sin(2*pi*(f_t*t/T + f_h*y/H + f_w*x/W) + phi);
* X = N(0,1) + 0.5 * F in fp32, with independent noise streams for Q, K, V;
* rotary position embedding on Q and K in fp32 (theta 10000), with the head
  dimension split into t:h:w sections (2D h:w for images); inside a section
  of size s, channel pair (2k, 2k+1) turns by pos * theta^(-2k/s), pos being
  the token's own grid coordinate;
* finally every tensor is rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    frames: int
    height: int
    width: int
    win_t: int
    win_h: int
    win_w: int
    keep: float
    sink: bool
    rope: tuple  # (t, h, w) channel split; t = 0 for images
    text_tokens: int = 0  # joint-attention text tokens, stored after the video tokens

    @property
    def num_video_tokens(self) -> int:
        return self.frames * self.height * self.width

    @property
    def num_tokens(self) -> int:
        return self.num_video_tokens + self.text_tokens

    @property
    def num_blocks(self) -> int:
        return (self.num_tokens + 63) // 64

    def with_keep(self, keep: float) -> "Workload":
        return replace(self, keep=keep, name=f"{self.name}@keep{keep:g}")


# Shapes of the paper's workloads.  Window shapes are this library's reading
# of the unreleased permutation details: 8x8 spatial tiles for images and the
# tiny clip, 4x4x4 spatio-temporal tiles for the video DiT grids.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, 4, 16, 16, 1, 8, 8, 0.5, True, (24, 20, 20)),
    "image": Workload("image", 1, 24, 128, 1, 64, 64, 1, 8, 8, 0.5, False, (0, 64, 64)),
    "video480p": Workload("video480p", 1, 12, 128, 21, 30, 52, 4, 4, 4, 0.2, True, (44, 42, 42)),
    "video720p": Workload("video720p", 1, 40, 128, 21, 45, 80, 4, 4, 4, 0.2, True, (44, 42, 42)),
    # Qwen-image-edit shape (image, 60% sparsity): the latent size is not given, so the
    # 64x64 image grid stands in, kept at 40% of the key blocks, 2D 8x8 windows, no sink.
    "qwen_image": Workload("qwen_image", 1, 24, 128, 1, 64, 64, 1, 8, 8, 0.4, False, (0, 64, 64)),
    # A video DiT with joint video-text attention: 256 text tokens after the 480p latent,
    # grouped with the first frame into the full-attention region.
    "video480p_text": Workload("video480p_text", 1, 12, 128, 21, 30, 52, 4, 4, 4, 0.2, True, (44, 42, 42), 256),
}
SWEEP_KEEPS = (1.0, 0.5, 0.2, 0.1, 0.05)


def _field(wl: Workload, g: torch.Generator, device) -> torch.Tensor:
    T, H, W, d = wl.frames, wl.height, wl.width, wl.head_dim
    freqs = torch.randint(0, 3, (wl.heads, d, 3), generator=g, device=device).to(torch.float32)
    phase = torch.rand((wl.heads, d), generator=g, device=device, dtype=torch.float32) * (2 * math.pi)
    t = torch.arange(T, device=device, dtype=torch.float32) / T
    y = torch.arange(H, device=device, dtype=torch.float32) / H
    x = torch.arange(W, device=device, dtype=torch.float32) / W
    arg = (freqs[:, :, 0, None, None, None] * t[:, None, None]
           + freqs[:, :, 1, None, None, None] * y[None, :, None]
           + freqs[:, :, 2, None, None, None] * x[None, None, :])      # [heads, d, T, H, W]
    arg = 2 * math.pi * arg + phase[:, :, None, None, None]
    return torch.sin(arg).reshape(wl.heads, d, -1).transpose(1, 2).contiguous()  # [heads, N, d]


def _rope_(x: torch.Tensor, wl: Workload, theta: float = 10000.0) -> None:
    """In-place rotary embedding on x [B, heads, N, d] (fp32)."""
    T, H, W = wl.frames, wl.height, wl.width
    dev = x.device
    coords = (
        torch.arange(T, device=dev).repeat_interleave(H * W),
        torch.arange(H, device=dev).repeat_interleave(W).repeat(T),
        torch.arange(W, device=dev).repeat(T * H),
    )
    c0 = 0
    for size, pos in zip(wl.rope, coords):
        if size == 0:
            continue
        k = torch.arange(size // 2, device=dev, dtype=torch.float64)
        inv = theta ** (-2.0 * k / size)
        ang = (pos.to(torch.float64)[:, None] * inv[None, :]).to(torch.float32)  # [N, size/2]
        cos, sin = torch.cos(ang), torch.sin(ang)
        a = x[..., c0:c0 + size:2].clone()
        b = x[..., c0 + 1:c0 + size:2].clone()
        x[..., c0:c0 + size:2] = a * cos - b * sin
        x[..., c0 + 1:c0 + size:2] = a * sin + b * cos
        c0 += size
    assert c0 == wl.head_dim


def make_qkv(wl: Workload, device="cpu", seed: int = 0, batch: int | None = None):
    """Return (q, k, v) bf16 [B, heads, N, d] on `device`: the video tokens in
    [F,H,W] order (field + noise, RoPE on Q and K), then the text tokens (noise
    only, no positional rotation)."""
    B = wl.batch if batch is None else batch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    field = _field(wl, g, device)
    out = []
    for idx in range(3):
        gi = torch.Generator(device=device)
        gi.manual_seed(seed + 1 + idx)
        x = torch.randn((B, wl.heads, wl.num_tokens, wl.head_dim), generator=gi, device=device,
                        dtype=torch.float32)
        nv = wl.num_video_tokens
        x[:, :, :nv].add_(field, alpha=0.5)
        if idx < 2:
            _rope_(x[:, :, :nv], wl)
        out.append(x.to(torch.bfloat16))
        del x
    return tuple(out)


def random_grid_case(rng, max_tokens: int = 4096):
    """A small random geometry for property tests: (T, H, W, wt, wh, ww, sink)."""
    while True:
        T = int(rng.integers(1, 6))
        H = int(rng.integers(1, 24))
        W = int(rng.integers(1, 24))
        if T * H * W <= max_tokens:
            break
    return (T, H, W, int(rng.integers(1, 5)), int(rng.integers(1, 9)), int(rng.integers(1, 9)),
            bool(rng.integers(0, 2)))
