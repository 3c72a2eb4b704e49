"""Seeded synthetic workloads shaped like the backbones HeadKV is evaluated on.

This module only draws inputs.  It holds none of the method's arithmetic and
serves both the CUDA path (tests, bench) and the CPU oracle (tests), which
receive the very same bf16/fp32 tensors.

Recipe (per layer): K and V are i.i.d. N(0, 1).  Queries carry a planted
attention pattern.  A "planted Local" head's query at position t is
4 * mean(k at t-1..t-4 and at the three positions around t - pitch, i.e.
t-pitch-1, t-pitch, t-pitch+1) + N(0, 1), pitch being the raster row length
of the image grid, so the head looks at its left and upper neighbours; a
"planted Global" head's query is 4 * mean(k at 8 positions drawn uniformly
from 0..t-1, redrawn at every position) + N(0, 1).  Positions before 0 are
dropped and a query with nothing to look at is pure noise.  Which heads are
planted Local is a seeded random subset per layer, shared by the sequences
(the first workload fixes heads 0..11).  bf16 workloads are drawn in fp32
and rounded once.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    num_seqs: int          # S: sequences (CFG doubles the image batch)
    num_layers: int
    num_heads: int
    head_dim: int
    dtype: str             # "f32" | "bf16"
    prefix_len: int        # class token or text prefix
    image_tokens: int
    prefill_image: int     # image tokens produced before classification
    row_pitch: int         # raster row length (image row + line-break token)
    local_heads: int       # planted Local heads per layer
    local_window: int      # W
    rho: tuple             # (num, den)
    ste_m: int             # M
    near_dist: int         # D
    images: int            # images produced per pass (S/2 under CFG)
    score_window: int = 8  # r
    fixed_local: bool = False  # planted Local heads are 0..local_heads-1

    @property
    def max_len(self) -> int:
        return self.prefix_len + self.image_tokens

    @property
    def prefill_len(self) -> int:
        return self.prefix_len + self.prefill_image

    @property
    def decode_steps(self) -> int:
        return self.max_len - self.prefill_len

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # single attention layer, LlamaGen-like, fp32, 16x16 image
    "llamagen_1layer_f32": Workload(
        "llamagen_1layer_f32", num_seqs=1, num_layers=1, num_heads=20, head_dim=64,
        dtype="f32", prefix_len=1, image_tokens=256, prefill_image=64, row_pitch=16,
        local_heads=12, local_window=20, rho=(1, 4), ste_m=16, near_dist=32, images=1,
        fixed_local=True),
    # LlamaGen-XL-shaped stack, 24x24 image, CFG 2 x 32
    "llamagen_xl": Workload(
        "llamagen_xl", num_seqs=64, num_layers=36, num_heads=20, head_dim=64, dtype="bf16",
        prefix_len=1, image_tokens=576, prefill_image=96, row_pitch=24, local_heads=12,
        local_window=28, rho=(1, 6), ste_m=32, near_dist=48, images=32),
    # Janus-Pro-1B-shaped stack
    "janus_pro_1b": Workload(
        "janus_pro_1b", num_seqs=32, num_layers=24, num_heads=16, head_dim=128,
        dtype="bf16", prefix_len=64, image_tokens=576, prefill_image=128, row_pitch=24,
        local_heads=8, local_window=28, rho=(1, 8), ste_m=32, near_dist=48, images=16),
    # Janus-Pro-7B-shaped stack at the three compression ratios
    **{f"janus_pro_7b_rho{den}": Workload(
        f"janus_pro_7b_rho{den}", num_seqs=32, num_layers=30, num_heads=32, head_dim=128,
        dtype="bf16", prefix_len=64, image_tokens=576, prefill_image=128, row_pitch=24,
        local_heads=16, local_window=28, rho=(1, den), ste_m=32, near_dist=48, images=16)
       for den in (4, 6, 8)},
    # Lumina-mGPT-768-shaped stack: 48 rows of 48 image tokens + 1 line break
    "lumina_mgpt_768": Workload(
        "lumina_mgpt_768", num_seqs=16, num_layers=32, num_heads=32, head_dim=128,
        dtype="bf16", prefix_len=128, image_tokens=48 * 49, prefill_image=256,
        row_pitch=49, local_heads=16, local_window=56, rho=(1, 6), ste_m=64,
        near_dist=98, images=8),
}


def planted_local_heads(w: Workload, layer: int, seed: int) -> torch.Tensor:
    """Bool [H]: heads planted Local in this layer."""
    mask = torch.zeros(w.num_heads, dtype=torch.bool)
    if w.fixed_local:
        mask[: w.local_heads] = True
        return mask
    g = torch.Generator().manual_seed(seed * 7919 + layer * 104729 + 17)
    mask[torch.randperm(w.num_heads, generator=g)[: w.local_heads]] = True
    return mask


@torch.no_grad()
def generate_layer(w: Workload, layer: int, seed: int = 0, device="cpu",
                   num_seqs: int | None = None, max_len: int | None = None):
    """(q, k, v), each [S, H, L, d] in the workload's dtype, on `device`."""
    S = w.num_seqs if num_seqs is None else num_seqs
    L = w.max_len if max_len is None else max_len
    H, d = w.num_heads, w.head_dim
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(seed * 1000003 + layer * 9176 + 1)
    k = torch.randn(S, H, L, d, generator=g, device=dev)
    v = torch.randn(S, H, L, d, generator=g, device=dev)
    q = torch.randn(S, H, L, d, generator=g, device=dev)
    local = planted_local_heads(w, layer, seed).to(dev)

    # planted Local: left neighbours and the three upper neighbours
    p = w.row_pitch
    offsets = [1, 2, 3, 4, p + 1, p, p - 1]
    acc = torch.zeros(S, H, L, d, device=dev)
    cnt = torch.zeros(L, device=dev)
    for o in offsets:
        if 0 < o < L:
            acc[:, :, o:] += k[:, :, : L - o]
            cnt[o:] += 1
    mean_local = acc / cnt.clamp(min=1)[None, None, :, None]

    # planted Global: 8 uniformly drawn earlier positions per query
    t = torch.arange(L, device=dev, dtype=torch.float32)
    mean_global = torch.zeros(S, H, L, d, device=dev)
    for s in range(S):
        u = torch.rand(H, L, 8, generator=g, device=dev)
        idx = torch.minimum((u * t[None, :, None]).long(),
                            (t.long() - 1).clamp(min=0)[None, :, None])
        rows = torch.gather(k[s], 1, idx.reshape(H, L * 8, 1).expand(H, L * 8, d))
        mean_global[s] = rows.view(H, L, 8, d).mean(dim=2)
    mean_global[:, :, 0] = 0.0  # position 0 has nothing earlier to look at

    planted = torch.where(local[None, :, None, None], mean_local, mean_global)
    q = q + 4.0 * planted
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)
