"""Named Wan-shaped workloads for block-sparse video attention.

Each workload is a latent token grid T x H x W split into tt x th x tw cube
tiles (64 tokens), with the number of key tiles each query tile keeps.  The
grid sizes follow the Wan 2.1 video shapes the FastVideo distillation docs
(page "Distillation", section "Model Overview") and the SparkDiffusion news
item quote in pixels (480P / 720P, 61-81 frames), read through a 4x temporal,
8x spatial VAE and a 2x2 patchify.  The 97 %-sparse workload with a linear
branch mirrors SparkDiffusion's RoLA setting (3 % of blocks kept, paragraph 2)
and TurboDiffusion's sparse-linear attention (section "稀疏、蒸馏与全链路量化").
"""
from dataclasses import dataclass, asdict


def ceil_div(a: int, b: int) -> int:
    return (a + b - 1) // b


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    head_dim: int
    T: int
    H: int
    W: int
    topk: int
    amplitude: float          # noise scale a in  x = a*N(0,1) + tile offset
    linear: bool = False      # add the elu+1 linear-attention branch
    tile: tuple = (4, 4, 4)

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def tile_grid(self) -> tuple:
        tt, th, tw = self.tile
        return (ceil_div(self.T, tt), ceil_div(self.H, th), ceil_div(self.W, tw))

    @property
    def num_tiles(self) -> int:
        a, b, c = self.tile_grid
        return a * b * c

    @property
    def sparsity(self) -> float:
        return 1.0 - self.topk / self.num_tiles

    def fine_flops(self) -> float:
        """Effective FLOPs of the fine pass on the selected blocks only:
        4 * N_valid * k * 64 * d per (batch, head) -- two contractions (scores
        and weighted values), 2 FLOPs per multiply-add."""
        vol = self.tile[0] * self.tile[1] * self.tile[2]
        return 4.0 * self.N * self.topk * vol * self.head_dim * self.heads * self.B

    def shape_args(self) -> dict:
        return dict(B=self.B, heads=self.heads, head_dim=self.head_dim, T=self.T,
                    H=self.H, W=self.W, tt=self.tile[0], th=self.tile[1],
                    tw=self.tile[2])

    def as_dict(self) -> dict:
        d = asdict(self)
        d["tile"] = list(self.tile)
        d["N"] = self.N
        d["num_tiles"] = self.num_tiles
        return d


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_4x32x32", 1, 2, 64, 4, 32, 32, 13, 1.0),
        Workload("wan1.3b_480p", 1, 12, 128, 16, 28, 52, 73, 0.7),
        Workload("wan14b_480p", 1, 40, 128, 20, 28, 52, 46, 0.7),
        Workload("wan14b_720p_ragged", 1, 40, 128, 21, 45, 80, 144, 0.7),
        Workload("sparse97_linear_480p", 1, 12, 128, 16, 28, 52, 11, 0.7, linear=True),
    ]
}

# The workload the throughput figure is quoted on.
HEADLINE = "wan14b_480p"
