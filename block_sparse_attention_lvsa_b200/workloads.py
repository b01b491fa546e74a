"""Workload shapes used by the tests and the benchmark.

Pure data: frame counts, tokens per frame, heads, head size and the
sparsity parameters of each synthetic workload.  Nothing here computes any
part of the attention method.

The Wan-2.1 shapes follow the LVSA explainer ("LVSA: Training-Free Sparse
Attention for Long Video Diffusion", technical summary, section 4 on
computational efficiency: Wan 2.1 1.3B / 14B at 1x and 6x the training
horizon, budget C equal to the 21-frame training horizon of section 2).  The
LoSA workload follows the LoSA article (section on efficiency and quality:
one dense measuring step, then a frozen block index, Wan2.1 models).
"""
from __future__ import annotations

import dataclasses
from typing import Optional


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int            # latent frames
    P: int            # tokens per frame
    H: int            # heads
    d: int            # head size
    C: Optional[int] = None       # LVSA frame budget
    W: Optional[int] = None       # LVSA local window size
    T_per: Optional[int] = None   # LVSA anchor period
    steps: int = 1                # denoising steps
    block: int = 128              # LoSA block size (tokens)
    tau: Optional[float] = None   # LoSA retained-mass fraction
    locality: float = 0.0         # amplitude of the frame sinusoid added to q, k
    perturb: float = 0.0          # per-step perturbation amplitude (LoSA reuse)
    seed_base: int = 0            # seeds are seed_base + step

    @property
    def N(self) -> int:
        return self.T * self.P

    @property
    def scale(self) -> float:
        return self.d ** -0.5


WORKLOADS = {
    # tiny LVSA case the oracle finishes in seconds
    "tiny": Workload("tiny", T=8, P=64, H=2, d=64, C=4, W=3, T_per=4, steps=4,
                     seed_base=1000),
    # Wan-2.1-1.3B at 1x horizon, budget = all 21 frames (equals dense)
    "wan1.3b_1x_dense": Workload("wan1.3b_1x_dense", T=21, P=1560, H=12, d=128,
                                 C=21, W=7, T_per=5, steps=5, seed_base=2000),
    # same shape, C=11, W=7, T_per=5
    "wan1.3b_1x_c11": Workload("wan1.3b_1x_c11", T=21, P=1560, H=12, d=128,
                               C=11, W=7, T_per=5, steps=5, seed_base=2000),
    # Wan-2.1-1.3B at 6x horizon: the headline workload
    "wan1.3b_6x": Workload("wan1.3b_6x", T=126, P=1560, H=12, d=128,
                           C=21, W=15, T_per=6, steps=40, seed_base=3000),
    # balanced variant of the 6x workload (|G_s| + W = C at every step)
    "wan1.3b_6x_tper21": Workload("wan1.3b_6x_tper21", T=126, P=1560, H=12, d=128,
                                  C=21, W=15, T_per=21, steps=40, seed_base=3000),
    # LoSA on Wan-2.1-14B-shaped attention
    "wan14b_losa": Workload("wan14b_losa", T=21, P=1560, H=40, d=128,
                            block=128, tau=0.99, steps=40, locality=2.0,
                            perturb=0.1, seed_base=4000),
    # HunyuanVideo-1.5-shaped long video at 1.5x and 2x its 129-frame
    # training horizon (193 and 257 frames).  The LVSA explainer names the
    # model, the horizons and the memory check (section 4) but not its
    # latent shape; readings: a causal video VAE with 4x temporal
    # compression gives 1 + (frames - 1) / 4 latent frames (33 at the
    # training horizon, 49 and 65 here), 720p with 16x spatial compression
    # and no further patching gives 80 x 45 = 3600 tokens per frame, 16 heads
    # of 128 channels; budget C = the 33-frame training horizon (as C = 21
    # for Wan), T_per = 6 as in the Wan workloads, W = C - |G_s|.
    "hunyuan1.5_1.5x": Workload("hunyuan1.5_1.5x", T=49, P=3600, H=16, d=128, C=33, W=24,
                                T_per=6, steps=50, seed_base=6000),
    "hunyuan1.5_2x": Workload("hunyuan1.5_2x", T=65, P=3600, H=16, d=128, C=33, W=22,
                              T_per=6, steps=50, seed_base=7000),
    # 720p long video with 14B heads, LVSA plus LoSA selection
    "720p_14b": Workload("720p_14b", T=63, P=3600, H=40, d=128, C=21, W=15,
                         T_per=6, steps=40, block=128, tau=0.99, locality=2.0,
                         seed_base=5000),
}
