"""The five synthetic workloads of the hot path, described at the pixel level.

No arithmetic of the method lives here: the token grid is derived from
(frames, height, width) by the library call ``wan_token_grid`` (product side)
or by ``oracle.grid.token_grid`` (test side).  Shapes stand in for the pages'
workloads; the tensors themselves are seeded N(0, 1) draws
(``inputs.py``), since no trained weights or datasets are used.

index  name          video                  batch heads text  sampler
0      tiny          5 frames  64 x 64      1     2     16    1 step, shift 5
1      480p-17f      17 frames 480 x 832    1     12    512   shift 5
2      480p-81f      81 frames 480 x 832    2     12    512   (cond + uncond)
3      720p-81f      81 frames 720 x 1280   1     40    512
4      480p-165f     165 frames 480 x 832   1     40    512   40 steps, shift 12

The tiny case is the 2 x 4 x 4 token grid (latent 16 x 2 x 8 x 8), written
as the pixel video that produces it.
"""

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    frames: int
    height: int
    width: int
    batch: int
    heads: int
    head_dim: int
    text_tokens: int        # Lk, the padded text length
    text_len_lo: int        # valid text lengths are uniform in [lo, hi]
    text_len_hi: int
    shift: float
    steps: int
    theta: float = 10000.0


WORKLOADS = (
    Workload(0, "tiny", 5, 64, 64, 1, 2, 128, 16, 11, 11, 5.0, 1),
    Workload(1, "480p-17f", 17, 480, 832, 1, 12, 128, 512, 32, 512, 5.0, 40),
    Workload(2, "480p-81f", 81, 480, 832, 2, 12, 128, 512, 32, 512, 5.0, 40),
    Workload(3, "720p-81f", 81, 720, 1280, 1, 40, 128, 512, 32, 512, 12.0,
             40),
    Workload(4, "480p-165f", 165, 480, 832, 1, 40, 128, 512, 32, 512, 12.0,
             40),
)


def by_name(name):
    for w in WORKLOADS:
        if w.name == name:
            return w
    raise KeyError(name)
