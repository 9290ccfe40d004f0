"""Cache-store inputs placed on the e4m3 rounding boundaries (plain numpy, no library
or oracle code): every element of a row sits within a few fp32 ulps of
midpoint * scale, where midpoint is halfway between two neighbouring e4m3 values and
scale = amax / 448 is the row's FP8 scale.  Rounding x / scale to e4m3 then hangs on
the last bits of the quotient, so two ways of forming it that differ by one fp32 ulp
(a division versus a multiplication by a reciprocal) give different codes on a few
percent of these elements.  The first element of each row is its amax."""
import numpy as np
import torch


def e4m3_midpoints() -> np.ndarray:
    """Midpoints between neighbouring non-negative finite e4m3 values (float64)."""
    vals = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    return (vals[:-1] + vals[1:]) / 2


def boundary_rows(n_rows: int, dim: int, seed: int) -> np.ndarray:
    g = np.random.default_rng(seed)
    mids = e4m3_midpoints()
    mids = mids[mids < 440.0]                   # keep |x| below the row's amax
    out = np.empty((n_rows, dim), np.float32)
    for r in range(n_rows):
        amax = np.float32(np.exp(g.uniform(np.log(1e-2), np.log(1e2))))
        scale = np.float32(amax / np.float32(448.0))
        m = g.choice(mids, dim - 1)
        x = (m * np.float64(scale)).astype(np.float32)
        # a few ulps either side of the boundary
        x = (x.view(np.int32) + g.integers(-3, 4, dim - 1).astype(np.int32)).view(np.float32)
        x = x * np.where(g.random(dim - 1) < 0.5, np.float32(-1.0), np.float32(1.0))
        out[r, 0] = amax
        out[r, 1:] = x
    return out
