"""Seeded synthetic inputs shaped like a 12B hybrid Mamba-Transformer's linear layers.

This module only draws random numbers (numpy PCG64 streams) and casts them to
bf16 with torch's round-to-nearest-even CPU cast.  It holds none of the NVFP4
method's arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Workloads (full sizes; tests use the same recipes at smaller shapes):
  tiny    X, W 256x256 fp32 N(0,1); 4 entries per tensor scaled x50 (seed 1)
  qsweep  A 8192x8192, B 16384x5120 bf16: 0.02 * Student-t(df=3) with 0.01% of
          positions scaled x100 (seed 2)
  fprop   X 8192x5120 N(0,1), W 20480x5120 N(0, 0.02^2), bf16 (seed 3)
  wgrad   dY 16384x20480 bf16: N(0,1) * 1e-3 * s_i with s_i = |t_df=2| per row;
          X 16384x5120 N(0,1) (seed 4)
  mlp     X 8192x5120 N(0,1); W1 20480x5120, W2 5120x20480 N(0, 0.02^2);
          dY2 8192x5120 N(0, 1e-3^2), all bf16 (seed 5)
"""
import numpy as np
import torch

TOKENS, HIDDEN, FFN = 8192, 5120, 20480


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 array -> uint16 bf16 bit patterns (torch CPU cast, round-to-nearest-even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_torch_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16)


def normal(rng, shape, std=1.0):
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def with_outliers(rng, x, count, factor):
    """Scale `count` distinct positions (drawn without replacement) by `factor`."""
    pos = rng.choice(x.size, size=count, replace=False)
    flat = x.reshape(-1)
    flat[pos] *= np.float32(factor)
    return x


def student_t(rng, shape, df, scale):
    return (rng.standard_t(df, size=shape) * scale).astype(np.float32)


def heavy_rows(rng, shape, std, df):
    """N(0,1) * std * s_i, one s_i = |t_df| per row (heavy-tailed row magnitudes)."""
    s = np.abs(rng.standard_t(df, size=(shape[0], 1))).astype(np.float32)
    return normal(rng, shape) * np.float32(std) * s


def tiny(seed=1, n=256):
    rng = np.random.default_rng(seed)
    X = with_outliers(rng, normal(rng, (n, n)), 4, 50.0)
    W = with_outliers(rng, normal(rng, (n, n)), 4, 50.0)
    return {"X": X, "W": W}


def qsweep(seed=2, shapes=((8192, 8192), (16384, 5120)), outlier_frac=1e-4):
    rng = np.random.default_rng(seed)
    out = {}
    for name, shp in zip(("A", "B"), shapes):
        x = student_t(rng, shp, 3, 0.02)
        cnt = int(round(outlier_frac * x.size))
        out[name] = bf16_bits(with_outliers(rng, x, max(cnt, 1), 100.0))
    return out


def fprop(seed=3, M=TOKENS, N=FFN, K=HIDDEN):
    rng = np.random.default_rng(seed)
    return {"X": bf16_bits(normal(rng, (M, K))), "W": bf16_bits(normal(rng, (N, K), 0.02))}


def wgrad(seed=4, M=2 * TOKENS, N=FFN, K=HIDDEN):
    rng = np.random.default_rng(seed)
    return {"dY": bf16_bits(heavy_rows(rng, (M, N), 1e-3, 2)),
            "X": bf16_bits(normal(rng, (M, K)))}


def mlp(seed=5, M=TOKENS, H=HIDDEN, F=FFN, data_seed=None):
    """The MLP block's inputs.  With data_seed, X and dY2 (a data-parallel
    rank's token shard) come from their own generator while W1 and W2 stay
    those of `seed`, so every rank holds the same weights."""
    rng = np.random.default_rng(seed)
    w = {"X": bf16_bits(normal(rng, (M, H))),
         "W1": bf16_bits(normal(rng, (F, H), 0.02)),
         "W2": bf16_bits(normal(rng, (H, F), 0.02)),
         "dY2": bf16_bits(normal(rng, (M, H), 1e-3))}
    if data_seed is not None:
        drng = np.random.default_rng(data_seed)
        w["X"] = bf16_bits(normal(drng, (M, H)))
        w["dY2"] = bf16_bits(normal(drng, (M, H), 1e-3))
    return w
