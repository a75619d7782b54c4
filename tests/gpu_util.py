"""Helpers shared by the GPU parity tests."""
import numpy as np

BF16_TOL = 2e-2   # max|gpu - oracle| / max|oracle| for bf16 paths
F32_TOL = 1e-4    # same, fp32 path


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (den if den > 0 else 1.0))


def dev(a, dtype):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(dtype).contiguous()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))
