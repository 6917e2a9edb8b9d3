"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no arithmetic of the quantization method: it only draws
random tensors (numpy PCG64, fixed seeds) and rounds them to bf16 with
round-to-nearest-even (torch's float32 -> bfloat16 cast).  Both the CUDA path
and the CPU oracle consume the same bytes.

Workloads (the pages' models and datasets are not available; these are
stand-ins with the same shapes and value distributions):

* ``pr1``      -- one 256x1024 tensor, N(0,1), 0.5% of entries (1311, without
                  replacement) multiplied by 20; a 256x1024 N(0, 0.02) weight.
* ``fwd_8b``   -- activations 8192x4096, N(0,1) with 0.1% of the channels
                  (4 columns) multiplied by 50; weight 14336x4096 N(0, 0.02).
                  Shapes of the 8B hybrid model in the NVFP4 pretraining
                  write-up, §五.
* ``bwd_8b``   -- output gradient 8192x14336 ~ Laplace(0, 1e-4) with 0.01% of
                  entries set to +-1e-2 (random sign).
* ``sweep``    -- 4096xN, N(0,1) with 0.1% channel outliers x50.
* ``step_12b`` -- tokens 16384, hidden 5120, FFN 20480 (12B hybrid model of
                  the same write-up, §三): activations, up-projection weight
                  and output gradient with the distributions above.
"""
import numpy as np
import torch


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32 numpy -> bf16 torch tensor (round to nearest even), on CPU."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor -> numpy uint16 bit patterns (same shape)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def normal_with_entry_outliers(rows, cols, seed, frac=0.005, factor=20.0):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((rows, cols), dtype=np.float32)
    n = int(round(frac * rows * cols))
    idx = rng.choice(rows * cols, size=n, replace=False)
    a.reshape(-1)[idx] *= np.float32(factor)
    return to_bf16(a)


def normal_with_channel_outliers(rows, cols, seed, frac=0.001, factor=50.0):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((rows, cols), dtype=np.float32)
    n = max(1, int(round(frac * cols)))
    ch = rng.choice(cols, size=n, replace=False)
    a[:, ch] *= np.float32(factor)
    return to_bf16(a)


def weight(rows, cols, seed, std=0.02):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    return to_bf16(a)


def laplace_with_spikes(rows, cols, seed, scale=1e-4, frac=1e-4, spike=1e-2):
    rng = np.random.default_rng(seed)
    a = rng.laplace(0.0, scale, size=(rows, cols)).astype(np.float32)
    n = max(1, int(round(frac * rows * cols)))
    idx = rng.choice(rows * cols, size=n, replace=False)
    sign = np.where(rng.random(n) < 0.5, -1.0, 1.0).astype(np.float32)
    a.reshape(-1)[idx] = sign * np.float32(spike)
    return to_bf16(a)


# Shapes of the named workloads.
PR1 = dict(x=(256, 1024), w=(256, 1024))
FWD_8B = dict(x=(8192, 4096), w=(14336, 4096))
BWD_8B = dict(dy=(8192, 14336))
STEP_12B = dict(tokens=16384, hidden=5120, ffn=20480)
SWEEP_N = (256, 1024, 4096, 16384, 65536, 262144)


def pr1():
    return dict(x=normal_with_entry_outliers(*PR1["x"], seed=0),
                w=weight(*PR1["w"], seed=1))


def layer(tokens, hidden, out_features, seed=0):
    """Activations [tokens, hidden], weight [out, hidden], grad-output
    [tokens, out] for one linear layer."""
    return dict(x=normal_with_channel_outliers(tokens, hidden, seed=seed),
                w=weight(out_features, hidden, seed=seed + 1),
                dy=laplace_with_spikes(tokens, out_features, seed=seed + 2))


def fwd_bwd_8b(seed=0):
    return layer(FWD_8B["x"][0], FWD_8B["x"][1], FWD_8B["w"][0], seed=seed)


def step_12b(seed=0):
    s = STEP_12B
    return layer(s["tokens"], s["hidden"], s["ffn"], seed=seed)


def sweep(n, seed=0):
    return normal_with_channel_outliers(4096, n, seed=seed)


# ---------------------------------------------------------------------------
# Device-side draws with the same distributions, for timing runs whose
# tensors are too large to draw on the host in reasonable time (torch's
# counter-based CUDA generator, fixed seeds; bf16 by round-to-nearest-even).
# ---------------------------------------------------------------------------
def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def device_normal_with_channel_outliers(rows, cols, seed, device, frac=0.001, factor=50.0):
    g = _gen(seed, device)
    a = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    n = max(1, int(round(frac * cols)))
    ch = torch.randperm(cols, generator=g, device=device)[:n]
    a[:, ch] *= factor
    return a.to(torch.bfloat16)


def device_weight(rows, cols, seed, device, std=0.02):
    g = _gen(seed, device)
    return (torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def device_laplace_with_spikes(rows, cols, seed, device, scale=1e-4, frac=1e-4, spike=1e-2):
    g = _gen(seed, device)
    u = torch.rand((rows, cols), generator=g, device=device, dtype=torch.float32) - 0.5
    # inverse CDF of Laplace(0, scale); u = -0.5 (probability 2^-24) is nudged to avoid log(0)
    a = -scale * torch.sign(u) * torch.log1p(-2.0 * u.abs().clamp(max=0.5 - 2.0 ** -25))
    n = max(1, int(round(frac * rows * cols)))
    idx = torch.randint(0, rows * cols, (n,), generator=g, device=device)
    sign = torch.where(torch.rand((n,), generator=g, device=device) < 0.5, -1.0, 1.0)
    a.view(-1)[idx] = sign * spike
    return a.to(torch.bfloat16)


def device_layer(tokens, hidden, out_features, seed, device):
    return dict(x=device_normal_with_channel_outliers(tokens, hidden, seed, device),
                w=device_weight(out_features, hidden, seed + 1, device),
                dy=device_laplace_with_spikes(tokens, out_features, seed + 2, device))


def device_sweep(n, seed, device):
    return device_normal_with_channel_outliers(4096, n, seed, device)
