"""Seeded synthetic inputs for the NVFP4 linear-layer workloads.

Only random-number generation lives here (no quantisation arithmetic): both the
CUDA path and the CPU oracle are fed from these tensors.  Every generator is
seeded and returns a BF16 torch tensor on the requested device (values are
drawn in FP32 and rounded to BF16).

Workloads (the 12B hybrid Mamba-Transformer and 3B-class models of the NVIDIA
NVFP4 pretraining summary, plus a tiny case and a quantiser sweep):
  tiny      A, B [256 x 256] ~ N(0,1), 1 % of entries x50 (outliers); seed 0
  qsweep    [n x n], n in {4096, 8192, 16384}, Student-t(nu=3) * 0.1; seed 1
  mlp3b     X [8192 x 3072] ~ N(0,1), W [8192 x 3072] ~ N(0,0.02),
            dY [8192 x 8192] ~ N(0,1e-3); seeds 2, 3, 4
  hybrid12b tokens 16384, hidden 5120, FFN 20480: W_up [20480 x 5120],
            W_down [5120 x 20480] ~ N(0,0.014); X [16384 x 5120] and the
            down-projection input [16384 x 20480] ~ N(0,1) with 0.1 % x100
            outliers; dY ~ N(0,1e-3); seeds 10..
  spectrum  [m x n] = U diag(sigma) V^T with orthonormal U, V from seeded
            Gaussians and sigma evenly spaced in [smin, smax] (Newton-Schulz
            inputs with a known polar factor)
  layer3b   32768 tokens: QKV 3072->9216, O 3072->3072, gate-up 3072->16384,
            down 8192->3072 (weights N(0,0.02), activations N(0,1), dY
            N(0,1e-3)); seeds 20..; square GEMMs n^3, n in 4096..32768, seeds 30+i
The second parameter of N(0, s) is the standard deviation.
"""

import torch


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std=1.0, seed=0, device="cpu", outlier_frac=0.0, outlier_mult=1.0):
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std
    if outlier_frac > 0:
        mask = torch.rand(shape, generator=g, device=device) < outlier_frac
        x = torch.where(mask, x * outlier_mult, x)
    return x.to(torch.bfloat16)


def student_t(shape, nu=3, scale=0.1, seed=1, device="cpu"):
    """Student-t with integer nu: z / sqrt(chi2_nu / nu), chi2_nu a sum of nu squared normals."""
    g = _gen(seed, device)
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(nu):
        chi2 += torch.randn(shape, generator=g, device=device, dtype=torch.float32) ** 2
    return (z / torch.sqrt(chi2 / nu) * scale).to(torch.bfloat16)


def tiny(device="cpu"):
    a = normal((256, 256), 1.0, seed=0, device=device, outlier_frac=0.01, outlier_mult=50.0)
    b = normal((256, 256), 1.0, seed=100, device=device, outlier_frac=0.01, outlier_mult=50.0)
    return a, b


def qsweep(n, device="cpu"):
    return student_t((n, n), 3, 0.1, seed=1, device=device)


def mlp3b(device="cpu"):
    x = normal((8192, 3072), 1.0, seed=2, device=device)
    w = normal((8192, 3072), 0.02, seed=3, device=device)
    dy = normal((8192, 8192), 1e-3, seed=4, device=device)
    return x, w, dy


HYBRID12B = {"tokens": 16384, "hidden": 5120, "ffn": 20480}


def hybrid12b(device="cpu"):
    T, H, F = HYBRID12B["tokens"], HYBRID12B["hidden"], HYBRID12B["ffn"]
    return {
        "w_up": normal((F, H), 0.014, seed=10, device=device),
        "w_down": normal((H, F), 0.014, seed=11, device=device),
        "x_up": normal((T, H), 1.0, seed=12, device=device, outlier_frac=0.001, outlier_mult=100.0),
        "x_down": normal((T, F), 1.0, seed=13, device=device, outlier_frac=0.001, outlier_mult=100.0),
        "dy_up": normal((T, F), 1e-3, seed=14, device=device),
        "dy_down": normal((T, H), 1e-3, seed=15, device=device),
    }


LAYER3B = {"tokens": 32768, "linears": {"qkv": (9216, 3072), "o": (3072, 3072), "gate_up": (16384, 3072),
                                        "down": (3072, 8192)}}


def layer3b_linear(name, device="cpu"):
    T = LAYER3B["tokens"]
    N, K = LAYER3B["linears"][name]
    base = 20 + 3 * list(LAYER3B["linears"]).index(name)
    return (normal((T, K), 1.0, seed=base, device=device),
            normal((N, K), 0.02, seed=base + 1, device=device),
            normal((T, N), 1e-3, seed=base + 2, device=device))


def square(n, i=0, device="cpu"):
    return normal((n, n), 1.0, seed=30 + 2 * i, device=device), normal((n, n), 1.0, seed=31 + 2 * i, device=device)


def spectrum(m, n, smin=0.1, smax=1.0, seed=0, device="cpu"):
    """[m x n], m <= n: U diag(sigma) V^T with sigma evenly spaced in [smin, smax]."""
    g = _gen(seed, "cpu")
    u, _ = torch.linalg.qr(torch.randn((m, m), generator=g, dtype=torch.float64))
    v, _ = torch.linalg.qr(torch.randn((n, m), generator=g, dtype=torch.float64))
    sigma = torch.linspace(smin, smax, m, dtype=torch.float64)
    return ((u * sigma) @ v.T).to(torch.float32).to(torch.bfloat16).to(device)
