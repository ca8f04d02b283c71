"""Seeded synthetic inputs for the quantization path.

This module only draws random numbers: it holds none of the quantization
arithmetic, so that the CUDA path and the CPU oracle can both be fed from it.
Every generator is deterministic for a given (seed, device). Large tensors are
drawn on the device they will be used on; a CPU copy of the same tensor serves
the oracle.

Workloads (shapes from the source pages and their benchmark tables):
  * tiny jagged:   A (256, 512) ~ N(0,1) * 2^U(-4,4) per row, G=4 groups from
                   multinomial counts of 16-row units (one group may be empty)
  * blockwise:     activations (16384, 4096) ~ N(0,1) with 1% outliers x100;
                   weight (14336, 4096) ~ N(0, 0.02)   (Llama-3-8B MLP shapes)
  * jagged bwd:    grad_out, input (65536, 4096) ~ Student-t(3), G=16 groups
                   with Dirichlet(0.5) sizes in units of 16 rows
  * MX 3-D:        expert weights (E, 8192, 5120) ~ N(0, 0.02)
  * MX activation: tokens (65536, 7168) ~ N(0,1), G=64 Dirichlet(0.3) groups
  * scale sweep:   uint8 scales uniform in [0, 254], G=8 Dirichlet(1.0) groups
"""
import numpy as np
import torch


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def largest_remainder(weights, total):
    """Integer sizes proportional to `weights` that sum to `total`
    (largest-remainder rounding, ties to the lowest index)."""
    w = np.asarray(weights, dtype=np.float64)
    exact = w / w.sum() * total
    base = np.floor(exact).astype(np.int64)
    left = int(total - base.sum())
    frac = exact - base
    order = sorted(range(len(w)), key=lambda i: (-frac[i], i))
    for i in order[:left]:
        base[i] += 1
    return base


def offsets_from_sizes(sizes):
    return torch.tensor(np.cumsum(np.asarray(sizes, dtype=np.int64)), dtype=torch.int32)


def multinomial_offsets(total, groups, unit, seed):
    """Group ends along a dimension of `total` rows: `total/unit` units dealt
    to `groups` groups by a uniform multinomial draw (empty groups possible)."""
    g = _gen(seed, "cpu")
    n_units = total // unit
    draws = torch.multinomial(torch.ones(groups), n_units, replacement=True, generator=g)
    counts = torch.bincount(draws, minlength=groups).numpy() * unit
    return offsets_from_sizes(counts)


def dirichlet_offsets(total, groups, alpha, seed, unit=1):
    """Group ends with Dirichlet(alpha) proportions of total/unit units."""
    rng = np.random.default_rng(int(seed))
    p = rng.dirichlet([alpha] * groups)
    sizes = largest_remainder(p, total // unit) * unit
    return offsets_from_sizes(sizes)


def normal_bf16(shape, std, seed, device="cpu"):
    g = _gen(seed, device)
    return (torch.randn(shape, generator=g, device=device) * std).to(torch.bfloat16)


def row_scaled_normal_bf16(rows, cols, seed, device="cpu", lo=-4.0, hi=4.0):
    """N(0,1) * 2^u with u ~ U(lo, hi) drawn once per row."""
    g = _gen(seed, device)
    x = torch.randn((rows, cols), generator=g, device=device)
    u = torch.rand((rows, 1), generator=g, device=device) * (hi - lo) + lo
    return (x * torch.exp2(u)).to(torch.bfloat16)


def outlier_normal_bf16(rows, cols, seed, device="cpu", p=0.01, factor=100.0):
    """N(0,1) where a Bernoulli(p) mask of elements is multiplied by `factor`."""
    g = _gen(seed, device)
    x = torch.randn((rows, cols), generator=g, device=device)
    m = torch.rand((rows, cols), generator=g, device=device) < p
    return torch.where(m, x * factor, x).to(torch.bfloat16)


def student_t3_bf16(rows, cols, seed, device="cpu"):
    """Student-t with 3 degrees of freedom: Z / sqrt(chi2_3 / 3), the chi-square
    drawn as a sum of three squared standard normals."""
    g = _gen(seed, device)
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 24) // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        z = torch.randn((4, r1 - r0, cols), generator=g, device=device)
        chi2 = z[1] * z[1] + z[2] * z[2] + z[3] * z[3]
        out[r0:r1] = (z[0] / torch.sqrt(chi2 / 3.0)).to(torch.bfloat16)
    return out


def uniform_u8(shape, lo, hi, seed, device="cpu"):
    g = _gen(seed, device)
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.int32).to(torch.uint8)


# ---- workloads --------------------------------------------------------------

def tiny_jagged(device="cpu", seed=0, rows=256, cols=512, groups=4, unit=16):
    a = row_scaled_normal_bf16(rows, cols, seed, device)
    offs = multinomial_offsets(rows, groups, unit, seed)
    return a, offs


def forced_empty_offsets():
    return torch.tensor([64, 64, 192, 256], dtype=torch.int32)


def blockwise_act(device="cpu", rows=16384, cols=4096, seed=1):
    return outlier_normal_bf16(rows, cols, seed, device)


def blockwise_weight(device="cpu", rows=14336, cols=4096, seed=2):
    return normal_bf16((rows, cols), 0.02, seed, device)


def jagged_bwd(device="cpu", rows=65536, cols=4096, groups=16, seeds=(3, 4, 5), unit=16):
    grad_out = student_t3_bf16(rows, cols, seeds[0], device)
    inp = student_t3_bf16(rows, cols, seeds[1], device)
    offs = dirichlet_offsets(rows, groups, 0.5, seeds[2], unit=unit)
    return grad_out, inp, offs


def mx3d_weight(E, device="cpu", N=8192, K=5120, seed=None):
    seed = 6 + E if seed is None else seed
    g = _gen(seed, device)
    w = torch.empty((E, N, K), dtype=torch.bfloat16, device=device)
    for e in range(E):
        w[e] = (torch.randn((N, K), generator=g, device=device) * 0.02).to(torch.bfloat16)
    return w


def mx_act(device="cpu", rows=65536, cols=7168, groups=64, seeds=(7, 8)):
    x = normal_bf16((rows, cols), 1.0, seeds[0], device)
    offs = dirichlet_offsets(rows, groups, 0.3, seeds[1])
    return x, offs


def scale_sweep_k(rows, cols, device="cpu", groups=8, seeds=(9, 11)):
    """The scale sweep with its G groups along the columns (K) instead."""
    s = uniform_u8((rows, cols), 0, 254, seeds[0], device)
    offs = dirichlet_offsets(cols, groups, 1.0, seeds[1])
    return s, offs


def scale_sweep(rows, cols, device="cpu", groups=8, seeds=(9, 10)):
    s = uniform_u8((rows, cols), 0, 254, seeds[0], device)
    offs = dirichlet_offsets(rows, groups, 1.0, seeds[1])
    return s, offs
