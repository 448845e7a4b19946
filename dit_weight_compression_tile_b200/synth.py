"""Seeded synthetic weight matrices shaped like the EntroPack workloads.

Random numbers only: nothing of the compression method lives here, so the oracle's
tests and the product's tests and benchmark can share these generators.  Every draw
uses a CPU ``torch.Generator`` so the values do not depend on the device; BF16 values
come from an fp32 draw rounded to nearest even by ``Tensor.to``.

Workloads (the pages' README example and the denoiser weight sets the method targets):
  * ``gaussian(rows, cols, std, seed)`` -- i.i.d. N(0, std^2), the README's
    ``randn * 0.02`` example.
  * ``row_lognormal(rows, cols, seed)`` -- rows with std 0.02 * exp(0.3 g_r), g_r ~ N(0,1).
  * ``dit_layer(block, layer)`` -- one linear weight of a 28-block, hidden-3072 DiT:
    Student-t(5) entries scaled to std 0.02, times a per-row log-normal(0, 0.3) scale.
  * ``gaussian_outliers(rows, cols, seed)`` -- N(0, 0.02^2) with 0.1% of the entries
    (exact count, distinct positions) replaced by +-8 sigma.
"""
import numpy as np
import torch

DIT_BLOCKS = 28
DIT_HIDDEN = 3072
# (rows, cols) of the four linear weights of one DiT block: qkv, out, MLP up, MLP down
DIT_LAYERS = ((3072, 9216), (3072, 3072), (3072, 12288), (12288, 3072))


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def gaussian(rows, cols, std=0.02, seed=0, dtype=torch.bfloat16):
    g = _gen(seed)
    return (torch.randn(rows, cols, generator=g) * std).to(dtype)


def row_lognormal(rows, cols, seed=1, std=0.02, sigma=0.3, dtype=torch.bfloat16):
    g = _gen(seed)
    row_std = std * torch.exp(sigma * torch.randn(rows, 1, generator=g))
    return (torch.randn(rows, cols, generator=g) * row_std).to(dtype)


def student_t(rows, cols, nu, g):
    z = torch.randn(rows, cols, generator=g)
    chi2 = torch.zeros(rows, cols)
    for _ in range(nu):
        chi2 += torch.randn(rows, cols, generator=g) ** 2
    return z / torch.sqrt(chi2 / nu)


def dit_layer(block, layer, dtype=torch.bfloat16):
    rows, cols = DIT_LAYERS[layer]
    g = _gen(100 + 4 * block + layer)
    row_scale = torch.exp(0.3 * torch.randn(rows, 1, generator=g))
    t = student_t(rows, cols, 5, g) / float(np.sqrt(5.0 / 3.0))  # unit variance
    return (t * 0.02 * row_scale).to(dtype)


def gaussian_outliers(rows, cols, seed=3, std=0.02, frac=0.001, sigmas=8.0, dtype=torch.bfloat16):
    g = _gen(seed)
    w = torch.randn(rows, cols, generator=g) * std
    n = rows * cols
    k = int(round(frac * n))
    rng = np.random.default_rng(seed)
    pos = torch.from_numpy(rng.choice(n, size=k, replace=False, shuffle=False).astype(np.int64))
    sign = torch.from_numpy(rng.integers(0, 2, size=k).astype(np.float32) * 2 - 1)
    w.view(-1)[pos] = sign * (sigmas * std)
    return w.to(dtype)


# The workloads as (name, tensor factory, container, target bpp list)
def workloads():
    return {
        "readme_256": (lambda: gaussian(256, 256, 0.02, 0), "bf16", [3.5]),
        "lognormal_4096": (lambda: row_lognormal(4096, 4096, 1), "bf16", [4.0]),
        "int8_8192": (lambda: gaussian(8192, 8192, 0.02, 2), "int8", [3.0]),
        "fp8_8192": (lambda: gaussian(8192, 8192, 0.02, 2), "fp8_e4m3", [3.0]),
        "outlier_sweep_8192x28672": (lambda: gaussian_outliers(8192, 28672, 3), "bf16",
                                     [0.5, 1.0, 2.0, 3.5, 5.0, 8.0]),
    }
