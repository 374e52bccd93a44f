"""Seeded synthetic inputs for the tests and the benchmark.

This module only draws random numbers and builds matrices with prescribed
spectra; it holds none of the optimizer's arithmetic, and both the CUDA path
and the CPU oracle receive exactly the tensors it produces.

Workloads (the shapes are those of the model families the pages train; all
values are synthetic, no dataset or trained weights are involved):
  tiny        one fp32 64 x 128 matrix, 3 Muon steps (plain Muon: alpha = 0)
  gpt2_small  12 layers x {4 x 768x768, 768x3072, 3072x768}, bf16 W/G/G_prev
  llama_430m  24 layers x {4 x 1024x1024, 2 x 4096x1024, 1024x4096}, bf16
  moe_gram    64 x 2048x768 + 64 x 768x2048 + 1 x 16384x2048, fp16, spectra
              log-spaced from 1 to 1/kappa (kappa in 1e1, 1e2, 1e3)
  llama3_8b   32 layers x {2 x 4096x4096, 2 x 1024x4096, 2 x 14336x4096,
              4096x14336}, bf16 W/G/G_prev, fp32 A/M
Seeds: matrix j of workload c at step t uses 1000 c + 16 j + t.
Layered workloads give `layer_size`, the matrices per layer, so that a
leading slice of whole layers can be taken (smaller cases of the same shapes).
"""
import math

import torch

QUINTIC = (3.4445, -4.7750, 2.0315)


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian(shape, seed, device="cpu", dtype=torch.float32, std=1.0):
    g = _gen(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


def orthonormal(n, k, seed, device="cpu"):
    """n x k matrix with orthonormal columns (QR of a Gaussian), k <= n."""
    g = _gen(seed, device)
    a = torch.randn(n, k, generator=g, device=device, dtype=torch.float32)
    q, r = torch.linalg.qr(a)
    return q * torch.sign(torch.diagonal(r)).unsqueeze(0)


def with_spectrum(rows, cols, sigma, seed, device="cpu"):
    """U diag(sigma) V^T with random orthonormal U (rows x r), V (cols x r)."""
    sigma = torch.as_tensor(sigma, dtype=torch.float32, device=device)
    r = sigma.numel()
    U = orthonormal(rows, r, seed, device)
    V = orthonormal(cols, r, seed + 7919, device)
    return (U * sigma.unsqueeze(0)) @ V.T


def low_rank_plus_noise(rows, cols, seed, device="cpu", rank=16, noise=1e-3):
    """sum_{i<rank} 1/(i+1) u_i v_i^T + noise * N(0, 1)."""
    sig = torch.tensor([1.0 / (i + 1) for i in range(min(rank, rows, cols))])
    return with_spectrum(rows, cols, sig, seed, device) + gaussian((rows, cols), seed + 104729, device, std=noise)


def power_law(rows, cols, seed, device="cpu", scale=1e-3, exponent=1.0):
    """scale * U diag(i^-exponent) V^T, full rank."""
    r = min(rows, cols)
    sig = scale * torch.arange(1, r + 1, dtype=torch.float32) ** (-exponent)
    return with_spectrum(rows, cols, sig, seed, device)


def log_spectrum(rows, cols, kappa, seed, device="cpu"):
    """U diag(sigma) V^T with sigma log-spaced from 1 down to 1/kappa."""
    r = min(rows, cols)
    sig = torch.logspace(0.0, -math.log10(kappa), r)
    return with_spectrum(rows, cols, sig, seed, device)


def seed_of(config_index, j, t):
    return 1000 * config_index + 16 * j + t


# ---------------------------------------------------------------- workloads

def _layers(n, per_layer):
    out = []
    for _ in range(n):
        out.extend(per_layer)
    return out


WORKLOADS = {
    "tiny": dict(index=1, shapes=[(64, 128)], w_dtype=torch.float32, ns_dtype=torch.float32,
                 grad="gaussian", muon_steps=3,
                 hp=dict(mu=0.95, eta=0.02, **{"lambda": 0.0}, gamma=1.0, beta_a=0.9, alpha=0.0)),
    "gpt2_small": dict(index=2, shapes=_layers(12, [(768, 768)] * 4 + [(768, 3072), (3072, 768)]), layer_size=6,
                       w_dtype=torch.bfloat16, ns_dtype=torch.bfloat16, grad="rank16", muon_steps=3,
                       hp=dict(mu=0.95, eta=0.02, **{"lambda": 0.0}, gamma=1.0, beta_a=0.9, alpha=0.5)),
    "llama_430m": dict(index=3, shapes=_layers(24, [(1024, 1024)] * 4 + [(4096, 1024)] * 2 + [(1024, 4096)]),
                       layer_size=7,
                       w_dtype=torch.bfloat16, ns_dtype=torch.bfloat16, grad="power", muon_steps=3,
                       hp=dict(mu=0.95, eta=0.02, **{"lambda": 0.1}, gamma=1.0, beta_a=0.9, alpha=0.5)),
    "moe_gram": dict(index=4, shapes=[(2048, 768)] * 64 + [(768, 2048)] * 64 + [(16384, 2048)],
                     w_dtype=torch.float16, ns_dtype=torch.float16, grad="logspec", muon_steps=1,
                     hp=dict(mu=0.95, eta=0.02, **{"lambda": 0.0}, gamma=1.0, beta_a=0.9, alpha=0.5)),
    "llama3_8b": dict(index=5, shapes=_layers(32, [(4096, 4096)] * 2 + [(1024, 4096)] * 2 +
                                              [(14336, 4096)] * 2 + [(4096, 14336)]), layer_size=7,
                      w_dtype=torch.bfloat16, ns_dtype=torch.bfloat16, grad="power", muon_steps=3,
                      hp=dict(mu=0.95, eta=0.02, **{"lambda": 0.1}, gamma=1.0, beta_a=0.9, alpha=0.5)),
}


# Vector-valued parameters of the model families (updated with AdamW, not the
# orthogonalised step): embeddings, layer-norm weights and biases, biases.
def _gpt2_vectors():
    out = [(50257, 768), (1024, 768)]                       # token, position embeddings
    for _ in range(12):
        out += [(768,), (768,), (2304,), (768,), (768,), (768,), (3072,), (768,)]
    return out + [(768,), (768,)]                           # final layer norm


VECTOR_SHAPES = {"gpt2_small": _gpt2_vectors()}


def gradient(workload, j, t, rows, cols, device="cpu", kappa=1e3):
    """Gradient of matrix j at step t for a workload (fp32)."""
    w = WORKLOADS[workload]
    seed = seed_of(w["index"], j, t)
    kind = w["grad"]
    if kind == "gaussian":
        return gaussian((rows, cols), seed, device)
    if kind == "rank16":
        return low_rank_plus_noise(rows, cols, seed, device)
    if kind == "power":
        return power_law(rows, cols, seed, device)
    if kind == "logspec":
        return log_spectrum(rows, cols, kappa, seed, device)
    raise ValueError(kind)


def initial_weight(workload, j, rows, cols, device="cpu"):
    w = WORKLOADS[workload]
    seed = seed_of(w["index"], j, 15)
    std = 1.0 if workload == "tiny" else 0.02
    return gaussian((rows, cols), seed, device, std=std)


def tiny_sequence():
    """The tiny workload's draws from one generator seeded 0, in order:
    W0, G0, G1, G2 (each 64 x 128, N(0, 1))."""
    g = torch.Generator()
    g.manual_seed(0)
    return [torch.randn(64, 128, generator=g) for _ in range(4)]
