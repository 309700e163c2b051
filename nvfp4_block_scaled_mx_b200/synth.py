"""Seeded synthetic inputs for the microscaling W4A4 linear layer.

This module holds no quantization or GEMM arithmetic: it only draws activations ``A [M, K]`` and
weights ``W [N, K]`` (nn.Linear layout) as bf16 tensors with the shapes and value distributions of
the serving workloads (hidden size 5120, MLP width 17408 with fused gate+up 34816, attention
projection 7168, vocabulary-sized lm_head 151936).  Both the CUDA path and the CPU oracle consume
the same bytes, so the generator itself does not affect parity.

Recipes (all fp32 samples rounded to bf16 with round-to-nearest-even by ``Tensor.to``):
  normal       N(0, std)
  student_t3   0.5 * Z / sqrt(chi2_3 / 3)           (heavy-tailed decode activations)
  silu         z * sigmoid(z), z ~ N(0, 1)          (post-activation skew of a down projection)
  outliers     a seeded permutation picks round(frac * K) channels, scaled by `factor` for all rows
"""
import torch

# name -> problem description.  fmt: "mxfp4" | "nvfp4" | "mxfp8"; rules apply to MX formats.
CONFIGS = {
    "tiny": dict(seed=0, M=16, N=256, K=256, fmt="mxfp4", a_rule="ceil", w_rule="even", out="fp32",
                 a=dict(kind="normal", std=1.0), w=dict(kind="normal", std=0.02)),
    "decode": dict(seed=1, M=32, N=5120, K=5120, fmt="mxfp4", a_rule="ceil", w_rule="even", out="bf16",
                   a=dict(kind="student_t3", outlier_frac=0.001, outlier_factor=50.0),
                   w=dict(kind="normal", std=0.02)),
    "prefill_gate_up": dict(seed=2, M=8192, N=34816, K=5120, fmt="mxfp4", a_rule="ceil", w_rule="even",
                            out="bf16", a=dict(kind="normal", std=1.0, outlier_frac=0.01, outlier_factor=20.0),
                            w=dict(kind="normal", std=0.02)),
    "down_nvfp4": dict(seed=3, M=8192, N=5120, K=17408, fmt="nvfp4", a_rule="even", w_rule="even",
                       out="bf16", a=dict(kind="silu"), w=dict(kind="normal", std=0.015)),
    "attn_mxfp8": dict(seed=4, M=8192, N=7168, K=5120, fmt="mxfp8", a_rule="even", w_rule="even",
                       out="bf16", a=dict(kind="normal", std=1.0), w=dict(kind="normal", std=0.02)),
    "lm_head": dict(seed=4, M=2048, N=151936, K=5120, fmt="mxfp4", a_rule="ceil", w_rule="even",
                    out="bf16", a=dict(kind="normal", std=1.0), w=dict(kind="normal", std=0.02),
                    stream=1),
    # fused in_proj_a/in_proj_b of the linear-attention blocks: N = 48 + 48 = 96 (MXFP8)
    "in_proj_ba": dict(seed=5, M=8192, N=96, K=5120, fmt="mxfp8", a_rule="even", w_rule="even", out="bf16",
                       a=dict(kind="normal", std=1.0), w=dict(kind="normal", std=0.02)),
}

_CHUNK_ROWS = 4096


def _draw(rows, K, gen, device, kind, std=1.0, **_):
    if kind == "normal":
        return torch.randn(rows, K, generator=gen, device=device) * std
    if kind == "student_t3":
        z = torch.randn(rows, K, generator=gen, device=device)
        chi2 = torch.randn(3, rows, K, generator=gen, device=device).square().sum(0)
        return 0.5 * z / torch.sqrt(chi2 / 3.0)
    if kind == "silu":
        z = torch.randn(rows, K, generator=gen, device=device)
        return z * torch.sigmoid(z)
    raise ValueError(kind)


def draw_matrix(rows, K, spec, gen, device="cpu"):
    """One bf16 [rows, K] matrix per `spec`, drawn in row chunks to bound fp32 scratch."""
    out = torch.empty(rows, K, dtype=torch.bfloat16, device=device)
    for r0 in range(0, rows, _CHUNK_ROWS):
        r1 = min(rows, r0 + _CHUNK_ROWS)
        out[r0:r1] = _draw(r1 - r0, K, gen, device, **spec).to(torch.bfloat16)
    frac = spec.get("outlier_frac", 0.0)
    if frac > 0:
        n_out = int(round(frac * K))
        perm = torch.randperm(K, generator=gen, device=device)
        ch = perm[:n_out]
        out[:, ch] = (out[:, ch].float() * spec["outlier_factor"]).to(torch.bfloat16)
    return out


def make_generator(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_inputs(name, device="cpu", M=None, N=None, K=None, seed=None):
    """Draw (A, W) for a named problem; M/N/K/seed may be overridden for parity sweeps."""
    cfg = dict(CONFIGS[name])
    M = cfg["M"] if M is None else M
    N = cfg["N"] if N is None else N
    K = cfg["K"] if K is None else K
    seed = cfg["seed"] if seed is None else seed
    gen = make_generator(seed * 1000 + cfg.get("stream", 0), device)
    A = draw_matrix(M, K, cfg["a"], gen, device)
    W = draw_matrix(N, K, cfg["w"], gen, device)
    return A, W


def random_bf16(shape, seed, std=1.0, device="cpu"):
    gen = make_generator(seed, device)
    return (torch.randn(*shape, generator=gen, device=device) * std).to(torch.bfloat16)
