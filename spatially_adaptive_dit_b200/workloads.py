"""Seeded synthetic workloads for the spatially adaptive DiT attention path.

This module only *draws inputs*: shapes, sizes, value distributions and
structure of the workloads the SAFE-DiT pages evaluate (Lumina-Next style
generations at 1024^2 / 2560^2 / 3072^2, text prompts with padding), and
nothing of the method's arithmetic.  Both the CUDA path and the fp64 oracle
are fed from here; neither implements anything in this file.

Recipe (all draws from a torch.Generator seeded with 1234 + config id, with a
per-tensor offset so that tensors are independent):
  * Q, K, V and the cross-attention tensors: N(0, 1) in fp32, rounded to bf16
    with round-to-nearest-even (torch's cast);
  * text validity: the first `n_valid` of L text positions are valid, the rest
    are padding; content tokens are the valid positions except the first
    (BOS-like) and the last valid one (EOS-like);
  * CFG predictions eps_c, eps_u: N(0, 1) fp32, [N, F];
  * masks: all-zero; per-row constant c_i ~ U(-4, 4); text-padding style
    (trailing 1/8 of the keys -inf, else 0); non-uniform bias N(0, 1);
  * clustered scores: 8 Gaussian blobs on the sqrt(N) x sqrt(N) grid, centres
    U over the grid, sigma ~ U(4, 16) patches, amplitude U(0.5, 1), plus
    1e-3 * U(0, 1) noise;
  * FFN block (model width D = H d, hidden width F = ffn_mult D): token
    states N(0,1) [B, N, D] bf16; W1 [F, D] and W2 [D, F] N(0,1) / sqrt(fan_in)
    (random init, nn.Linear layout), biases N(0, 0.02^2) fp32; the cached FFN
    output of the previous step N(0,1) [B, N, D] bf16; the fused Q|K|V
    projection W_qkv [3D, D] N(0,1) / sqrt(D) bf16 with bias N(0, 0.02^2).
"""
from dataclasses import dataclass, field
from fractions import Fraction
import math

import torch

SEED_BASE = 1234


@dataclass(frozen=True)
class Workload:
    name: str
    cid: int            # config id (seed offset)
    B: int              # batch (b=0 cond, b=1 uncond when B == 2)
    H: int              # heads
    N: int              # image tokens
    d: int              # head dim
    L: int              # text length
    n_valid: int        # valid text positions (prefix)
    rho: Fraction       # sensitive fraction |S| / N
    grid: int           # sqrt(N)
    F: int = 16         # per-token prediction width for CFG
    gamma_ctx: float = 3.0
    gamma_sens: float = 5.0
    warmup: int = 1     # dense warm-up steps feeding the partition
    period: int = 5     # anchor period
    steps: int = 10     # denoising steps in one trajectory
    fp32_inputs: bool = False
    rho_sweep: tuple = field(default_factory=tuple)
    ffn_mult: int = 4   # FFN hidden width / model width

    @property
    def D_model(self) -> int:
        return self.H * self.d

    @property
    def D_ff(self) -> int:
        return self.ffn_mult * self.H * self.d

    @property
    def k(self) -> int:
        """|S| = round-half-up(rho * N), computed exactly."""
        return k_of(self.rho, self.N)


def k_of(rho, N: int) -> int:
    x = Fraction(rho) * N
    return int(math.floor(x + Fraction(1, 2)))


TINY = Workload("tiny", 0, B=1, H=2, N=256, d=64, L=32, n_valid=20, rho=Fraction(1, 4), grid=16,
                warmup=2, period=3, steps=4, fp32_inputs=True)
W1024 = Workload("1024", 1, B=2, H=24, N=4096, d=96, L=256, n_valid=128, rho=Fraction(3, 10), grid=64)
W2560 = Workload("2560", 2, B=2, H=24, N=25600, d=96, L=256, n_valid=128, rho=Fraction(3, 10), grid=160,
                 warmup=1, period=5, steps=10)
W3072 = Workload("3072", 3, B=2, H=24, N=36864, d=96, L=256, n_valid=160, rho=Fraction(3, 10), grid=192,
                 rho_sweep=(Fraction(1, 10), Fraction(2, 10), Fraction(3, 10), Fraction(5, 10), Fraction(1)))
STRESS = Workload("stress", 4, B=1, H=32, N=16384, d=128, L=256, n_valid=128, rho=Fraction(3, 10), grid=128)

ALL = {w.name: w for w in (TINY, W1024, W2560, W3072, STRESS)}


def _gen(w: Workload, offset: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(SEED_BASE + w.cid + 7919 * offset)
    return g


def normal(shape, w: Workload, offset: int, device="cpu", dtype=torch.bfloat16):
    """N(0,1) drawn in fp32 then rounded to `dtype` (RNE)."""
    g = _gen(w, offset, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return x if dtype == torch.float32 else x.to(dtype)


def uniform(shape, lo, hi, w: Workload, offset: int, device="cpu", dtype=torch.float32):
    g = _gen(w, offset, device)
    x = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    return (lo + (hi - lo) * x).to(dtype)


# Tensor offsets (kept distinct so every tensor is an independent draw).
OFF_Q, OFF_K, OFF_V, OFF_QX, OFF_KTXT, OFF_KS, OFF_VS, OFF_EPSC, OFF_EPSU = range(1, 10)
OFF_MASK_ROW, OFF_MASK_BIAS, OFF_BLOB = 20, 21, 22
OFF_X, OFF_W1, OFF_B1, OFF_W2, OFF_B2, OFF_YCACHE, OFF_WQKV, OFF_BQKV = 30, 31, 32, 33, 34, 35, 36, 37
STEP_STRIDE = 100


def qkv(w: Workload, step: int = 0, device="cpu"):
    """Self-attention Q, K, V [B,H,N,d] bf16 for one denoising step."""
    o = STEP_STRIDE * step
    shape = (w.B, w.H, w.N, w.d)
    return (normal(shape, w, OFF_Q + o, device), normal(shape, w, OFF_K + o, device),
            normal(shape, w, OFF_V + o, device))


def fresh_sensitive_kv(w: Workload, k: int, step: int, device="cpu"):
    """Fresh K, V of the sensitive rows only, compact [B,H,k,d] bf16 (the
    projections of an SRSU step run on the S rows alone)."""
    o = STEP_STRIDE * step
    shape = (w.B, w.H, k, w.d)
    return normal(shape, w, OFF_KS + o, device), normal(shape, w, OFF_VS + o, device)


def text(w: Workload, step: int = 0, device="cpu"):
    """Cross-attention inputs: image queries [B,H,N,d], text keys [B,H,L,d]
    (bf16), key validity [B,L] uint8, content flags [L] uint8."""
    o = STEP_STRIDE * step
    q_img = normal((w.B, w.H, w.N, w.d), w, OFF_QX + o, device)
    k_txt = normal((w.B, w.H, w.L, w.d), w, OFF_KTXT + o, device)
    key_valid = torch.zeros((w.B, w.L), dtype=torch.uint8, device=device)
    key_valid[:, : w.n_valid] = 1
    content = torch.zeros((w.L,), dtype=torch.uint8, device=device)
    content[1: w.n_valid - 1] = 1
    return q_img, k_txt, key_valid, content


def cfg_preds(w: Workload, step: int = 0, device="cpu", F=None):
    """Conditional / unconditional noise predictions [N, F] fp32."""
    o = STEP_STRIDE * step
    F = w.F if F is None else F
    return (normal((w.N, F), w, OFF_EPSC + o, device, torch.float32),
            normal((w.N, F), w, OFF_EPSU + o, device, torch.float32))


MASK_KINDS = ("zero", "rowconst", "textpad", "bias")


def mask(w: Workload, kind: str, device="cpu", dtype=torch.bfloat16, rows=None):
    """Additive image self-attention mask [1,1,N,N] (or only `rows` of it,
    [1,1,len(rows),N], for sampled checks).  Kinds: 'zero' (all valid),
    'rowconst' (c_i ~ U(-4,4) along each row), 'textpad' (trailing 1/8 of
    the keys -inf), 'bias' (N(0,1) everywhere)."""
    N = w.N
    nr = N if rows is None else len(rows)
    if kind == "zero":
        m = torch.zeros((nr, N), device=device, dtype=dtype)
    elif kind == "rowconst":
        c = uniform((N, 1), -4.0, 4.0, w, OFF_MASK_ROW, device)
        if rows is not None:
            c = c[torch.as_tensor(rows, device=c.device)]
        m = c.expand(nr, N).to(dtype).contiguous()
    elif kind == "textpad":
        m = torch.zeros((nr, N), device=device, dtype=dtype)
        m[:, N - N // 8:] = float("-inf")
    elif kind == "bias":
        if rows is None:
            m = normal((N, N), w, OFF_MASK_BIAS, device, dtype)
        else:
            full = normal((N, N), w, OFF_MASK_BIAS, device, dtype)
            m = full[torch.as_tensor(rows, device=full.device)].contiguous()
    else:
        raise ValueError(kind)
    return m.view(1, 1, nr, N)


def blob_scores(w: Workload, device="cpu"):
    """Clustered Gaussian-blob score field [N] fp64 on the grid (row-major)."""
    G = w.grid
    g = _gen(w, OFF_BLOB, "cpu")
    nb = 8
    cx = torch.rand(nb, generator=g, dtype=torch.float64) * G
    cy = torch.rand(nb, generator=g, dtype=torch.float64) * G
    sig = 4.0 + 12.0 * torch.rand(nb, generator=g, dtype=torch.float64)
    amp = 0.5 + 0.5 * torch.rand(nb, generator=g, dtype=torch.float64)
    noise = 1e-3 * torch.rand(G * G, generator=g, dtype=torch.float64)
    yy, xx = torch.meshgrid(torch.arange(G, dtype=torch.float64), torch.arange(G, dtype=torch.float64),
                            indexing="ij")
    field = torch.zeros((G, G), dtype=torch.float64)
    for b in range(nb):
        field += amp[b] * torch.exp(-((xx - cx[b]) ** 2 + (yy - cy[b]) ** 2) / (2 * sig[b] ** 2))
    return (field.reshape(-1) + noise).to(device)


def ffn_weights(w: Workload, device="cpu", D=None, F=None):
    """FFN parameters: W1 [F, D], W2 [D, F] bf16 (N(0,1)/sqrt(fan_in), rounded
    after scaling), b1 [F], b2 [D] fp32 N(0, 0.02^2)."""
    D = w.D_model if D is None else D
    F = w.D_ff if F is None else F
    w1 = (normal((F, D), w, OFF_W1, device, torch.float32) / math.sqrt(D)).to(torch.bfloat16)
    w2 = (normal((D, F), w, OFF_W2, device, torch.float32) / math.sqrt(F)).to(torch.bfloat16)
    b1 = 0.02 * normal((F,), w, OFF_B1, device, torch.float32)
    b2 = 0.02 * normal((D,), w, OFF_B2, device, torch.float32)
    return w1, b1, w2, b2


def ffn_states(w: Workload, step: int = 0, device="cpu", D=None):
    """Token states entering the FFN [B, N, D] bf16 and the FFN cache of the
    previous step [B, N, D] bf16."""
    D = w.D_model if D is None else D
    o = STEP_STRIDE * step
    return (normal((w.B, w.N, D), w, OFF_X + o, device),
            normal((w.B, w.N, D), w, OFF_YCACHE + o, device))


def qkv_proj_weights(w: Workload, device="cpu", D=None):
    """Fused Q|K|V projection: W_qkv [3D, D] bf16 (N(0,1)/sqrt(D)), b [3D]
    fp32 N(0, 0.02^2); output features ordered (q|k|v, head, d)."""
    D = w.D_model if D is None else D
    wq = (normal((3 * D, D), w, OFF_WQKV, device, torch.float32) / math.sqrt(D)).to(torch.bfloat16)
    bq = 0.02 * normal((3 * D,), w, OFF_BQKV, device, torch.float32)
    return wq, bq
