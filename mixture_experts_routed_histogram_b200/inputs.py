"""Seeded synthetic inputs for the routed-expert MoE MLP workloads.

This module only draws random tensors and builds router logits from them; it holds none
of the method's arithmetic (no routing, permutation, quantisation or expert math).  Both
the CUDA path and the CPU oracle consume what it returns.

Workloads (shapes and value recipes):
  tiny            T=64, H=256, E=8, k=2, I=128, softmax top-2 renormalised.
  qwen3_30b_a3b   T=8192, H=2048, E=128, k=8, I=768, softmax top-8 renormalised
                  (shape of the Qwen3-30B-A3B rows of the Liger-Kernel PR #1463 benchmark).
  llama4_scout    T=8192, H=5120, E=16, k=1, I=8192, sigmoid weight of the top-1 logit
                  (shape of the Llama 4 Scout rows of the same benchmark).
  fp8_mxfp4       T in {128, 1024, 8192, 16384}, H=2560, E=512, k=10, I=640, softmax top-10
                  renormalised, uniform expert load (FlashInfer PR #6465 workload).
  decode          T in {1, 8, 32, 128, 256}, H=4096, E=8, k=2, I=14336, softmax top-2
                  renormalised, Zipf(1.2)-skewed expert choice with one expert never chosen.
  nemotron_relu2  T=8192, H=2688, E=128, k=6, I=1856, ReLU2 (non-gated squared ReLU, W1
                  [E, I, H]), softmax top-6 renormalised, gaussian routing: the
                  Nemotron-3.5-Lightning shape FlashInfer PR #5129 measures.
  qwen3_30b_a3b_shared1
                  the Qwen3-30B-A3B shape plus one shared expert (expert 128, weight 1 on
                  every token): the shared-expert fold at a realistic size.
  grid_d{D}_e{E}_k{k}
                  the parameter grid of the Liger-Kernel PR #1463 benchmark: T=8192,
                  H=I=D in {2048, 4096}, E in {8, 16, 32, 64, 128}, k in {1, 2, 4, 8} with
                  k < E (38 shapes), softmax top-k renormalised, gaussian routing.

Values: x ~ N(0,1) bf16; W13 ~ N(0, 1/H) and W2 ~ N(0, 1/I) bf16 (fan-in scaling).
Router logits:
  gaussian  logits = fp32(x) @ Wg, Wg ~ N(0, 1/H) fp32 [H, E]: near-uniform load.
  uniform   assignment a = t*k + j goes to expert a mod E: those k logits are
            8 + 0.5*U(0,1), the others N(0,1) clipped to [-3, 3]; per-expert counts then
            differ by at most one.
  zipf      a seeded permutation gives the experts ranks 1..E; logit = -1.2*ln(rank) +
            Gumbel(0,1) (so top-k samples k distinct experts with probability ~ rank^-1.2);
            the rank-E expert gets -1e4 so at least one expert is always empty.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    score: str = "softmax"       # "softmax" | "sigmoid"
    renorm: bool = True
    dtype: str = "bf16"          # "bf16" | "fp8_mxfp4"
    routing: str = "gaussian"    # "gaussian" | "uniform" | "zipf"
    act: str = "swiglu"          # "swiglu" (W13 [E, 2I, H]) | "relu2" (W1 [E, I, H])
    n_shared: int = 0            # shared experts E .. E+n_shared-1 (weights hold E + n_shared)

    def with_T(self, T: int) -> "Workload":
        return replace(self, T=T)

    @property
    def R(self) -> int:
        """Rows of the expert-sorted space: routed and shared slots of every token."""
        return self.T * (self.k + self.n_shared)

    @property
    def E_all(self) -> int:
        return self.E + self.n_shared

    @property
    def gemm1_rows(self) -> int:
        """Weight rows per expert of GEMM1: 2I (gate + up) or I (ReLU2)."""
        return self.I if self.act == "relu2" else 2 * self.I

    def flops(self) -> float:
        """Expert FLOPs of one forward pass: 2*H*(2I or I) (GEMM1) + 2*I*H (GEMM2) per row
        of the expert-sorted space (routed slots, plus the shared experts' when there are
        any; router, activation elementwise and combine excluded)."""
        return 2.0 * self.R * self.H * (self.gemm1_rows + self.I)


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 128, 8, 2),
    "qwen3_30b_a3b": Workload("qwen3_30b_a3b", 8192, 2048, 768, 128, 8),
    "llama4_scout": Workload("llama4_scout", 8192, 5120, 8192, 16, 1, score="sigmoid",
                             renorm=False),
    "fp8_mxfp4": Workload("fp8_mxfp4", 8192, 2560, 640, 512, 10, dtype="fp8_mxfp4",
                          routing="uniform"),
    "decode": Workload("decode", 32, 4096, 14336, 8, 2, routing="zipf"),
    "nemotron_relu2": Workload("nemotron_relu2", 8192, 2688, 1856, 128, 6, act="relu2"),
    "qwen3_30b_a3b_shared1": Workload("qwen3_30b_a3b_shared1", 8192, 2048, 768, 128, 8,
                                      n_shared=1),
}
GRID = {f"grid_d{d}_e{e}_k{k}": Workload(f"grid_d{d}_e{e}_k{k}", 8192, d, d, e, k)
        for d in (2048, 4096) for e in (8, 16, 32, 64, 128) for k in (1, 2, 4, 8) if k < e}
WORKLOADS.update(GRID)
FP8_T_SWEEP = (128, 1024, 8192, 16384)
DECODE_T_SWEEP = (1, 8, 32, 128, 256)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_x(wl: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(wl.T, wl.H, generator=g, device=device).to(torch.bfloat16)


def make_weights(wl: Workload, seed: int = 0, device="cpu"):
    """W13 bf16 [E, 2I, H] (gate rows then up rows; W1 [E, I, H] for ReLU2) and W2 bf16
    [E, H, I], drawn one expert at a time to bound the temporary fp32 memory."""
    g = _gen(seed + 1, device)
    w13 = torch.empty(wl.E_all, wl.gemm1_rows, wl.H, dtype=torch.bfloat16, device=device)
    w2 = torch.empty(wl.E_all, wl.H, wl.I, dtype=torch.bfloat16, device=device)
    s13, s2 = 1.0 / math.sqrt(wl.H), 1.0 / math.sqrt(wl.I)
    for e in range(wl.E_all):
        w13[e] = (torch.randn(wl.gemm1_rows, wl.H, generator=g, device=device) * s13).to(torch.bfloat16)
    for e in range(wl.E_all):
        w2[e] = (torch.randn(wl.H, wl.I, generator=g, device=device) * s2).to(torch.bfloat16)
    return w13, w2


# Synthetic MXFP4 weights are drawn directly as codes and scale bytes (no quantiser runs
# here): magnitudes of the e2m1 codes 0..7 (values 0, .5, 1, 1.5, 2, 3, 4, 6) follow this
# table, the sign is a fair coin, and each 32-element block's UE8M0 byte is
# 127 + floor(log2(1/sqrt(fan_in))) - 2 + U{0,1,2}, so values have about the spread of
# N(0, 1/fan_in) weights.
E2M1_MAGNITUDE_PROBS = (0.16, 0.30, 0.20, 0.13, 0.10, 0.07, 0.03, 0.01)


def _mx_block(rows: int, K: int, fan_in: int, g: torch.Generator, device):
    probs = torch.tensor(E2M1_MAGNITUDE_PROBS, device=device)
    mag = torch.multinomial(probs, rows * K, replacement=True, generator=g).to(torch.uint8)
    sign = torch.randint(0, 2, (rows * K,), generator=g, device=device, dtype=torch.uint8) << 3
    codes = (mag | sign).view(rows, K // 2, 2)
    packed = (codes[..., 0] | (codes[..., 1] << 4)).contiguous()
    b0 = 127 + math.floor(math.log2(1.0 / math.sqrt(fan_in))) - 2
    sf = (b0 + torch.randint(0, 3, (rows, K // 32), generator=g, device=device)).to(torch.uint8)
    return packed, sf


def make_weights_mxfp4(wl: Workload, seed: int = 0, device="cpu"):
    """MXFP4 W13 (packed [E, 2I, H/2] + scales [E, 2I, H/32]) and W2 (packed [E, H, I/2] +
    scales [E, H, I/32]), element 2i in the low nibble of byte i."""
    g = _gen(seed + 3, device)
    w13p = torch.empty(wl.E_all, 2 * wl.I, wl.H // 2, dtype=torch.uint8, device=device)
    w13s = torch.empty(wl.E_all, 2 * wl.I, wl.H // 32, dtype=torch.uint8, device=device)
    w2p = torch.empty(wl.E_all, wl.H, wl.I // 2, dtype=torch.uint8, device=device)
    w2s = torch.empty(wl.E_all, wl.H, wl.I // 32, dtype=torch.uint8, device=device)
    for e in range(wl.E_all):
        w13p[e], w13s[e] = _mx_block(2 * wl.I, wl.H, wl.H, g, device)
        w2p[e], w2s[e] = _mx_block(wl.H, wl.I, wl.I, g, device)
    return w13p, w13s, w2p, w2s


def make_logits(wl: Workload, x: torch.Tensor, seed: int = 0) -> torch.Tensor:
    """Router logits fp32 [T, E] per the workload's routing recipe."""
    device = x.device
    g = _gen(seed + 2, device)
    T, E, k = wl.T, wl.E, wl.k
    if wl.routing == "gaussian":
        wg = torch.randn(wl.H, E, generator=g, device=device) / math.sqrt(wl.H)
        prev = torch.backends.cuda.matmul.allow_tf32
        torch.backends.cuda.matmul.allow_tf32 = False
        try:
            return (x.float() @ wg).contiguous()
        finally:
            torch.backends.cuda.matmul.allow_tf32 = prev
    if wl.routing == "uniform":
        lg = torch.randn(T, E, generator=g, device=device).clamp_(-3.0, 3.0)
        a = torch.arange(T * k, device=device)
        tok, ex = a // k, a % E
        lg[tok, ex] = 8.0 + 0.5 * torch.rand(T * k, generator=g, device=device)
        return lg.contiguous()
    if wl.routing == "zipf":
        perm = torch.randperm(E, generator=g, device=device)
        rank = torch.empty(E, device=device)
        rank[perm] = torch.arange(1, E + 1, device=device, dtype=torch.float32)
        u = torch.rand(T, E, generator=g, device=device).clamp_(1e-12, 1.0 - 1e-7)
        gumbel = -torch.log(-torch.log(u))
        lg = -1.2 * torch.log(rank)[None, :] + gumbel
        lg[:, perm[E - 1]] = -1e4
        return lg.contiguous()
    raise ValueError(wl.routing)


def make_inputs(wl: Workload, seed: int = 0, device="cpu", weights: bool = True) -> dict:
    """x, logits and the weights in the workload's format (bf16, or MXFP4 codes + scales
    under keys w13, w13_sf, w2, w2_sf)."""
    x = make_x(wl, seed, device)
    out = {"x": x, "logits": make_logits(wl, x, seed), "w13_sf": None, "w2_sf": None}
    if weights:
        if wl.dtype == "fp8_mxfp4":
            out["w13"], out["w13_sf"], out["w2"], out["w2_sf"] = make_weights_mxfp4(wl, seed, device)
        else:
            out["w13"], out["w2"] = make_weights(wl, seed, device)
    return out


def parity_tokens(T: int, n: int = 256, seed: int = 0) -> np.ndarray:
    """Seeded token subset for oracle checks at large T: n tokens without replacement,
    always including 0 and T-1, sorted."""
    if T <= n:
        return np.arange(T, dtype=np.int64)
    rng = np.random.default_rng(seed)
    pick = rng.choice(np.arange(1, T - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, T - 1], pick])).astype(np.int64)


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (moved to host)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(b: np.ndarray) -> torch.Tensor:
    """bf16 tensor from uint16 bit patterns."""
    return torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
