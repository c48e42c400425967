"""Seeded synthetic workloads for the GDLA forward pass.

This module only draws random tensors of the right shapes and names the
workloads; it holds none of the layer's arithmetic, so the CUDA path and the
fp64 oracle can both be fed from it.

Shapes follow the GDLA statement in "Motif 3: Technical Report", section
"Architecture": a compressed KV latent of width d_c, a decoupled rotary key of
width d_R, n_kv shared key/value heads, g*n_N signal and n_N = n_kv noise query
heads of width d_n + d_R, and value width d_v. The five named workloads are the
parity and throughput cases used by the tests and the benchmark.

Value recipe (every tensor from one seeded torch generator, drawn in a fixed
order):
  * weights: W_UKV ~ N(0,1)/sqrt(d_c); gamma = 1 + 0.1*N(0,1) (a non-trivial
    RMSNorm gain, so a kernel that ignores it fails parity);
  * activations c_KV, k_R, q: N(0,1) * s, with s = 1 ("unit": realistic,
    peaked attention) or s = 1/sqrt(last dim) ("fan_in": the literal reading,
    near-uniform attention);
  * lambda logits and gate logits: N(0,1).
The decode cache holds the normalised latent and the rotated rotary key, which
are drawn directly (see ``make_decode_inputs``).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    L: int
    d_c: int = 512
    d_R: int = 64
    n_kv: int = 16
    d_n: int = 128
    d_v: int = 128
    g: int = 2
    d_q: int = 1536
    dtype: str = "bf16"
    mask: str = "causal"
    window: int = 0

    @property
    def n_N(self) -> int:
        return self.n_kv

    @property
    def n_S(self) -> int:
        return self.g * self.n_kv

    @property
    def H_q(self) -> int:
        return self.n_S + self.n_N

    @property
    def d_qk(self) -> int:
        return self.d_n + self.d_R

    def pairs_per_row_sum(self) -> int:
        """Visible (query, key) pairs of one sequence under the mask."""
        L, W = self.L, self.window
        if self.mask == "sliding" and W < L:
            return W * (W + 1) // 2 + (L - W) * W
        return L * (L + 1) // 2

    def algorithmic_flops(self) -> float:
        """Work the method must do: the expansion GEMM plus QK and PV over the
        visible pairs of every query head. Masked tiles earn nothing."""
        expand = 2.0 * self.B * self.L * self.d_c * self.n_kv * (self.d_n + self.d_v)
        attn = 2.0 * (self.d_qk + self.d_v) * self.pairs_per_row_sum() * self.H_q * self.B
        return expand + attn


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    T: int
    d_c: int = 512
    d_R: int = 64
    n_kv: int = 16
    d_n: int = 128
    d_v: int = 128
    g: int = 2
    dtype: str = "bf16"
    mask: str = "causal"
    window: int = 0

    @property
    def n_N(self) -> int:
        return self.n_kv

    @property
    def n_S(self) -> int:
        return self.g * self.n_kv

    @property
    def H_q(self) -> int:
        return self.n_S + self.n_N

    @property
    def d_qk(self) -> int:
        return self.d_n + self.d_R

    def algorithmic_bytes(self, seqlens=None) -> float:
        """Bytes the method must move: the latent cache read once, W_UKV, and the
        per-token query, lambda, gate and output."""
        esz = 4 if self.dtype == "fp32" else 2
        tokens = self.B * self.T if seqlens is None else int(sum(int(s) for s in seqlens))
        cache = tokens * (self.d_c + self.d_R) * esz
        w = self.d_c * self.n_kv * (self.d_n + self.d_v) * esz
        q = self.B * self.H_q * self.d_qk * esz
        lam = self.B * self.n_S * 4
        gate = self.B * self.n_S * self.d_v * esz
        out = self.B * self.n_S * self.d_v * esz
        return float(cache + w + q + lam + gate + out + self.B * 4)


# The named workloads (sizes as the tests and the benchmark use them).
PREFILL = {
    "tiny_fp32": PrefillShape("tiny fp32 prefill, causal, B=1 L=128 d_c=64 d_R=16 n_kv=4 d=32 g=2",
                              B=1, L=128, d_c=64, d_R=16, n_kv=4, d_n=32, d_v=32, g=2, d_q=64, dtype="fp32"),
    "b4_l4k_g2": PrefillShape("bf16 prefill, causal, B=4 L=4096 g=2", B=4, L=4096, g=2),
    "b1_l32k_g3": PrefillShape("bf16 prefill, causal, B=1 L=32768 g=3", B=1, L=32768, g=3),
    # the same kernel configuration at a size a full counter capture replays quickly
    "b2_l8k_g3": PrefillShape("bf16 prefill, causal, B=2 L=8192 g=3", B=2, L=8192, g=3),
    "b2_l64k_swa4k": PrefillShape("bf16 prefill, sliding window W=4096, B=2 L=65536 g=2", B=2, L=65536, g=2,
                                  mask="sliding", window=4096),
    # the report's own attention layout: 16 KV heads with g = 4 (80 query heads); its
    # sliding layers use a 128-token window
    "b1_l32k_g4_swa128": PrefillShape("bf16 prefill, sliding window W=128, B=1 L=32768 g=4 (80 heads)", B=1,
                                      L=32768, g=4, mask="sliding", window=128),
    "b1_l32k_g4": PrefillShape("bf16 prefill, causal, B=1 L=32768 g=4 (80 heads)", B=1, L=32768, g=4),
}
DECODE = {
    "b64_t32k": DecodeShape("bf16 decode, B=64, 32768-token latent cache, g=2", B=64, T=32768, g=2),
    # a quarter-size case for profiler captures (0.6 GB of cache, still far above L2)
    "b16_t32k": DecodeShape("bf16 decode, B=16, 32768-token latent cache, g=2", B=16, T=32768, g=2),
    # the report's 80 query heads (g = 4) over the same cache
    "b64_t32k_g4": DecodeShape("bf16 decode, B=64, 32768-token latent cache, g=4 (80 heads)", B=64, T=32768, g=4),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen, device, scale=1.0, dtype=torch.float32):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_prefill_inputs(shape: PrefillShape, seed: int = 0, device="cpu", act: str = "unit", **override):
    """Random prefill inputs for ``shape`` (dict of tensors on ``device``).

    Keys: c_kv [B,L,d_c], gamma [d_c], k_rope [B,L,d_R],
    q [B,L,n_S+n_N,d_n+d_R] (signal heads first, then noise; nope part then
    pre-RoPE rotary part), w_ukv [d_c, n_kv*(d_n+d_v)], lam_logits [B,L,n_S]
    (fp32 always), gate_logits [B,L,n_S,d_v].
    """
    s = dataclasses.replace(shape, **override) if override else shape
    dt = torch_dtype(s.dtype)
    gen = _gen(seed, device)

    def act_scale(fan):
        return 1.0 if act == "unit" else 1.0 / math.sqrt(fan)

    out = {}
    out["w_ukv"] = _randn((s.d_c, s.n_kv * (s.d_n + s.d_v)), gen, device, 1.0 / math.sqrt(s.d_c), dt)
    gam = _randn((s.d_c,), gen, device, 0.1)
    out["gamma"] = (gam + 1.0).to(dt)
    out["c_kv"] = _randn((s.B, s.L, s.d_c), gen, device, act_scale(s.d_c), dt)
    out["k_rope"] = _randn((s.B, s.L, s.d_R), gen, device, act_scale(s.d_R), dt)
    out["q"] = _randn((s.B, s.L, s.H_q, s.d_qk), gen, device, act_scale(s.d_qk), dt)
    out["lam_logits"] = _randn((s.B, s.L, s.n_S), gen, device, 1.0, torch.float32)
    out["gate_logits"] = _randn((s.B, s.L, s.n_S, s.d_v), gen, device, 1.0, dt)
    return out


def make_gate_inputs(shape: PrefillShape, d_x: int = 2048, seed: int = 0, device="cpu"):
    """Random inputs of the gate and lambda projections for the token layout of
    ``shape``: c_q [B,L,d_q] (query latent), gamma_q [d_q] = 1 + 0.1 N(0,1),
    w_g [d_q, n_S*d_v] ~ N(0,1)/sqrt(d_q), x [B,L,d_x] (layer input; its width is
    the caller's), w_lambda [d_x, n_S] ~ N(0,1)/sqrt(d_x)."""
    dt = torch_dtype(shape.dtype)
    gen = _gen(seed, device)
    out = {}
    out["c_q"] = _randn((shape.B, shape.L, shape.d_q), gen, device, 1.0, dt)
    out["gamma_q"] = (_randn((shape.d_q,), gen, device, 0.1) + 1.0).to(dt)
    out["w_g"] = _randn((shape.d_q, shape.n_S * shape.d_v), gen, device, 1.0 / math.sqrt(shape.d_q), dt)
    out["x"] = _randn((shape.B, shape.L, d_x), gen, device, 1.0, dt)
    out["w_lambda"] = _randn((d_x, shape.n_S), gen, device, 1.0 / math.sqrt(d_x), dt)
    return out


def make_decode_inputs(shape: DecodeShape, seed: int = 0, device="cpu", act: str = "fan_in", seqlens=None):
    """Random decode inputs for ``shape`` (dict of tensors on ``device``).

    Keys: c_cache [B,T,d_c] (stands for the normalised latent), kr_cache
    [B,T,d_R] (stands for the rotated rotary key), q [B,n_S+n_N,d_n+d_R]
    (rotary part pre-RoPE), w_ukv, lam_logits [B,n_S] fp32, gate_logits
    [B,n_S,d_v], seqlens [B] int32.

    With act="fan_in" the cache rows are N(0,1)/sqrt(d_c+d_R) (the literal
    N(0,1)/sqrt(fan_in) recipe with the 576-wide cache row as fan-in); with
    act="unit" they are N(0,1) so the softmax is peaked. q is N(0,1).
    """
    s = shape
    dt = torch_dtype(s.dtype)
    gen = _gen(seed, device)
    cs = 1.0 if act == "unit" else 1.0 / math.sqrt(s.d_c + s.d_R)
    out = {}
    out["w_ukv"] = _randn((s.d_c, s.n_kv * (s.d_n + s.d_v)), gen, device, 1.0 / math.sqrt(s.d_c), dt)
    out["c_cache"] = _randn((s.B, s.T, s.d_c), gen, device, cs, dt)
    out["kr_cache"] = _randn((s.B, s.T, s.d_R), gen, device, cs, dt)
    out["q"] = _randn((s.B, s.H_q, s.d_qk), gen, device, 1.0, dt)
    out["lam_logits"] = _randn((s.B, s.n_S), gen, device, 1.0, torch.float32)
    out["gate_logits"] = _randn((s.B, s.n_S, s.d_v), gen, device, 1.0, dt)
    if seqlens is None:
        seqlens = [s.T] * s.B
    out["seqlens"] = torch.tensor(list(seqlens), dtype=torch.int32, device=device)
    return out


def sample_rows(shape: PrefillShape, n_random: int = 32, seed: int = 1):
    """Deterministic query rows (b, i) for sampled parity at full size: rows
    0, 1, 127, 128, W-1, W, W+1 (sliding), L-1 and ``n_random`` seeded rows,
    spread over the batch."""
    L = shape.L
    fixed = [0, 1, 127, 128, L - 1]
    if shape.mask == "sliding":
        fixed += [shape.window - 1, shape.window, shape.window + 1]
    gen = torch.Generator().manual_seed(seed)
    rnd = torch.randint(0, L, (n_random,), generator=gen).tolist()
    rows = []
    for b in range(shape.B):
        for i in fixed:
            if 0 <= i < L:
                rows.append((b, i))
    bsel = torch.randint(0, shape.B, (n_random,), generator=gen).tolist()
    rows += list(zip(bsel, rnd))
    rows = sorted(set(rows))
    return rows
