"""Synthetic workloads shaped like the decode layers the pages discuss (no method arithmetic).

Five workloads, each a single decode layer:

  tiny      1 seq, 1 q-head / 1 kv-head, d 128, ctx 1024, fp32; K ~ N(0,1) with 4 fixed key
            channels x20; V, q ~ N(0,1). Codec: 2-bit Lloyd-Max + 128-bit QJL on K and V.
  llama8b   batch 16, 32 q-heads / 8 kv-heads, d 128, ctx 8192, bf16; keys carry 6 fixed
            outlier channels per kv-head x15; V ~ N(0,1). Codec: 2-bit LM + QJL on K and V.
  llama70b  batch 64, 64 / 8 heads, d 128, ctx 32768, bf16; 8 key channels per kv-head drawn
            from Student-t(3), others N(0,1). Codec: K 3-bit LM + QJL, V 3-bit LM.
  onebit    batch 256, 32 / 8 heads, d 128, ctx 16384, bf16; K and V ~ N(0,1) times a fixed
            per-(kv-head, channel) scale, log-uniform in [0.1, 10], separate for K and V.
            Codec: rotation + one sign bit per coordinate + fp16 norm for K and V.
  mla_fp4   batch 1, 64 q-heads sharing one 512-dim latent (~N(0,1)) plus a 64-dim bf16 RoPE
            key per token, ctx 2^20; FP4 E2M1 latent, one E4M3 scale per 16 channels;
            absorbed query [64, 576] ~ N(0,1).

Seeds: data_seed = 0x5EED0000 + index, rot_seed = data_seed ^ 0xA5, qjl_seed = data_seed ^ 0x5A.
Bulk tensors are drawn per sequence with torch generators seeded from (data_seed, tensor, b),
so a caller can draw any subset of sequences on any device; values differ between CPU and CUDA
generators, so parity tests always hand the device tensors themselves to the oracle.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch

from .rng import rotation_signs, rotation_signs_per_head, qjl_matrix


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ctx: int
    dtype: str                 # "f32" or "bf16" (K, V and q)
    k_mode: str                # "lm_qjl" | "lm" | "sign1" | "fp4"
    v_mode: str
    k_bits: int
    v_bits: int
    qjl_dim: int
    key_structure: str         # "outlier" | "student_t" | "channel_scale" | "none"
    key_channels: int = 0      # channels per kv-head with the key structure
    key_factor: float = 1.0    # outlier multiplier
    latent_dim: int = 0
    rope_dim: int = 0
    rot_per_head: bool = False  # one rotation diagonal per KV head
    sink_tokens: int = 0        # mixed-precision window: first tokens kept in bf16
    recent_tokens: int = 0      # and last tokens kept in bf16
    paged: bool = False         # cache tiles in a shuffled pool of 64-token pages (block table)

    @property
    def data_seed(self) -> int:
        return 0x5EED0000 + self.index

    @property
    def rot_seed(self) -> int:
        return self.data_seed ^ 0xA5

    @property
    def qjl_seed(self) -> int:
        return self.data_seed ^ 0x5A

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 1, 1, 128, 1024, "f32", "lm_qjl", "lm_qjl", 2, 2, 128,
                     "outlier", 4, 20.0),
    "llama8b": Workload("llama8b", 1, 16, 32, 8, 128, 8192, "bf16", "lm_qjl", "lm_qjl", 2, 2,
                        128, "outlier", 6, 15.0),
    "llama70b": Workload("llama70b", 2, 64, 64, 8, 128, 32768, "bf16", "lm_qjl", "lm", 3, 3, 128,
                         "student_t", 8),
    "onebit": Workload("onebit", 3, 256, 32, 8, 128, 16384, "bf16", "sign1", "sign1", 1, 1, 0,
                       "channel_scale"),
    "mla_fp4": Workload("mla_fp4", 4, 1, 64, 1, 512, 1 << 20, "bf16", "fp4", "fp4", 4, 4, 0,
                        "none", 0, 1.0, 512, 64),
}


# Variants of the 8B-shaped layer for the codec features beside the main path: the KIVI-style codec,
# OSCAR's mixed-precision window (64 sink + 256 recent tokens in bf16: 0.24% of a 128k context), and
# a paged cache (pages of 64 tokens in a shuffled pool).
VARIANTS = {
    "llama8b_kivi": WORKLOADS["llama8b"].with_(name="llama8b_kivi", k_mode="kivi", v_mode="kivi", qjl_dim=0),
    "llama8b_window": WORKLOADS["llama8b"].with_(name="llama8b_window", sink_tokens=64, recent_tokens=256),
    "llama8b_paged": WORKLOADS["llama8b"].with_(name="llama8b_paged", paged=True),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name] if name in WORKLOADS else VARIANTS[name]


# ---- fixed per-(kv-head, channel) structure ------------------------------------------------

def key_channel_choice(w: Workload) -> np.ndarray:
    """[n_kv_heads, key_channels] channel indices carrying the key structure."""
    rng = np.random.Generator(np.random.PCG64(w.data_seed))
    return np.stack([rng.choice(w.head_dim, size=w.key_channels, replace=False)
                     for _ in range(w.n_kv_heads)]) if w.key_channels else \
        np.zeros((w.n_kv_heads, 0), dtype=np.int64)


def channel_scales(w: Workload, which: str) -> np.ndarray:
    """[n_kv_heads, head_dim] log-uniform scales in [0.1, 10] (which = "k" or "v")."""
    rng = np.random.Generator(np.random.PCG64([w.data_seed, 1 if which == "k" else 2]))
    return np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=(w.n_kv_heads, w.head_dim)))


def rotation_and_sketch(w: Workload):
    """The method's random draws for this workload: (signs int8 [d] -- or [n_kv_heads, d] with a
    per-head rotation --, S float32 [m, d] or None)."""
    signs = (rotation_signs_per_head(w.rot_seed, w.n_kv_heads, w.head_dim) if w.rot_per_head
             else rotation_signs(w.rot_seed, w.head_dim))
    S = qjl_matrix(w.qjl_seed, w.qjl_dim, w.head_dim) if w.qjl_dim else None
    return signs, S


# ---- bulk tensors ---------------------------------------------------------------------------

_TENSOR_IDS = {"k": 1, "v": 2, "q": 3, "latent": 4, "rope": 5, "k_new": 6, "v_new": 7,
               "latent_new": 8, "rope_new": 9}


def _gen(w: Workload, tensor: str, b: int, device, step: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((w.data_seed * 1_000_003 + _TENSOR_IDS[tensor] * 65_537 + b * 257 + step)
                  & 0x7FFFFFFFFFFFFFFF)
    return g


def _keys(w: Workload, b: int, T: int, device, tensor: str, step: int = 0) -> torch.Tensor:
    """One sequence's keys [Hkv, T, d] in fp32."""
    g = _gen(w, tensor, b, device, step)
    x = torch.randn((w.n_kv_heads, T, w.head_dim), generator=g, device=device)
    if w.key_structure == "outlier":
        ch = torch.as_tensor(key_channel_choice(w), device=device)
        for h in range(w.n_kv_heads):
            x[h, :, ch[h]] *= w.key_factor
    elif w.key_structure == "student_t":
        ch = torch.as_tensor(key_channel_choice(w), device=device)
        for h in range(w.n_kv_heads):
            zz = torch.randn((4, T, w.key_channels), generator=g, device=device)
            chi2 = (zz[1:] ** 2).sum(0)
            x[h, :, ch[h]] = zz[0] / torch.sqrt(chi2 / 3.0)
    elif w.key_structure == "channel_scale":
        x *= torch.as_tensor(channel_scales(w, "k"), dtype=torch.float32, device=device)[:, None, :]
    return x


def _values(w: Workload, b: int, T: int, device, tensor: str, step: int = 0) -> torch.Tensor:
    g = _gen(w, tensor, b, device, step)
    x = torch.randn((w.n_kv_heads, T, w.head_dim), generator=g, device=device)
    if w.key_structure == "channel_scale":
        x *= torch.as_tensor(channel_scales(w, "v"), dtype=torch.float32, device=device)[:, None, :]
    return x


def generate(w: Workload, device="cpu", seqs=None, ctx: int | None = None, step: int | None = None):
    """Synthetic tensors for the sequences ``seqs`` (default: all) of workload ``w``.

    ctx overrides the context length (tests use shorter contexts with the same
    distributions). With ``step`` given, draws instead the single new token that decode step
    ``step`` appends (K/V or latent/rope with T = 1).

    LM workloads -> {"k": [nb, Hkv, T, d], "v": same, "q": [nb, Hq, d]}
    MLA workload -> {"latent": [nb, T, C], "rope": [nb, T, R], "q": [nb, Hq, C + R]}
    All in the workload's dtype on ``device``.
    """
    seqs = list(range(w.batch)) if seqs is None else list(seqs)
    T = (w.ctx if ctx is None else ctx) if step is None else 1
    dt = w.torch_dtype
    st = 0 if step is None else step + 1
    if w.k_mode == "fp4":
        lat, rope, q = [], [], []
        for b in seqs:
            g = _gen(w, "latent" if step is None else "latent_new", b, device, st)
            lat.append(torch.randn((T, w.latent_dim), generator=g, device=device).to(dt))
            g = _gen(w, "rope" if step is None else "rope_new", b, device, st)
            rope.append(torch.randn((T, w.rope_dim), generator=g, device=device).to(dt))
            g = _gen(w, "q", b, device, st)
            q.append(torch.randn((w.n_q_heads, w.latent_dim + w.rope_dim), generator=g,
                                 device=device).to(dt))
        return {"latent": torch.stack(lat), "rope": torch.stack(rope), "q": torch.stack(q)}
    ks, vs, qs = [], [], []
    for b in seqs:
        ks.append(_keys(w, b, T, device, "k" if step is None else "k_new", st).to(dt))
        vs.append(_values(w, b, T, device, "v" if step is None else "v_new", st).to(dt))
        g = _gen(w, "q", b, device, st)
        qs.append(torch.randn((w.n_q_heads, w.head_dim), generator=g, device=device).to(dt))
    return {"k": torch.stack(ks), "v": torch.stack(vs), "q": torch.stack(qs)}
