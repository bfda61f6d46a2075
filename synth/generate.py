"""Workload recipes and a counter-based generator (splitmix64 + Box-Muller).

Every value is a pure function of (seed, config id, b, h, tensor id, element
index), so any head of any workload can be regenerated on its own, on the CPU or
on a CUDA device, without generating the rest.  The generator is written with
torch int64 tensor arithmetic (two's-complement wrap-around gives the same bits
as uint64 arithmetic), so one definition serves both devices.

Recipe (readings of the workload descriptions where they are silent):
  * splitmix64: state_i = key + (i+1)*0x9E3779B97F4A7C15, output = mix(state_i)
    with the published splitmix64 finaliser (Steele, Lea, Flood 2014).
  * U(0,1): ((z >> 11) + 0.5) / 2^53, never 0 or 1.
  * N(0,1) for element i: Box-Muller on the uniforms of draws 2i and 2i+1,
    sqrt(-2 ln u1) * cos(2 pi u2), evaluated in float64.
  * "N(mu, s)" reads s as a standard deviation.
  * gates: alpha_t = sigmoid(N(mu_a, sd_a)), beta_t = sigmoid(N(mu_b, sd_b)),
    float64 then rounded to float32.
  * bf16 inputs: float32 value rounded to nearest-even bf16.
  * codebook entries: N(0,1) / sqrt(d_qk/2) (the stated /4 at d_h=16 and /8 at
    d_h=64; the same rule is applied where a workload does not state it).
  * long-context keys: for t < T_full/2, k'_t = P[u_t] + 0.1*N(0,1), P being
    4096 N(0,1) pattern vectors per (b,h) and u_t uniform on [0,4096);
    computed in float64, rounded to float32 then bf16.  Other keys i.i.d.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB


def _s64(c: int) -> int:
    """uint64 constant -> the int64 with the same bits."""
    return c - (1 << 64) if c >= (1 << 63) else c


_GAMMA_S = _s64(_GAMMA)
_MIX1_S = _s64(_MIX1)
_MIX2_S = _s64(_MIX2)

# tensor ids of the streams
TID_Q, TID_K, TID_V, TID_ALPHA, TID_BETA, TID_C1, TID_C2, TID_M0 = 1, 2, 3, 4, 5, 6, 7, 8
TID_PATTERN, TID_PICK, TID_NOISE = 9, 10, 11
TID_GDN_Q, TID_GDN_K, TID_GDN_S0 = 12, 13, 14
TID_DECAY = 15


def _mix_int(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * _MIX1) & _M64
    z = ((z ^ (z >> 27)) * _MIX2) & _M64
    return z ^ (z >> 31)


def stream_key(seed: int, cfg_id: int, b: int, h: int, tid: int) -> int:
    """64-bit key of one (seed, config, b, h, tensor) stream."""
    z = _mix_int(seed + _GAMMA)
    for field in (cfg_id, b, h, tid):
        z = _mix_int(z + (field + 1) * _GAMMA)
    return z


def _shr(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bits."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def splitmix64_stream(key: torch.Tensor, idx: torch.Tensor) -> torch.Tensor:
    """Output number idx (int64 tensor) of the splitmix64 stream with the given key(s)."""
    z = key + (idx + 1) * _GAMMA_S
    z = (z ^ _shr(z, 30)) * _MIX1_S
    z = (z ^ _shr(z, 27)) * _MIX2_S
    return z ^ _shr(z, 31)


def uniform01(z: torch.Tensor) -> torch.Tensor:
    return (_shr(z, 11).to(torch.float64) + 0.5) * (2.0 ** -53)


def std_normal(key: torch.Tensor, idx: torch.Tensor) -> torch.Tensor:
    """float64 N(0,1) number idx of the stream (Box-Muller, cosine branch)."""
    u1 = uniform01(splitmix64_stream(key, 2 * idx))
    u2 = uniform01(splitmix64_stream(key, 2 * idx + 1))
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


@dataclasses.dataclass(frozen=True)
class SDMConfig:
    """One workload.  Field names follow the pages' notation."""
    name: str
    cfg_id: int
    B: int
    H: int
    T: int
    d_qk: int
    d_v: int
    n_sub: int          # sqrt(N): rows per sub-key codebook
    k: int              # per-half top-k
    W: int              # write slots per step
    R: int              # read slots per step
    in_dtype: str       # 'f32' or 'bf16' for q', k', v, C1, C2
    alpha_mu: float
    alpha_sd: float
    beta_mu: float
    beta_sd: float
    m0_sd: float = 0.0          # 0 -> M_0 = 0
    key_patterns: int = 0       # >0: recurring key patterns
    pattern_noise: float = 0.1
    pattern_until: int = 0      # keys t < pattern_until are patterned

    @property
    def N(self) -> int:
        return self.n_sub * self.n_sub

    @property
    def d_h(self) -> int:
        return self.d_qk // 2

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def cb_sd(self) -> float:
        return 1.0 / math.sqrt(self.d_h)

    def with_(self, **kw) -> "SDMConfig":
        return dataclasses.replace(self, **kw)

    def dims(self) -> Dict[str, int]:
        return dict(B=self.B, H=self.H, T=self.T, d_qk=self.d_qk, d_v=self.d_v,
                    n_sub=self.n_sub, k=self.k, W=self.W, R=self.R,
                    in_dtype=0 if self.in_dtype == 'f32' else 1)


CONFIGS = [
    SDMConfig("tiny-fp32", 0, B=1, H=1, T=256, d_qk=32, d_v=16, n_sub=32, k=8, W=8, R=8,
              in_dtype='f32', alpha_mu=3.0, alpha_sd=1.0, beta_mu=0.0, beta_sd=1.0),
    SDMConfig("small", 1, B=4, H=8, T=2048, d_qk=128, d_v=64, n_sub=256, k=32, W=64, R=64,
              in_dtype='bf16', alpha_mu=3.0, alpha_sd=1.0, beta_mu=0.0, beta_sd=1.0),
    SDMConfig("pages-scale-N2^20", 2, B=2, H=4, T=8192, d_qk=128, d_v=64, n_sub=1024, k=64,
              W=64, R=64, in_dtype='bf16', alpha_mu=4.0, alpha_sd=1.0, beta_mu=0.0, beta_sd=1.0),
    SDMConfig("long-context-N2^20", 3, B=1, H=8, T=65536, d_qk=256, d_v=128, n_sub=1024, k=128,
              W=128, R=128, in_dtype='bf16', alpha_mu=4.0, alpha_sd=1.0, beta_mu=0.0, beta_sd=1.0,
              key_patterns=4096, pattern_noise=0.1, pattern_until=32768),
    SDMConfig("high-batch-N2^18", 4, B=64, H=16, T=4096, d_qk=128, d_v=64, n_sub=512, k=64,
              W=64, R=64, in_dtype='bf16', alpha_mu=3.0, alpha_sd=1.0, beta_mu=-1.0, beta_sd=1.0,
              m0_sd=0.02),
]


def config(i: int) -> SDMConfig:
    return CONFIGS[i]


def _round_input(x64: torch.Tensor, in_dtype: str) -> torch.Tensor:
    """float64 draw -> float32 holding the input dtype's value."""
    x32 = x64.to(torch.float32)
    if in_dtype == 'bf16':
        x32 = x32.to(torch.bfloat16).to(torch.float32)
    return x32


def _keys(cfg: SDMConfig, seed: int, tid: int, bs, hs, device) -> torch.Tensor:
    ks = [[_s64(stream_key(seed, cfg.cfg_id, b, h, tid)) for h in hs] for b in bs]
    return torch.tensor(ks, dtype=torch.int64, device=device)


def _normals(cfg, seed, tid, bs, hs, shape_tail, device) -> torch.Tensor:
    """[len(bs), len(hs), *shape_tail] float64 normals; element index = row-major
    offset within one head's [*shape_tail] block."""
    key = _keys(cfg, seed, tid, bs, hs, device).view(len(bs), len(hs), *([1] * len(shape_tail)))
    numel = 1
    for s in shape_tail:
        numel *= s
    idx = torch.arange(numel, dtype=torch.int64, device=device).view(1, 1, *shape_tail)
    return std_normal(key, idx)


def gen_head_inputs(cfg: SDMConfig, b: int, h: int, seed: int = 0,
                    device: str = 'cpu', t_end: Optional[int] = None,
                    with_m0: bool = True) -> Dict[str, torch.Tensor]:
    """All inputs of one (b,h) head as float32 tensors (bf16-exact where the
    workload is bf16).  Shapes: q,k [T,d_qk], v [T,d_v], alpha,beta [T],
    C1,C2 [n,d_h], M0 [N,d_v].  t_end truncates the time axis (a prefix)."""
    return _gen(cfg, [b], [h], seed, device, t_end, with_m0, squeeze=True)


def gen_inputs(cfg: SDMConfig, seed: int = 0, device: str = 'cpu',
               t_end: Optional[int] = None, with_m0: bool = True,
               b0: int = 0, h0: int = 0, h1: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All inputs, full layout: q,k [B,H,T,d_qk], v [B,H,T,d_v], alpha,beta [B,H,T],
    C1,C2 [H,n,d_h], M0 [B,H,N,d_v] (float32 values).  b0 offsets the batch
    index (rows [b0, b0+B) of a larger batch); h0, h1 select the heads [h0, h1)
    of the cfg.H heads (default all), so that a rectangle of the head grid is
    the same slice of the full inputs."""
    h1 = cfg.H if h1 is None else h1
    return _gen(cfg, list(range(b0, b0 + cfg.B)), list(range(h0, h1)), seed, device, t_end,
                with_m0, squeeze=False)


def _gen(cfg, bs, hs, seed, device, t_end, with_m0, squeeze):
    T = cfg.T if t_end is None else t_end
    out = {}
    # q' ~ N(0,1)
    out['q'] = _round_input(_normals(cfg, seed, TID_Q, bs, hs, (T, cfg.d_qk), device), cfg.in_dtype)
    # k': i.i.d. N(0,1), or recurring patterns for t < pattern_until
    k64 = _normals(cfg, seed, TID_K, bs, hs, (T, cfg.d_qk), device)
    if cfg.key_patterns > 0 and cfg.pattern_until > 0:
        tp = min(T, cfg.pattern_until)
        P = _normals(cfg, seed, TID_PATTERN, bs, hs, (cfg.key_patterns, cfg.d_qk), device)
        pk = _keys(cfg, seed, TID_PICK, bs, hs, device).view(len(bs), len(hs), 1)
        tt = torch.arange(tp, dtype=torch.int64, device=device).view(1, 1, tp)
        bits = max(1, int(math.log2(cfg.key_patterns)))
        assert (1 << bits) == cfg.key_patterns, "pattern count must be a power of two"
        pick = _shr(splitmix64_stream(pk, tt), 64 - bits)          # uniform on [0, P)
        noise = _normals(cfg, seed, TID_NOISE, bs, hs, (tp, cfg.d_qk), device)
        patt = torch.gather(P, 2, pick.unsqueeze(-1).expand(len(bs), len(hs), tp, cfg.d_qk))
        k64[:, :, :tp, :] = patt + cfg.pattern_noise * noise
    out['k'] = _round_input(k64, cfg.in_dtype)
    out['v'] = _round_input(_normals(cfg, seed, TID_V, bs, hs, (T, cfg.d_v), device), cfg.in_dtype)
    za = _normals(cfg, seed, TID_ALPHA, bs, hs, (T,), device)
    zb = _normals(cfg, seed, TID_BETA, bs, hs, (T,), device)
    out['alpha'] = torch.sigmoid(cfg.alpha_mu + cfg.alpha_sd * za).to(torch.float32)
    out['beta'] = torch.sigmoid(cfg.beta_mu + cfg.beta_sd * zb).to(torch.float32)
    # codebooks: per head, shared over the batch (b field fixed at 0)
    c1 = _normals(cfg, seed, TID_C1, [0], hs, (cfg.n_sub, cfg.d_h), device)[0] * cfg.cb_sd
    c2 = _normals(cfg, seed, TID_C2, [0], hs, (cfg.n_sub, cfg.d_h), device)[0] * cfg.cb_sd
    out['C1'] = _round_input(c1, cfg.in_dtype)
    out['C2'] = _round_input(c2, cfg.in_dtype)
    if with_m0:
        if cfg.m0_sd > 0:
            out['M0'] = (cfg.m0_sd * _normals(cfg, seed, TID_M0, bs, hs, (cfg.N, cfg.d_v),
                                              device)).to(torch.float32)
        else:
            out['M0'] = torch.zeros(len(bs), len(hs), cfg.N, cfg.d_v, dtype=torch.float32,
                                    device=device)
    if squeeze:
        for name in list(out):
            if name in ('C1', 'C2'):
                out[name] = out[name][0]
            else:
                out[name] = out[name][0, 0]
    return out


def gen_gdn_inputs(cfg: SDMConfig, d_k: Optional[int] = None, seed: int = 0, device: str = 'cpu',
                   s0_sd: float = 0.0, t_end: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Inputs of the dense Gated DeltaNet baseline matched to an SDM workload:
    same B, H, T, d_v, gates and value stream; q', k' of width d_k (default W,
    the matched query dimension) drawn N(0, I) and L2-normalised in float64
    before rounding to the input dtype (GDN normalises its keys and queries);
    S_0 = 0 unless s0_sd > 0.  Shapes: q, k [B,H,T,d_k], v [B,H,T,d_v],
    alpha, beta [B,H,T], S0 [B,H,d_v,d_k] (float32 values)."""
    d_k = cfg.W if d_k is None else d_k
    T = cfg.T if t_end is None else t_end
    bs, hs = list(range(cfg.B)), list(range(cfg.H))
    out = {}
    for name, tid in (('q', TID_GDN_Q), ('k', TID_GDN_K)):
        x = _normals(cfg, seed, tid, bs, hs, (T, d_k), device)
        out[name] = _round_input(x / torch.linalg.vector_norm(x, dim=-1, keepdim=True),
                                 cfg.in_dtype)
    out['v'] = _round_input(_normals(cfg, seed, TID_V, bs, hs, (T, cfg.d_v), device), cfg.in_dtype)
    za = _normals(cfg, seed, TID_ALPHA, bs, hs, (T,), device)
    zb = _normals(cfg, seed, TID_BETA, bs, hs, (T,), device)
    out['alpha'] = torch.sigmoid(cfg.alpha_mu + cfg.alpha_sd * za).to(torch.float32)
    out['beta'] = torch.sigmoid(cfg.beta_mu + cfg.beta_sd * zb).to(torch.float32)
    if s0_sd > 0:
        out['S0'] = (s0_sd * _normals(cfg, seed, TID_GDN_S0, bs, hs, (cfg.d_v, d_k),
                                      device)).to(torch.float32)
    else:
        out['S0'] = torch.zeros(cfg.B, cfg.H, cfg.d_v, d_k, dtype=torch.float32, device=device)
    return out


def gen_decay_rate(cfg: SDMConfig, seed: int = 0, device: str = 'cpu', b0: int = 0,
                   t_end: Optional[int] = None) -> torch.Tensor:
    """Decay rates of the selective-decay write rule, [B,H,T] float32:
    a_t = -softplus(N(0, 1)) (negative, as a Mamba-2 style input-dependent rate;
    the Raven page gives no distribution), computed in float64."""
    T = cfg.T if t_end is None else t_end
    z = _normals(cfg, seed, TID_DECAY, list(range(b0, b0 + cfg.B)), list(range(cfg.H)), (T,),
                 device)
    return (-torch.nn.functional.softplus(z)).to(torch.float32)
