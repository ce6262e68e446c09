"""Seeded synthetic inputs for the MoE layer forward.

This module is shared by the tests, the benchmark and the oracle harness.  It
holds no step of the layer's arithmetic: it only draws numbers.

Generator (counter-based, device-agnostic):
  * every tensor has a fixed id; element ``i`` of tensor ``tid`` under seed ``s``
    is a pure function of ``(s, tid, i)``, so any slice (one expert's weights,
    a sample of token rows) can be regenerated alone, on the CPU or the GPU,
    with identical bits;
  * the hash is Chris Wellons' public "lowbias32" 32-bit integer mixer, with
    its two 32x32-bit multiplies split into 16-bit halves so that every
    intermediate fits a non-negative int64 (torch integer ops are then exact
    and identical on CPU and CUDA);
  * a normal draw is an Irwin-Hall(4) sum of four 16-bit uniforms, centred
    and scaled to unit variance: ``z = (2*S - 4*65535) * sqrt(3)/131072``.
    The centred integer is exact in fp32, and the scale is ONE fp32 multiply,
    so CPU and GPU agree bit for bit; bf16 tensors are then rounded to nearest
    even by torch.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = [
    "MoeShape", "CONFIGS", "TENSOR_IDS", "config", "normal", "normal_slice",
    "zipf_logit_offset", "make_inputs", "expert_slice", "token_ids",
]

_M32 = 0xFFFFFFFF
_CHUNK = 1 << 20       # elements generated per pass on the CPU (bounds int64 temporaries)
_CHUNK_GPU = 1 << 26   # ... and on a GPU (fewer, larger launches)


def _chunk(device) -> int:
    return _CHUNK_GPU if torch.device(device).type == "cuda" else _CHUNK


@dataclass(frozen=True)
class MoeShape:
    """One MoE layer workload: sizes plus the input recipe."""
    name: str
    T: int
    d: int
    E: int
    G: int
    K: int
    M: int
    d_ff: int
    n_shared: int
    d_ff_shared: int
    x_sigma: float          # x ~ N(0, x_sigma)
    e_sigma: float          # router weights ~ N(0, e_sigma), fp32
    bias_sigma: float       # balance bias ~ N(0, bias_sigma), fp32
    zipf_s: float = 0.0     # > 0: per-expert logit offset log(Zipf(s) popularity)
    seed: int = 0
    note: str = field(default="", compare=False)

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k in
                ("T", "d", "E", "G", "K", "M", "d_ff", "n_shared", "d_ff_shared")}

    def replace(self, **kw) -> "MoeShape":
        d = dict(self.__dict__)
        d.update(kw)
        return MoeShape(**d)


def _inv_sqrt(n: int) -> float:
    return 1.0 / math.sqrt(n)


# The five workloads.  Weights are N(0,1)/sqrt(fan_in) everywhere (fan_in = d
# for gate/up, d_ff for down).
CONFIGS = {
    "tiny": MoeShape("tiny", T=64, d=128, E=16, G=4, K=4, M=2, d_ff=64,
                     n_shared=1, d_ff_shared=64,
                     x_sigma=_inv_sqrt(128), e_sigma=_inv_sqrt(128), bias_sigma=0.1),
    "mid": MoeShape("mid", T=4096, d=2048, E=64, G=8, K=6, M=3, d_ff=1408,
                    n_shared=2, d_ff_shared=1408,
                    x_sigma=_inv_sqrt(2048), e_sigma=0.05, bias_sigma=0.05),
    "v3": MoeShape("v3", T=8192, d=7168, E=256, G=8, K=8, M=4, d_ff=2048,
                   n_shared=1, d_ff_shared=2048,
                   x_sigma=1.0, e_sigma=_inv_sqrt(7168), bias_sigma=0.0),
    "decode": MoeShape("decode", T=128, d=7168, E=256, G=8, K=8, M=4, d_ff=2048,
                       n_shared=1, d_ff_shared=2048,
                       x_sigma=1.0, e_sigma=_inv_sqrt(7168), bias_sigma=0.0),
    "skew": MoeShape("skew", T=32768, d=7168, E=256, G=8, K=8, M=4, d_ff=2048,
                     n_shared=1, d_ff_shared=2048,
                     x_sigma=1.0, e_sigma=_inv_sqrt(7168), bias_sigma=0.5, zipf_s=1.2),
}

# Reduced workloads for profiler captures: the V3 layer's dimensions and rows
# per expert (T*K/E = 256) with fewer experts, so that a capture holds a few
# GB on the device; DRAM traffic per token is that of the full layer.
# v3_ep: the V3 row width and top-8 over 4096 tokens and 32 narrow experts, for
# captures of the expert-parallel exchange kernels (2 ranks of 2048 tokens: one
# combine launch reads 235 MB, above L2) within a few GB.
# v3_ffn64: the V3 batch, router and routing exactly (T=8192, d=7168, E=256,
# K=8) with 64-wide expert FFNs, for captures of the route, dispatch and
# combine kernels at full size within a few GB (their work does not depend on
# d_ff).
PROFILE_CONFIGS = {
    "v3_e32": CONFIGS["v3"].replace(name="v3_e32", T=1024, E=32),
    "v3_ffn64": CONFIGS["v3"].replace(name="v3_ffn64", d_ff=64, d_ff_shared=64),
    "v3_ep": CONFIGS["v3"].replace(name="v3_ep", T=4096, E=32, d_ff=512),
}

# Fixed tensor ids: salt of the counter-based generator.
TENSOR_IDS = {
    "x": 1, "router_w": 2, "bias": 3, "w_gate": 4, "w_up": 5, "w_down": 6,
    "ws_gate": 7, "ws_up": 8, "ws_down": 9, "zipf_perm": 10, "y_perm": 11,
    "y_shared": 12, "scores": 13, "token_ids": 14,
}

# Vocabulary of DeepSeek-V3's tokenizer: the id range of synthetic token ids.
VOCAB = 129280


def config(name: str) -> MoeShape:
    return CONFIGS[name] if name in CONFIGS else PROFILE_CONFIGS[name]


# ---------------------------------------------------------------- hashing
def _mul32(a, c: int):
    """(a * c) mod 2**32 for a in [0, 2**32) with every partial product < 2**49."""
    lo, hi = c & 0xFFFF, c >> 16
    return (a * lo + (((a * hi) & 0xFFFF) << 16)) & _M32


def _mix32(x):
    """lowbias32 (C. Wellons): x^=x>>16; x*=0x7feb352d; x^=x>>15; x*=0x846ca68b; x^=x>>16."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _keys(seed: int, tid: int):
    k1 = _mix32(((seed & _M32) * 0x9E3779B1 + tid * 0x85EBCA77 + 0x165667B1) & _M32)
    k2 = _mix32(k1 ^ 0x27D4EB2F)
    k3 = _mix32(k2 ^ 0x61C88647)
    return k1, k2, k3


def _words(seed: int, tid: int, idx: torch.Tensor):
    """Two 32-bit words for each int64 element index."""
    k1, k2, k3 = _keys(seed, tid)
    lo = idx & _M32
    hi = idx >> 32
    a = _mix32(lo ^ k1)
    a = _mix32(a ^ hi ^ k2)
    b = _mix32(a ^ k3)
    return a, b


def _scale32(sigma: float) -> float:
    # The single fp32 multiplier: sigma * sqrt(3) / (2 * 65536).
    return float(torch.tensor(sigma * math.sqrt(3.0) / 131072.0, dtype=torch.float32))


def normal_slice(seed: int, tid: int, start: int, count: int, sigma: float,
                 dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """Elements [start, start+count) of the flat N(0, sigma) tensor (seed, tid)."""
    out = torch.empty(count, dtype=dtype, device=device)
    if sigma == 0.0 or count == 0:
        out.zero_()
        return out
    c = torch.tensor(_scale32(sigma), dtype=torch.float32, device=device)
    step = _chunk(device)
    for s in range(0, count, step):
        n = min(step, count - s)
        idx = torch.arange(start + s, start + s + n, dtype=torch.int64, device=device)
        a, b = _words(seed, tid, idx)
        acc = (a & 0xFFFF) + (a >> 16) + (b & 0xFFFF) + (b >> 16)
        z = (2 * acc - 4 * 65535).to(torch.float32) * c
        out[s:s + n] = z.to(dtype)
    return out


def normal(seed: int, tid: int, shape, sigma: float, dtype=torch.bfloat16,
           device="cpu") -> torch.Tensor:
    n = 1
    for s in shape:
        n *= int(s)
    return normal_slice(seed, tid, 0, n, sigma, dtype, device).view(*shape)


def zipf_logit_offset(E: int, s: float, seed: int) -> torch.Tensor:
    """log of Zipf(s) popularity, p_r = r^-s / sum_q q^-s over ranks r = 1..E.

    Ranks are assigned to experts by a seeded permutation (the order of the
    hash of each rank), so the popular experts are scattered over the groups.
    """
    r = torch.arange(1, E + 1, dtype=torch.float64)
    p = r.pow(-s)
    p = p / p.sum()
    h = torch.tensor([_mix32(_mix32(q ^ _keys(seed, TENSOR_IDS["zipf_perm"])[0]))
                      for q in range(E)], dtype=torch.int64)
    expert_of_rank = torch.argsort(h, stable=True)
    off = torch.empty(E, dtype=torch.float64)
    off[expert_of_rank] = torch.log(p)
    return off.to(torch.float32)


def expert_slice(shape: MoeShape, name: str, e: int, device="cpu") -> torch.Tensor:
    """One expert's weight matrix of a routed weight tensor, regenerated alone."""
    if name in ("w_gate", "w_up"):
        rows, cols, fan = shape.d_ff, shape.d, shape.d
    elif name == "w_down":
        rows, cols, fan = shape.d, shape.d_ff, shape.d_ff
    else:
        raise ValueError(name)
    n = rows * cols
    return normal_slice(shape.seed, TENSOR_IDS[name], e * n, n, _inv_sqrt(fan),
                        torch.bfloat16, device).view(rows, cols)


def make_inputs(shape: MoeShape, device="cpu", weights: bool = True) -> dict:
    """All layer inputs of a workload as torch tensors on ``device``.

    x [T,d] bf16; router_w [E,d] fp32; bias [E] fp32; logit_offset [E] fp32
    or None; w_gate/w_up [E,d_ff,d], w_down [E,d,d_ff] bf16; ws_gate/ws_up
    [n_shared,d_ff_shared,d], ws_down [n_shared,d,d_ff_shared] bf16.
    """
    sd, T, d, E = shape.seed, shape.T, shape.d, shape.E
    out = {
        "x": normal(sd, TENSOR_IDS["x"], (T, d), shape.x_sigma, torch.bfloat16, device),
        "router_w": normal(sd, TENSOR_IDS["router_w"], (E, d), shape.e_sigma,
                           torch.float32, device),
        "bias": normal(sd, TENSOR_IDS["bias"], (E,), shape.bias_sigma, torch.float32, device),
        "logit_offset": (zipf_logit_offset(E, shape.zipf_s, sd).to(device)
                         if shape.zipf_s > 0 else None),
    }
    if weights:
        ff, ns, ffs = shape.d_ff, shape.n_shared, shape.d_ff_shared
        out["w_gate"] = normal(sd, TENSOR_IDS["w_gate"], (E, ff, d), _inv_sqrt(d), torch.bfloat16, device)
        out["w_up"] = normal(sd, TENSOR_IDS["w_up"], (E, ff, d), _inv_sqrt(d), torch.bfloat16, device)
        out["w_down"] = normal(sd, TENSOR_IDS["w_down"], (E, d, ff), _inv_sqrt(ff), torch.bfloat16, device)
        if ns > 0:
            out["ws_gate"] = normal(sd, TENSOR_IDS["ws_gate"], (ns, ffs, d), _inv_sqrt(d), torch.bfloat16, device)
            out["ws_up"] = normal(sd, TENSOR_IDS["ws_up"], (ns, ffs, d), _inv_sqrt(d), torch.bfloat16, device)
            out["ws_down"] = normal(sd, TENSOR_IDS["ws_down"], (ns, d, ffs), _inv_sqrt(ffs), torch.bfloat16, device)
        else:
            out["ws_gate"] = out["ws_up"] = out["ws_down"] = None
    return out


def uniform01(seed: int, tid: int, shape, device="cpu") -> torch.Tensor:
    """fp32 uniform on (0, 1): (24-bit integer + 0.5) * 2^-24, exact in fp32."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=torch.float32, device=device)
    step = _chunk(device)
    for s in range(0, n, step):
        m = min(step, n - s)
        idx = torch.arange(s, s + m, dtype=torch.int64, device=device)
        a, _ = _words(seed, tid, idx)
        out[s:s + m] = ((a >> 8).to(torch.float32) + 0.5) * (2.0 ** -24)
    return out.view(*shape)


def random_routing(seed: int, T: int, E: int, K: int, zipf_s: float = 0.0,
                   device="cpu") -> torch.Tensor:
    """[T, K] int32: K distinct experts per token drawn without replacement.

    Weighted sampling by the Efraimidis-Spirakis keys u^(1/p_e) with Zipf(s)
    weights p_e (uniform when s == 0); an input for testing the dispatch
    alone on skewed or balanced expert loads.
    """
    u = uniform01(seed, TENSOR_IDS["scores"] + 100, (T, E), device).double()
    if zipf_s > 0:
        p = torch.arange(1, E + 1, dtype=torch.float64, device=device).pow(-zipf_s)
        keys = torch.log(u) / p
    else:
        keys = torch.log(u)
    return torch.topk(keys, K, dim=1).indices.to(torch.int32)


def token_ids(seed: int, T: int, vocab: int = VOCAB, device="cpu") -> torch.Tensor:
    """[T] int64 token ids with a Zipf-like (log-uniform) frequency over
    [0, vocab): id = floor(vocab^u) - 1 for u uniform on (0, 1), so small ids
    (frequent words) repeat often and large ones rarely, as in text."""
    u = uniform01(seed, TENSOR_IDS["token_ids"], (T,), device).double()
    ids = torch.floor(torch.pow(float(vocab), u)).to(torch.int64) - 1
    return ids.clamp_(0, vocab - 1)
