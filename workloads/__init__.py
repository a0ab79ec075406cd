"""Seeded synthetic workloads for the gated sliding-window attention core.

This module only draws random numbers and names shapes.  It holds none of the
method's arithmetic, so both the CUDA path (tests, bench) and the fp64 oracle
can take their inputs from it without sharing any computation.

Recipe (the pages measure whole-model training on their own corpus, which is
not used here; these synthetic tensors stand in for it):
  * ``torch.Generator(device).manual_seed(seed)``; ``randn`` in fp32, then
    rounded to bf16.  Draw order: q, k, v, g, wq, wk, dO.
  * Norm weights ``1 + 0.1 * N(0, 1)`` in fp32.
  * Gate logits ~ N(0, std^2) with std 2 for the forward-only shapes and 1
    for the training shape.
  * Decode: both rings ~N(0,1) (bf16), new q, k, v, g ~N(0,1), positions
    uniform in [128, 262144), drawn after the rings.
  * Global layers: the prefill draws q, k, v as above (its g is unused); the
    decode draws [N, Hkv, cap, D] caches ~N(0,1), then q, k, v, the norm
    weights and positions uniform in [1, cap).
"""
from dataclasses import dataclass, field

import torch

HEAD_DIM = 128
WINDOW = 128
ROT_DIM = 42
EPS = 1e-6


@dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    base: float
    g_std: float
    seed: int
    backward: bool = False
    D: int = HEAD_DIM
    W: int = WINDOW
    R: int = ROT_DIM
    eps: float = EPS

    @property
    def tokens(self) -> int:
        return self.B * self.T


@dataclass(frozen=True)
class Decode:
    name: str
    N: int
    layers: int
    Hq: int
    Hkv: int
    base: float
    seed: int
    pos_lo: int = 128
    pos_hi: int = 262144
    D: int = HEAD_DIM
    W: int = WINDOW
    R: int = ROT_DIM
    eps: float = EPS


# The five shapes the library is checked and measured on.
TINY = Prefill("tiny gated-SWA forward 1x256, 4q/1kv", B=1, T=256, Hq=4, Hkv=1,
               base=1e4, g_std=1.0, seed=0)
LAYER = Prefill("layer-shape prefill forward 4x4096, 32q/8kv", B=4, T=4096, Hq=32, Hkv=8,
                base=1e4, g_std=2.0, seed=1)
TRAIN = Prefill("training-shape forward+backward 1x16384, 32q/8kv", B=1, T=16384, Hq=32,
                Hkv=8, base=1e4, g_std=1.0, seed=2, backward=True)
LONG = Prefill("long-context prefill forward 1x262144, 32q/8kv, base 1e7", B=1, T=262144,
               Hq=32, Hkv=8, base=1e7, g_std=2.0, seed=3)
DECODE = Decode("decode step, 256 sequences x 27 gated-SWA layers, 128-slot rings", N=256,
                layers=27, Hq=32, Hkv=8, base=1e7, seed=4)

PREFILL_CONFIGS = {"tiny": TINY, "layer": LAYER, "train": TRAIN, "long": LONG}

# The global causal layers (5 of the 32): no window and no gate, so only q, k
# and v are drawn (g and the gate's std unused).
GLOBAL_PREFILL = Prefill("global-layer causal prefill 1x16384, 32q/8kv", B=1, T=16384, Hq=32,
                         Hkv=8, base=1e4, g_std=1.0, seed=6)


@dataclass(frozen=True)
class GlobalDecode:
    name: str
    N: int
    layers: int
    Hq: int
    Hkv: int
    cap: int
    base: float
    seed: int
    D: int = HEAD_DIM
    R: int = ROT_DIM
    eps: float = EPS


GLOBAL_DECODE = GlobalDecode("global-layer decode step, 64 sequences x 5 layers, 32K-slot caches",
                             N=64, layers=5, Hq=32, Hkv=8, cap=32768, base=1e7, seed=7)


def global_decode_layer_inputs(cfg: GlobalDecode, layer: int, device="cpu"):
    """One global layer's decode inputs: [N, Hkv, cap, D] K and V caches ~N(0,1),
    new q, k, v ~N(0,1), norm weights, positions uniform in [1, cap)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed * 1000 + layer)
    N, Hq, Hkv, D = cfg.N, cfg.Hq, cfg.Hkv, cfg.D
    out = {
        "k_cache": _randn((N, Hkv, cfg.cap, D), gen, device),
        "v_cache": _randn((N, Hkv, cfg.cap, D), gen, device),
        "q": _randn((N, Hq, D), gen, device),
        "k": _randn((N, Hkv, D), gen, device),
        "v": _randn((N, Hkv, D), gen, device),
    }
    out["wq"] = 1.0 + 0.1 * torch.randn((D,), generator=gen, device=device)
    out["wk"] = 1.0 + 0.1 * torch.randn((D,), generator=gen, device=device)
    out["pos"] = torch.randint(1, cfg.cap, (N,), generator=gen, device=device, dtype=torch.int64)
    return out


def _randn(shape, gen, device, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def prefill_inputs(cfg: Prefill, device="cpu", seed=None, with_grad_out=None):
    """q, g [B,T,Hq,D] and k, v [B,T,Hkv,D] bf16; wq, wk [D] fp32; optional dO."""
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed if seed is None else seed)
    B, T, Hq, Hkv, D = cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D
    out = {
        "q": _randn((B, T, Hq, D), gen, device),
        "k": _randn((B, T, Hkv, D), gen, device),
        "v": _randn((B, T, Hkv, D), gen, device),
        "g": _randn((B, T, Hq, D), gen, device, cfg.g_std),
    }
    out["wq"] = 1.0 + 0.1 * torch.randn((D,), generator=gen, device=device)
    out["wk"] = 1.0 + 0.1 * torch.randn((D,), generator=gen, device=device)
    if cfg.backward if with_grad_out is None else with_grad_out:
        out["dO"] = _randn((B, T, Hq, D), gen, device)
    return out


def fp8_prefill_inputs(cfg: Prefill, device="cpu", seed=None):
    """The inputs of :func:`prefill_inputs` with q, k and v quantised to FP8
    E4M3, one factor per tensor (its largest magnitude over 448, the E4M3
    maximum): q8, k8, v8 (torch.float8_e4m3fn) with qkv_scale [3] fp32, so that
    q ~ q8 * qkv_scale[0] etc.  g, wq, wk as there.  The quantisation only
    builds inputs: the library and the oracle both read the same bytes."""
    x = prefill_inputs(cfg, device=device, seed=seed, with_grad_out=False)
    out = {"g": x["g"], "wq": x["wq"], "wk": x["wk"]}
    scales = []
    for name in ("q", "k", "v"):
        t = x[name].float()
        s = float(t.abs().max()) / 448.0
        out[name + "8"] = (t / s).to(torch.float8_e4m3fn)
        scales.append(s)
    out["qkv_scale"] = torch.tensor(scales, dtype=torch.float32, device=device)
    return out


def decode_layer_inputs(cfg: Decode, layer: int, device="cpu", N=None):
    """Inputs of one layer's decode step: rings, new token tensors, positions."""
    N = cfg.N if N is None else N
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed * 1000 + layer)
    Hq, Hkv, W, D = cfg.Hq, cfg.Hkv, cfg.W, cfg.D
    out = {
        "k_cache": _randn((N, Hkv, W, D), gen, device),
        "v_cache": _randn((N, Hkv, W, D), gen, device),
        "q": _randn((N, Hq, D), gen, device),
        "k": _randn((N, Hkv, D), gen, device),
        "v": _randn((N, Hkv, D), gen, device),
        "g": _randn((N, Hq, D), gen, device),
    }
    out["wq"] = 1.0 + 0.1 * torch.randn((D,), generator=gen, device=device)
    out["wk"] = 1.0 + 0.1 * torch.randn((D,), generator=gen, device=device)
    out["pos"] = torch.randint(cfg.pos_lo, cfg.pos_hi, (N,), generator=gen, device=device,
                               dtype=torch.int64)
    return out


def custom_prefill(B, T, Hq, Hkv, base=1e4, g_std=1.0, seed=0, backward=False, W=WINDOW,
                   R=ROT_DIM, D=HEAD_DIM):
    """A prefill shape outside the five named ones (edge cases in the tests)."""
    return Prefill(f"custom {B}x{T} {Hq}q/{Hkv}kv W={W}", B=B, T=T, Hq=Hq, Hkv=Hkv,
                   base=base, g_std=g_std, seed=seed, backward=backward, W=W, R=R, D=D)
