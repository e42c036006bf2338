"""Seeded synthetic workloads for the CARVE recurrence (no method arithmetic here).

Both the CUDA path (through its tests and the benchmark) and the fp64 oracle consume
the arrays produced here, so this module holds only random-number generation, the
input recipe and dtype rounding.  It never evaluates a gate, a state or an output.

Generator: splitmix64 (Steele, Lea & Flood 2014, "Fast splittable pseudorandom number
generators") as a counter-based stream -- element n of stream s is mix(s + (n+1)*phi) --
turned into N(0,1) by the Box-Muller transform (Box & Muller 1958).  Every tensor has its
own stream id, so a tensor's values do not depend on which other tensors were drawn.

Recipe (the pages' 1.3B setting: 16 heads, d = 128; CARVE gist.science summary, section 4):
  q, k ~ N(0,1), then L2-normalised over the key axis per (token, head)
  v ~ N(0,1);  g_logit ~ N(-3, 0.5^2)  (so g = exp(-softplus(g_logit)) ~ 0.953)
  bx ~ N(0,1); w_logit ~ N(0,1);  A, B (the low-rank factors of U_b) ~ N(0, 0.02^2)
  S0 = 0 for sequence workloads; decode state S ~ N(0, 0.05^2).
  Decay parameters, when a workload uses them: A_dec (the log-amplitude, per head)
  = log U(0.5, 2), tau (the bias, per head and key channel) ~ N(0, 0.5^2).
  Packed variable-length batches: lengths ~ U{lo..hi} drawn until they fill the token budget.
bf16 workloads round q, k, v to bfloat16 (round-to-nearest-even) after normalisation;
the oracle then reads exactly those rounded values.
"""
from __future__ import annotations

import dataclasses
import numpy as np

_PHI = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_BLOCK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_key(seed: int, stream: int) -> np.uint64:
    z = np.array([(seed * 0x100000001B3 + stream * 0x9E3779B1 + 1) & 0xFFFFFFFFFFFFFFFF],
                 dtype=np.uint64)
    return _mix(z)[0]


def uniform01(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    """n doubles in (0, 1]: element j is splitmix64 output (offset + j) of the stream."""
    key = _stream_key(seed, stream)
    out = np.empty(n, dtype=np.float64)
    with np.errstate(over="ignore"):
        for lo in range(0, n, _BLOCK):
            hi = min(n, lo + _BLOCK)
            ctr = np.arange(offset + lo + 1, offset + hi + 1, dtype=np.uint64)
            z = _mix(key + ctr * _PHI)
            out[lo:hi] = ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)
    return out


def normal(seed: int, stream: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """Box-Muller normals, float64.  Pair j uses uniforms 2j and 2j+1 of the stream."""
    n = int(np.prod(shape))
    m = (n + 1) // 2
    out = np.empty(2 * m, dtype=np.float64)
    for lo in range(0, m, _BLOCK):
        hi = min(m, lo + _BLOCK)
        u = uniform01(seed, stream, 2 * (hi - lo), offset=2 * lo)
        r = np.sqrt(-2.0 * np.log(u[0::2]))
        th = (2.0 * np.pi) * u[1::2]
        out[2 * lo:2 * hi:2] = r * np.cos(th)
        out[2 * lo + 1:2 * hi:2] = r * np.sin(th)
    return (mean + std * out[:n]).reshape(shape)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-representable."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    assert np.all((u & np.uint32(0xFFFF)) == 0), "values are not bf16-representable"
    return (u >> np.uint32(16)).astype(np.uint16)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes of one synthetic workload."""
    name: str
    B: int
    H: int
    T: int
    K: int
    V: int
    R: int
    L: int
    io: str            # "fp32" or "bf16": dtype of q, k, v, o and their gradients
    seed: int
    mc_mode: int = 0   # 0: chunk-boundary state readout, 1: previous-chunk mean output
    steps: int = 0     # decode workloads: number of consecutive single-token steps


BASE_SEED = 20261202

# The five workloads of the 1.3B-layer study (16 heads, d = 128) plus the tiny fp32 check.
TINY_FP32 = Workload("tiny_fp32_B1_H2_T256_d64_L64", 1, 2, 256, 64, 64, 16, 64, "fp32", BASE_SEED + 0)
FWD_1P3B = Workload("fwd_1.3B_layer_B4_H16_T2048_d128_L64", 4, 16, 2048, 128, 128, 32, 64, "bf16", BASE_SEED + 1)
TRAIN_1P3B = Workload("train_1.3B_layer_B8_H16_T4096_d128_L64", 8, 16, 4096, 128, 128, 32, 64, "bf16", BASE_SEED + 2)


def long_context(L: int, mc_mode: int) -> Workload:
    return Workload(f"long_ctx_B1_H16_T65536_d128_L{L}_mc{mc_mode}", 1, 16, 65536, 128, 128, 32, L,
                    "bf16", BASE_SEED + 3, mc_mode)


DECODE = Workload("decode_B256_H16_d128_1000steps", 256, 16, 1, 128, 128, 32, 1, "bf16",
                  BASE_SEED + 4, steps=1000)

# stream ids (fixed forever: changing one changes every stored expectation)
_S_Q, _S_K, _S_V, _S_GL, _S_BX, _S_WL, _S_A, _S_B, _S_DO, _S_S0, _S_DS, _S_ADEC, _S_TAU, _S_LEN = range(1, 15)


def _l2norm_last(x: np.ndarray) -> np.ndarray:
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True))


def make_inputs(w: Workload, seed: int | None = None, T: int | None = None) -> dict:
    """Inputs of a sequence workload, as float32 arrays (bf16-rounded where the workload
    stores bf16).  Layouts: q, k, g_logit, bx [B,T,H,K]; v [B,T,H,V]; w_logit [B,T,H];
    A [H,K,R]; B [H,R,V]."""
    s = w.seed if seed is None else seed
    T = w.T if T is None else T
    B, H, K, V, R = w.B, w.H, w.K, w.V, w.R
    q = _l2norm_last(normal(s, _S_Q, (B, T, H, K))).astype(np.float32)
    k = _l2norm_last(normal(s, _S_K, (B, T, H, K))).astype(np.float32)
    v = normal(s, _S_V, (B, T, H, V)).astype(np.float32)
    if w.io == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    return dict(
        q=q, k=k, v=v,
        g_logit=normal(s, _S_GL, (B, T, H, K), -3.0, 0.5).astype(np.float32),
        bx=normal(s, _S_BX, (B, T, H, K)).astype(np.float32),
        w_logit=normal(s, _S_WL, (B, T, H)).astype(np.float32),
        A=normal(s, _S_A, (H, K, R), 0.0, 0.02).astype(np.float32),
        B=normal(s, _S_B, (H, R, V), 0.0, 0.02).astype(np.float32),
    )


def make_decay(w: Workload, seed: int | None = None) -> dict:
    """The decay's per-head parameters: A_dec [H] = log U(0.5, 2) and tau [H,K] ~ N(0, 0.5^2),
    float32."""
    s = w.seed if seed is None else seed
    amp = 0.5 + 1.5 * uniform01(s, _S_ADEC, w.H)
    return dict(A_dec=np.log(amp).astype(np.float32),
                tau=normal(s, _S_TAU, (w.H, w.K), 0.0, 0.5).astype(np.float32))


def make_lengths(total: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Sequence lengths for a packed batch of exactly `total` tokens: each drawn uniformly from
    [lo, hi] (integers) until the sum reaches `total`; the last one is cut to fit."""
    u = uniform01(seed, _S_LEN, max(1, 4 * total // max(lo, 1) + 4))
    lens, acc = [], 0
    for x in u:
        n = lo + min(int(x * (hi - lo + 1)), hi - lo)
        n = min(n, total - acc)
        lens.append(n)
        acc += n
        if acc == total:
            break
    assert acc == total
    return np.asarray(lens, dtype=np.int32)


def make_grad_out(w: Workload, seed: int | None = None, T: int | None = None) -> np.ndarray:
    """Upstream gradient dO ~ N(0,1) of shape [B,T,H,V] (bf16-rounded for bf16 workloads)."""
    s = w.seed if seed is None else seed
    T = w.T if T is None else T
    d = normal(s, _S_DO, (w.B, T, w.H, w.V)).astype(np.float32)
    return round_bf16(d) if w.io == "bf16" else d


def make_state(w: Workload, std: float, seed: int | None = None, stream: int = _S_S0) -> np.ndarray:
    """A float32 state [B,H,V,K] ~ N(0, std^2)."""
    s = w.seed if seed is None else seed
    return normal(s, stream, (w.B, w.H, w.V, w.K), 0.0, std).astype(np.float32)


def make_decode_pool(w: Workload, pool: int = 64, seed: int | None = None) -> dict:
    """Decode inputs: a pool of `pool` distinct seeded token sets; step j of a run reads
    pool entry j % pool.  q, k, g_logit, bx [P,B,H,K]; v [P,B,H,V]; w_logit [P,B,H];
    A [H,K,R]; B [H,R,V].  Drawn as a length-`pool` sequence workload, token axis first."""
    d = make_inputs(dataclasses.replace(w, T=pool), seed=seed)
    out = {}
    for key in ("q", "k", "v", "g_logit", "bx"):
        out[key] = np.ascontiguousarray(d[key].transpose(1, 0, 2, 3))
    out["w_logit"] = np.ascontiguousarray(d["w_logit"].transpose(1, 0, 2))
    out["A"], out["B"] = d["A"], d["B"]
    return out
