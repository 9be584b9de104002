"""Counter-based random inputs and the reference workload recipes.

Generator (defined here and implemented a second time, bit for bit, in
``synth/csrc/synth_gen.cu`` so that multi-GB tensors can be drawn on the GPU):

* Uniform bits: the c-th output of SplitMix64 (Steele, Lea & Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014) started
  from a per-(seed, stream) key: ``h(c) = mix64(key + (c + 1) * GAMMA)`` with
  the published golden-gamma increment and the published mix64 finaliser.
* Normals: the Box–Muller transform on pairs of outputs.  Pair p uses
  ``u1 = ((h(2p) >> 11) + 1) * 2^-53`` in (0, 1] and
  ``u2 = (h(2p+1) >> 11) * 2^-53`` in [0, 1); element 2p is ``r cos(2 pi u2)``
  and element 2p+1 is ``r sin(2 pi u2)`` with ``r = sqrt(-2 ln u1)``.
  ``ln``, ``cos`` and ``sin`` are evaluated with the series below using only
  IEEE +, -, *, / and sqrt (each correctly rounded, none fused), so numpy and
  the CUDA copy (compiled with ``-fmad=false``) produce identical doubles:
  - ``ln x``: x = m * 2^e with m in [sqrt(1/2), sqrt(2)); with
    t = (m - 1)/(m + 1), ln m = 2 t * sum_k t^(2k)/(2k+1) (k = 0..11, Horner),
    ln x = e * ln2 + ln m.
  - ``cos``/``sin`` of 2 pi u2: w = 4 u2, quadrant q = floor(w), a = (w - q) * pi/2
    in [0, pi/2), Taylor series of cos a and sin a to degree 22/23 (Horner in
    a^2), rotated by q quarter turns.
* Storage rounding: float64 -> bfloat16 round-to-nearest-even done directly on
  the float64 bit pattern (one rounding, no float32 step); float64 -> float32
  is numpy's correctly rounded cast.

Every workload below draws its tensors from this generator with a stated seed
and stream, so the oracle can regenerate any (batch, head) slice on the host
without holding the whole tensor.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX_C1 = 0xBF58476D1CE4E5B9
MIX_C2 = 0x94D049BB133111EB

# stream ids (one independent sequence per tensor role)
STREAM_Q = 1
STREAM_K = 2
STREAM_V = 3
STREAM_SINK = 4
STREAM_BIAS = 5
STREAM_KEY_FACTOR = 6
STREAM_KEY_INDEX = 7
STREAM_PAD = 8
STREAM_DOUT = 9

LN2 = 0.6931471805599453          # double nearest ln 2
HALF_PI = 1.5707963267948966      # double nearest pi/2
SQRT_HALF = 0.7071067811865476    # double nearest sqrt(1/2)

N_LOG_TERMS = 12                  # k = 0..11
N_TRIG_TERMS = 12                 # cos: a^0..a^22, sin: a^1..a^23


def _series_coefficients():
    """Coefficient tables shared with the CUDA copy (passed to it verbatim)."""
    log_c = [1.0 / float(2 * k + 1) for k in range(N_LOG_TERMS)]
    cos_c, sin_c = [], []
    fact = 1.0  # running k! in double, built by sequential products
    facts = [1.0]
    for k in range(1, 2 * N_TRIG_TERMS + 1):
        fact = fact * float(k)
        facts.append(fact)
    for k in range(N_TRIG_TERMS):
        sign = -1.0 if (k % 2) else 1.0
        cos_c.append(sign / facts[2 * k])
        sin_c.append(sign / facts[2 * k + 1])
    return (np.array(log_c, dtype=np.float64), np.array(cos_c, dtype=np.float64),
            np.array(sin_c, dtype=np.float64))


LOG_COEF, COS_COEF, SIN_COEF = _series_coefficients()


def _mix64_py(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX_C1) & MASK64
    z = ((z ^ (z >> 27)) * MIX_C2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    """64-bit key of the sequence for (seed, stream)."""
    return _mix64_py(_mix64_py(seed * GAMMA + 0x5851F42D4C957F2D) ^ (stream * 0xD1B54A32D192ED03))


def uniform_bits(key: int, start: int, count: int) -> np.ndarray:
    """h(c) for c in [start, start+count) as uint64."""
    c = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (c + np.uint64(1)) * np.uint64(GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX_C1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX_C2)
        z = z ^ (z >> np.uint64(31))
    return z


def uniform_f64(key: int, start: int, count: int) -> np.ndarray:
    """Uniform doubles in [0, 1): (h >> 11) * 2^-53."""
    return (uniform_bits(key, start, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _log_series(x: np.ndarray) -> np.ndarray:
    m, e = np.frexp(x)                       # x = m * 2^e, m in [0.5, 1)
    small = m < SQRT_HALF
    m = np.where(small, m * 2.0, m)
    e = np.where(small, e - 1, e).astype(np.float64)
    t = (m - 1.0) / (m + 1.0)
    t2 = t * t
    p = np.full_like(t, LOG_COEF[-1])
    for ck in LOG_COEF[-2::-1]:
        p = p * t2 + ck
    return e * LN2 + (2.0 * t) * p


def _sincos_turn(u: np.ndarray):
    """(cos, sin) of 2*pi*u for u in [0, 1)."""
    w = u * 4.0
    q = np.floor(w)
    a = (w - q) * HALF_PI
    a2 = a * a
    c = np.full_like(a, COS_COEF[-1])
    for ck in COS_COEF[-2::-1]:
        c = c * a2 + ck
    s = np.full_like(a, SIN_COEF[-1])
    for sk in SIN_COEF[-2::-1]:
        s = s * a2 + sk
    s = s * a
    qi = q.astype(np.int64) & 3
    cos_t = np.select([qi == 0, qi == 1, qi == 2], [c, -s, -c], s)
    sin_t = np.select([qi == 0, qi == 1, qi == 2], [s, c, -s], -c)
    return cos_t, sin_t


def normal_f64(key: int, start: int, count: int) -> np.ndarray:
    """Standard normal doubles for elements [start, start+count) of a stream."""
    if count <= 0:
        return np.zeros(0, dtype=np.float64)
    p0 = start // 2
    p1 = (start + count + 1) // 2
    npair = p1 - p0
    h = uniform_bits(key, 2 * p0, 2 * npair)
    u1 = ((h[0::2] >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * (2.0 ** -53)
    u2 = (h[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    r = np.sqrt(-2.0 * _log_series(u1))
    ct, st = _sincos_turn(u2)
    out = np.empty(2 * npair, dtype=np.float64)
    out[0::2] = r * ct
    out[1::2] = r * st
    off = start - 2 * p0
    return out[off:off + count]


# ----------------------------------------------------------------------------
# storage rounding
# ----------------------------------------------------------------------------

def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 bits, round to nearest even, one rounding.

    Values below the bfloat16 normal range flush to signed zero; the
    workloads never draw such values (a N(0,1) draw below 1e-38 in magnitude
    has probability ~1e-38).  Overflow raises.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    b = x.view(np.uint64)
    sign = (b >> np.uint64(63)).astype(np.uint16)
    mag = b & np.uint64(0x7FFFFFFFFFFFFFFF)
    lsb = (mag >> np.uint64(45)) & np.uint64(1)
    r = mag + np.uint64((1 << 44) - 1) + lsb
    e64 = ((r >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64)
    frac = ((r >> np.uint64(45)) & np.uint64(0x7F)).astype(np.uint16)
    e32 = e64 - 1023 + 127
    if np.any(e32 > 254):
        raise OverflowError("value outside the bfloat16 range")
    tiny = e32 <= 0
    e16 = np.where(tiny, 0, e32).astype(np.uint16)
    frac = np.where(tiny, 0, frac).astype(np.uint16)
    return (sign << np.uint16(15)) | (e16 << np.uint16(7)) | frac


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float64."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def sinusoidal_table(num_pos: int, dim: int, base: float = 10000.0) -> np.ndarray:
    """Fixed sin/cos position table (even dims sin, odd dims cos), float64.

    Input-side preprocessing for the RBF workload: a precomputed,
    non-rotating sinusoid added to query and key rows.
    """
    pos = np.arange(num_pos, dtype=np.float64)[:, None]
    i = np.arange(dim // 2, dtype=np.float64)[None, :]
    freq = base ** (-2.0 * i / dim)
    tab = np.zeros((num_pos, dim), dtype=np.float64)
    tab[:, 0::2] = np.sin(pos * freq)
    tab[:, 1::2] = np.cos(pos * freq)
    return tab


# ----------------------------------------------------------------------------
# workload recipes
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Recipe:
    name: str
    N: int
    Hq: int
    H: int
    L: int
    S: int
    E: int
    Ev: int
    dtype: str            # "bf16" or "f32"
    mode: str             # "dot" or "rbf"
    scale: float
    mask_kind: str        # "none", "causal", "window", "streaming"
    window: int = 0
    keep: int = 0         # streaming mask: initial tokens every later query sees
    n_sel: int = 0        # > 0: decode over a selected key list of this length per (n, KV head)
    keep_mask: str = "none"   # "random10": boolean keep mask, False where the random10 bias is -inf
    pad_left: float = 0.0     # per-batch left padding: kv_start[n] = floor(u * pad_left * S)
    pad_right: float = 0.0    # per-batch right padding: kv_end[n] = S - floor(u * pad_right * S)
    backward: bool = False    # the measured step is the backward pass (dout: N(0,1) draws of its own stream)
    sink: str = "none"    # "none", "fixed", "normal"
    sink_values: tuple = ()
    bias: str = "none"    # "none", "random10" or "mixed" (see bias_matrix)
    registers: int = 0    # zero K/V rows prepended (RBF workload)
    key_lognormal: bool = False
    sinusoid_pe: bool = False
    seed: int = 0
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.Hq // self.H


RECIPES = {
    r.name: r for r in [
        Recipe("tiny_rbf_sink_causal_f32", N=1, Hq=2, H=2, L=128, S=128, E=64, Ev=64,
               dtype="f32", mode="rbf", scale=1.0 / 8.0, mask_kind="causal",
               sink="fixed", sink_values=(0.0, 1.0), seed=0,
               note="tiny oracle case: RBF, causal, per-head sink logits [0, 1]"),
        Recipe("dot_causal_2k_bf16", N=4, Hq=16, H=16, L=2048, S=2048, E=128, Ev=128,
               dtype="bf16", mode="dot", scale=1.0 / math.sqrt(128.0), mask_kind="causal",
               seed=2, note="dot-product causal prefill"),
        Recipe("dot_bias10_2k_f32", N=4, Hq=16, H=16, L=2048, S=2048, E=128, Ev=128,
               dtype="f32", mode="dot", scale=1.0 / math.sqrt(128.0), mask_kind="none",
               bias="random10", seed=2,
               note="fp32, non-causal, additive 0/-inf mask on a random 10% (diagonal kept)"),
        Recipe("rbf_registers_4k_bf16", N=2, Hq=12, H=12, L=4100, S=4100, E=64, Ev=64,
               dtype="bf16", mode="rbf", scale=1.0 / 8.0, mask_kind="causal",
               registers=4, key_lognormal=True, sinusoid_pe=True, seed=3,
               note="RBF prefill with 4 zero register rows, lognormal key norms, sinusoidal PE"),
        Recipe("sink_gqa_window_16k_bf16", N=1, Hq=64, H=8, L=16384, S=16384, E=64, Ev=64,
               dtype="bf16", mode="dot", scale=1.0 / 8.0, mask_kind="window", window=4096,
               sink="normal", seed=4,
               note="sink-logit GQA sliding-window prefill"),
        Recipe("decode_sink_gqa_128k_bf16", N=32, Hq=32, H=8, L=1, S=131072, E=128, Ev=128,
               dtype="bf16", mode="dot", scale=1.0 / math.sqrt(128.0), mask_kind="none",
               sink="normal", seed=5,
               note="long-context decode, split over the key axis + combine"),
    ]
}


def shapes(r: Recipe) -> dict:
    return {
        "q": (r.N, r.Hq, r.L, r.E),
        "k": (r.N, r.H, r.S, r.E),
        "v": (r.N, r.H, r.S, r.Ev),
    }


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_round_bits(x)
    if dtype == "f32":
        return x.astype(np.float32)
    raise ValueError(dtype)


def _stored_to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_bits_to_f64(x)
    return np.asarray(x, dtype=np.float64)


def _slice_values_f64(r: Recipe, tensor: str, n: int, h: int) -> np.ndarray:
    """Unrounded float64 values of one (n, h) slice of q, k or v: (rows, dim)."""
    shp = shapes(r)[tensor]
    _, heads, rows, dim = shp
    stream = {"q": STREAM_Q, "k": STREAM_K, "v": STREAM_V}[tensor]
    key = stream_key(r.seed, stream)
    start = ((n * heads + h) * rows) * dim
    x = normal_f64(key, start, rows * dim).reshape(rows, dim)
    if r.key_lognormal and tensor == "k":
        fkey = stream_key(r.seed, STREAM_KEY_FACTOR)
        g = normal_f64(fkey, (n * heads + h) * rows, rows)
        x = x * np.exp(g)[:, None]
    if r.registers and tensor in ("k", "v"):
        x[: r.registers] = 0.0
    if r.sinusoid_pe and tensor in ("q", "k"):
        R = r.registers
        pe = sinusoidal_table(rows - R, dim)
        x[R:] = x[R:] + pe
    return x


def tensor_slice_f64(r: Recipe, tensor: str, n: int, h: int) -> np.ndarray:
    """Stored (rounded) values of one (n, h) slice, widened exactly to float64."""
    return _stored_to_f64(_store(_slice_values_f64(r, tensor, n, h), r.dtype), r.dtype)


def sink_logits(r: Recipe):
    if r.sink == "none":
        return None
    if r.sink == "fixed":
        return np.array(r.sink_values, dtype=np.float32)
    return normal_f64(stream_key(r.seed, STREAM_SINK), 0, r.Hq).astype(np.float32)


def bias_matrix(r: Recipe):
    """Additive [L, S] float32 bias or None.

    random10: each entry is -inf with probability 0.1 (uniform draw u < 0.1), 0
    otherwise; the diagonal j == i is always 0.
    mixed: the random10 pattern, and on the 128 x 128 blocks with
    (i // 128 + j // 128) odd every entry that is not -inf takes the finite value
    4 u' - 2 in [-2, 2), u' the (L*S + i*S + j)-th draw of the same stream.  Half
    the blocks thus hold general additive values and half only 0 / -inf.
    """
    if r.bias == "none":
        return None
    key = stream_key(r.seed, STREAM_BIAS)
    u = uniform_f64(key, 0, r.L * r.S).reshape(r.L, r.S)
    b = np.where(u < 0.1, -np.inf, 0.0)
    idx = np.arange(min(r.L, r.S))
    b[idx, idx] = 0.0
    if r.bias == "mixed":
        u2 = uniform_f64(key, r.L * r.S, r.L * r.S).reshape(r.L, r.S)
        blk = ((np.arange(r.L)[:, None] // 128) + (np.arange(r.S)[None, :] // 128)) % 2 == 1
        b = np.where(blk & np.isfinite(b), 4.0 * u2 - 2.0, b)
    elif r.bias != "random10":
        raise ValueError(f"unknown bias kind {r.bias!r}")
    return b.astype(np.float32)


def keep_matrix(r: Recipe) -> np.ndarray | None:
    """(L, S) bool keep mask or None.  random10: the complement of the random10
    bias pattern (the same draws): False with probability 0.1, True on the
    diagonal j == i."""
    if r.keep_mask == "none":
        return None
    u = uniform_f64(stream_key(r.seed, STREAM_BIAS), 0, r.L * r.S).reshape(r.L, r.S)
    keep = u >= 0.1
    idx = np.arange(min(r.L, r.S))
    keep[idx, idx] = True
    return keep


def pack_mask_bits(keep: np.ndarray) -> np.ndarray:
    """(L, S) bool -> (L, ceil(S/32)) uint32: bit j % 32 of word j // 32 is keep[:, j]
    (bits past S are 0)."""
    keep = np.asarray(keep, dtype=bool)
    L, S = keep.shape
    W = (S + 31) // 32
    padded = np.zeros((L, W * 32), dtype=bool)
    padded[:, :S] = keep
    return np.packbits(padded.reshape(L, W, 4, 8), axis=-1, bitorder="little").reshape(L, W * 4).view("<u4").copy()


def kv_ranges(r: Recipe):
    """(kv_start, kv_end) int32 arrays of length N, or (None, None) without padding."""
    if r.pad_left <= 0 and r.pad_right <= 0:
        return None, None
    u = uniform_f64(stream_key(r.seed, STREAM_PAD), 0, 2 * r.N).reshape(2, r.N)
    start = np.floor(u[0] * r.pad_left * r.S).astype(np.int32)
    end = (r.S - np.floor(u[1] * r.pad_right * r.S)).astype(np.int32)
    return start, end


def key_index_set(r: Recipe) -> np.ndarray | None:
    """(N, H, n_sel) int32 key lists, or None.  For each (n, KV head) one uniform
    draw per cached key; the n_sel keys with the largest draws, in decreasing
    draw order.  That is a uniformly random n_sel-subset in random order, the
    shape of a top-k selection's output (positions scattered over the cache,
    not sorted).  n_sel > S repeats the list cyclically."""
    if r.n_sel <= 0:
        return None
    key = stream_key(r.seed, STREAM_KEY_INDEX)
    out = np.empty((r.N, r.H, r.n_sel), dtype=np.int32)
    for n in range(r.N):
        for h in range(r.H):
            u = uniform_f64(key, (n * r.H + h) * r.S, r.S)
            order = np.argsort(-u, kind="stable")
            out[n, h] = np.resize(order, r.n_sel)
    return out


def generate(r: Recipe) -> dict:
    """Whole workload on the host (numpy).  bf16 tensors are uint16 bit arrays."""
    out = {}
    for t, shp in shapes(r).items():
        N, heads, rows, dim = shp
        arr = np.empty(shp, dtype=np.uint16 if r.dtype == "bf16" else np.float32)
        for n in range(N):
            for h in range(heads):
                arr[n, h] = _store(_slice_values_f64(r, t, n, h), r.dtype)
        out[t] = arr
    out["sink"] = sink_logits(r)
    out["bias"] = bias_matrix(r)
    out["key_idx"] = key_index_set(r)
    out["keep"] = keep_matrix(r)
    out["kv_start"], out["kv_end"] = kv_ranges(r)
    return out


def as_f64(r: Recipe, arr: np.ndarray) -> np.ndarray:
    """Widen a stored q/k/v array of recipe r exactly to float64."""
    return _stored_to_f64(arr, r.dtype)


def gpu_drawable(r: Recipe) -> bool:
    """True when q, k and v are plain iid N(0,1) draws (no per-key factors,
    registers or position table), i.e. the CUDA copy of the generator can draw
    them directly on the device."""
    return not (r.key_lognormal or r.registers or r.sinusoid_pe)
