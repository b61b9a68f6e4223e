"""Counter-based seeded generator for the synthetic LSA workloads (host side).

Every synthetic value is a pure function of (seed, tensor id, element counter), so
any slice of any tensor can be regenerated on its own: the CPU oracle rebuilds only
the rows it needs, and the device filler in ``csrc/synth_fill.cu`` writes the same
bytes straight into GPU memory for caches too large to build on the host.  The two
implementations agree bit for bit because every step below is either integer
arithmetic or a single correctly rounded float32 operation.

This module draws numbers and encodes them into the storage formats of the caches
(BF16, FP8 e4m3 with a per-token scale).  It contains none of the arithmetic of the
sparse-attention method itself.

Recipe (stated once here, repeated in the design notes):

* hash:      mix(z) is the splitmix64 finaliser; word(key, c) = mix(key + c * G),
             G = 0x9E3779B97F4A7C15, all arithmetic mod 2**64.
* key:       key(seed, tid) = mix(mix(seed + G) + tid * G).
* normal:    element i uses words 3i, 3i+1, 3i+2; their twelve 16-bit fields are
             summed (Irwin-Hall, n = 12): x = (2 * S - 786420) * 2**-17, which is
             exact in float32, has mean 0 and variance 1 (up to the 2**-32 grid).
* uniform:   top 24 bits of word(key, i) times 2**-24, in [0, 1).
* BF16:      float32 rounded to nearest even on the upper 16 bits.
* FP8 e4m3:  per token, amax = max |x|; scale = amax / 448; y = x * (448 / amax)
             (two float32 roundings); code = y rounded to nearest even on the OCP
             e4m3 grid, saturating at 448.  An all-zero row gets scale 1.
"""
from __future__ import annotations

import numpy as np

U64 = np.uint64
GOLD = U64(0x9E3779B97F4A7C15)
_M1 = U64(0xBF58476D1CE4E5B9)
_M2 = U64(0x94D049BB133111EB)

# Tensor ids.  Per-layer tensors add the layer number.
TID_IDX_KEYS = 1       # indexer key cache  [B, L, d_I]
TID_IDX_Q = 2          # indexer queries    [T, H_I, d_I]
TID_IDX_W = 3          # indexer head weights [T, H_I]
TID_DRAFT_IDX_KEYS = 4
TID_DRAFT_IDX_Q = 5
TID_DRAFT_IDX_W = 6
TID_KV = 16            # + layer: latent KV cache [B, L, D]
TID_Q = 48             # + layer: attention queries [T, H, D]
TID_V = 80             # + layer: separate V cache (non-MLA layout)
TID_PLANT = 112        # ranking hash used to choose planted positions / blocks
TID_LENGTHS = 113      # sequence lengths

ROW_SHIFT_L = 22       # element counter of cache entry (b, l, d): ((b << 22 | l) << 10) | d
ROW_SHIFT_D = 10
MAX_CACHE_LEN = 1 << ROW_SHIFT_L
MAX_CACHE_DIM = 1 << ROW_SHIFT_D


def mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser on uint64 arrays (wrapping arithmetic)."""
    z = np.asarray(z, dtype=U64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> U64(30))) * _M1
        z = (z ^ (z >> U64(27))) * _M2
    return z ^ (z >> U64(31))


def tensor_key(seed: int, tid: int) -> int:
    with np.errstate(over="ignore"):
        k0 = mix(U64(seed & 0xFFFFFFFFFFFFFFFF) + GOLD)
        return int(mix(k0 + U64(tid) * GOLD))


def words(key: int, ctr: np.ndarray) -> np.ndarray:
    ctr = np.asarray(ctr, dtype=U64)
    with np.errstate(over="ignore"):
        return mix(U64(key) + ctr * GOLD)


def normal_f32(key: int, ctr: np.ndarray) -> np.ndarray:
    """Irwin-Hall(12) standard normal draws, exact float32, for element counters ``ctr``."""
    ctr = np.asarray(ctr, dtype=U64)
    s = np.zeros(ctr.shape, dtype=U64)
    with np.errstate(over="ignore"):
        base = ctr * U64(3)
        for j in range(3):
            h = words(key, base + U64(j))
            s += (h & U64(0xFFFF)) + ((h >> U64(16)) & U64(0xFFFF)) \
                + ((h >> U64(32)) & U64(0xFFFF)) + (h >> U64(48))
    centred = 2 * s.astype(np.int64) - 786420
    return centred.astype(np.float32) * np.float32(2.0 ** -17)


def uniform_f32(key: int, ctr: np.ndarray) -> np.ndarray:
    h = words(key, ctr)
    return (h >> U64(40)).astype(np.float32) * np.float32(2.0 ** -24)


def cache_ctr(b: int, rows: np.ndarray, dim: int) -> np.ndarray:
    """Element counters of cache rows ``rows`` of sequence ``b``: shape [len(rows), dim]."""
    rows = np.asarray(rows, dtype=np.int64)
    assert dim <= MAX_CACHE_DIM and (rows.size == 0 or rows.max() < MAX_CACHE_LEN)
    rowctr = ((np.int64(b) << ROW_SHIFT_L) | rows).astype(U64) << U64(ROW_SHIFT_D)
    return rowctr[:, None] | np.arange(dim, dtype=U64)[None, :]


# ---------------------------------------------------------------- storage encodings

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to BF16 (nearest even); returns uint16 bit patterns. NaN stays NaN."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + U64(0x7FFF) + ((b >> U64(16)) & U64(1))) >> U64(16)
    isnan = np.isnan(x)
    out = rounded.astype(np.uint16)
    out[isnan] = ((b[isnan] >> U64(16)) | U64(0x40)).astype(np.uint16)
    return out


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _e4m3_grid() -> np.ndarray:
    """The 127 non-negative finite e4m3 magnitudes, index = code (0x00..0x7E)."""
    vals = np.empty(127, dtype=np.float64)
    for code in range(127):
        e, m = code >> 3, code & 7
        vals[code] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3_POS = _e4m3_grid()


def f32_to_e4m3(y: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest e4m3 code (ties to even code), saturating at 448."""
    y = np.asarray(y, dtype=np.float32)
    a = np.abs(y.astype(np.float64))
    a = np.minimum(a, 448.0)
    hi = np.searchsorted(_E4M3_POS, a, side="left")          # first grid value >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((hi & 1) == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    sign = np.signbit(y).astype(np.uint8) << np.uint8(7)   # a negative value that rounds to 0 keeps its sign
    return code | sign


def quantize_rows_e4m3(x: np.ndarray):
    """Per-row (per-token) FP8 e4m3 quantisation: returns (codes uint8 [..., D], scale float32 [...])."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    scale = np.where(amax > 0, safe / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    inv = np.where(amax > 0, np.float32(448.0) / safe, np.float32(1.0)).astype(np.float32)
    y = (x * inv[..., None]).astype(np.float32)
    return f32_to_e4m3(y), scale


# ---------------------------------------------------------------- planted signal

def query_direction(q_heads: np.ndarray) -> np.ndarray:
    """Planting direction for one query: sqrt(d) * u / |u| with u the sum of its indexer heads."""
    u = np.asarray(q_heads, dtype=np.float64).sum(axis=0)
    return (np.sqrt(u.size) * u / np.linalg.norm(u)).astype(np.float32)


def planted_rows(key_rows: np.ndarray, direction: np.ndarray) -> np.ndarray:
    """k = direction + 0.3 * noise, each step one float32 rounding (noise = the row's own draws)."""
    return (np.float32(0.3) * key_rows.astype(np.float32)).astype(np.float32) + direction[None, :]


def choose_without_replacement(seed: int, tid: int, stream: int, n_total: int, n_pick: int) -> np.ndarray:
    """n_pick distinct integers of [0, n_total): the ones with the smallest hash ranks, sorted."""
    key = tensor_key(seed, tid)
    ctr = (np.uint64(stream) << np.uint64(32)) | np.arange(n_total, dtype=U64)
    rank = words(key, ctr)
    pick = np.argsort(rank, kind="stable")[:n_pick]
    return np.sort(pick).astype(np.int64)
