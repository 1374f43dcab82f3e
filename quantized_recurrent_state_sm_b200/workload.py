"""Seeded synthetic workloads for the packed-state gated Delta-rule decode step.

This module only draws numbers: per-step inputs (q, k, v, beta), the per-head or
per-key-row retention gates, the row-impact weights, the outlier channel gains
and the fixed bit-allocation / pivot tables that a calibration pass would
export.  It performs none of the decode step's arithmetic (no state update, no
readout, no scale fitting, no quantisation, no packing), so both the CPU oracle
and the CUDA path can take their inputs from here.

Random numbers come from a counter-based generator: SplitMix64 (Steele, Lea and
Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014) applied to
a key derived from (seed, stream, request, head, step) and an element index.
Any (request, head, step) slice can therefore be produced on its own, which is
what lets the oracle run on a subsample of a large batch with exactly the
inputs the GPU sees for those requests.

Workload recipe (the pages evaluate on real models and text; none of that is
available, so these synthetic inputs stand in for it):

* k, q ~ N(0, 1) per element, then L2-normalised per (request, head, step);
  v ~ N(0, 1); beta = sigmoid(N(0, 1)).
* Gates: alpha = 0.5 ** (1 / h) with half-life h = 2 ** U(0, 12), i.e.
  log-uniform in [1, 4096] steps, per head (Gated-DeltaNet) or per
  (head, key row) (KDA).  Gates are fixed over steps and shared by requests,
  as the pages fix calibration offline per unit.
* Row-impact weights rho ~ LogNormal(0, sigma) per (head, key row).
* Bit tables: a greedy lifetime-weighted allocation under the average budget
  (FP16 pivots count 16 bits towards it), pivots = the longest-half-life units.
* Outlier stress: a few key channels and value channels per head get a fixed
  gain (applied to k before normalisation, to v directly).
"""
from __future__ import annotations

import heapq
import math
from dataclasses import dataclass, field

import numpy as np

U64 = np.uint64
_GOLDEN = U64(0x9E3779B97F4A7C15)
_M1 = U64(0xBF58476D1CE4E5B9)
_M2 = U64(0x94D049BB133111EB)

PIVOT_BITS = 16  # a pivot unit stores every value as an IEEE binary16 number

# stream identifiers for the counter-based generator
S_Q, S_K, S_V, S_BETA = 1, 2, 3, 4
S_GATE, S_RHO, S_OUT_K, S_OUT_V = 5, 6, 7, 8
S_Q_GAIN = 9

GDN, KDA = 0, 1


def splitmix64(x):
    """SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    x = np.asarray(x, dtype=U64)
    with np.errstate(over="ignore"):
        z = x + _GOLDEN
        z = (z ^ (z >> U64(30))) * _M1
        z = (z ^ (z >> U64(27))) * _M2
        return z ^ (z >> U64(31))


def derive_key(seed: int, *coords) -> np.ndarray:
    """Chain SplitMix64 over the coordinates; each coord may be an int array.

    Negative coordinates (warm-up steps) are mapped into uint64 by adding 2**32.
    """
    key = np.asarray(U64(seed & 0xFFFFFFFFFFFFFFFF))
    for c in coords:
        c = np.asarray(c, dtype=np.int64)
        c = (c + (1 << 32)).astype(U64)
        key = splitmix64(key ^ c)
    return key


def uniform01(key, idx) -> np.ndarray:
    """Uniform double in [0, 1) for each (key, idx) pair (broadcasting)."""
    key = np.asarray(key, dtype=U64)
    idx = np.asarray(idx, dtype=U64)
    bits = splitmix64(key ^ (idx * U64(0x100000001B3)))
    return (bits >> U64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(key, idx) -> np.ndarray:
    """Standard normal via Box-Muller from two counter-indexed uniforms."""
    idx = np.asarray(idx, dtype=np.int64)
    u1 = uniform01(key, 2 * idx)
    u2 = uniform01(key, 2 * idx + 1)
    return np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * math.pi * u2)


@dataclass(frozen=True)
class Config:
    index: int
    name: str
    variant: int            # GDN (scalar gate per head) or KDA (gate per key row)
    batch: int
    heads: int
    steps: int
    bits_choices: tuple
    avg_bits: float
    pivot_frac: float
    rho_sigma: float
    dk: int = 128
    dv: int = 128
    warmup: int = 32
    outlier_frac: float = 0.0
    outlier_gain: float = 1.0
    ls_iters: int = 1
    q_gain_sigma: float = 0.0  # per (head, key row) query gains ~ LogNormal(0, sigma) (0: none)

    @property
    def input_seed(self) -> int:
        return 0x5EED0000 + self.index

    @property
    def table_seed(self) -> int:
        return 0x7AB10000 + self.index

    @property
    def items(self) -> int:
        return self.batch * self.heads

    @property
    def kind(self) -> str:
        return "kda" if self.variant == KDA else "gdn"


CONFIGS = {
    0: Config(0, "gdn-int6-b4-h16", GDN, 4, 16, 64, (6,), 6.0, 0.0, 1.0),
    1: Config(1, "gdn-mixed468-b64-h32", GDN, 64, 32, 256, (4, 6, 8), 6.0, 0.02, 1.0),
    2: Config(2, "kda-mixed3to8-b128-h32", KDA, 128, 32, 256, (3, 4, 5, 6, 7, 8), 6.0, 0.01, 1.5),
    3: Config(3, "gdn-4bit-b512-h48", GDN, 512, 48, 1024, (3, 4, 6), 4.0, 0.01, 1.0),
    4: Config(4, "kda-outlier-b256-h32", KDA, 256, 32, 2048, (3, 4, 5, 6, 7, 8), 6.0, 0.01, 1.5,
              outlier_frac=0.02, outlier_gain=30.0),
}


def with_overrides(cfg: Config, **kw) -> Config:
    d = dict(cfg.__dict__)
    d.update(kw)
    return Config(**d)


# ----------------------------------------------------------------------------
# fixed tables (shared by every request)
# ----------------------------------------------------------------------------

def half_lives(cfg: Config) -> np.ndarray:
    """Half-life in steps, log-uniform in [1, 4096]: [H] (GDN) or [H, dk] (KDA)."""
    shape = (cfg.heads,) if cfg.variant == GDN else (cfg.heads, cfg.dk)
    key = derive_key(cfg.table_seed, S_GATE)
    u = uniform01(key, np.arange(int(np.prod(shape))))
    return np.exp2(12.0 * u).reshape(shape)


def gates64(cfg: Config) -> np.ndarray:
    """Retention gates alpha = 0.5 ** (1 / h) in float64."""
    return np.power(0.5, 1.0 / half_lives(cfg))


def gates(cfg: Config) -> np.ndarray:
    return gates64(cfg).astype(np.float32)


def rho(cfg: Config) -> np.ndarray:
    """Row-impact weights ~ LogNormal(0, sigma): float32 [H, dk], all > 0."""
    key = derive_key(cfg.table_seed, S_RHO)
    z = normal(key, np.arange(cfg.heads * cfg.dk))
    return np.exp(cfg.rho_sigma * z).astype(np.float32).reshape(cfg.heads, cfg.dk)


def allocate_bits(weights: np.ndarray, choices, avg_bits: float, n_pivots: int,
                  pivot_order: np.ndarray) -> np.ndarray:
    """Greedy lifetime-weighted bit allocation under an average budget.

    weights: lifetime weight per unit (larger = longer-lived).  The first
    n_pivots units of pivot_order become FP16 pivots (16 bits each, counted in
    the budget).  Every other unit starts at min(choices); the upgrade to the
    next allowed width with the largest weight * (4**-b - 4**-b') / (b' - b)
    that still fits the remaining budget is applied until none fits.  Ties go to
    the lower unit index.
    """
    n = weights.shape[0]
    choices = sorted(choices)
    bits = np.full(n, choices[0], dtype=np.int64)
    piv = np.asarray(pivot_order[:n_pivots], dtype=np.int64)
    bits[piv] = PIVOT_BITS
    budget = int(round(avg_bits * n))
    remaining = budget - int(bits.sum())
    if remaining < 0:
        raise ValueError("bit budget below the minimum width")
    nxt = {b: (choices[i + 1] if i + 1 < len(choices) else None) for i, b in enumerate(choices)}

    def gain(u):
        b = int(bits[u]); b2 = nxt[b]
        return weights[u] * (4.0 ** -b - 4.0 ** -b2) / (b2 - b), b2 - b

    heap = []
    is_piv = np.zeros(n, dtype=bool); is_piv[piv] = True
    for u in range(n):
        if not is_piv[u] and nxt[int(bits[u])] is not None:
            g, cost = gain(u)
            heap.append((-g, u, cost))
    heapq.heapify(heap)
    while heap and remaining > 0:
        negg, u, cost = heapq.heappop(heap)
        if cost > remaining:
            continue  # the budget only shrinks, so this upgrade never fits again
        bits[u] = nxt[int(bits[u])]
        remaining -= cost
        if nxt[int(bits[u])] is not None:
            g, c2 = gain(u)
            heapq.heappush(heap, (-g, u, c2))
    return bits


def bit_table(cfg: Config) -> np.ndarray:
    """Row widths, uint8 [H, dk]: values in cfg.bits_choices or 16 (pivot).

    Gated-DeltaNet allocates per head (every row of a head has one width);
    KDA allocates per key row.
    """
    h = half_lives(cfg)
    alpha = gates64(cfg)
    units = h.reshape(-1)
    abar = alpha.reshape(-1)  # one gate per unit, so exp(mean log alpha) = alpha
    w = 1.0 / (1.0 - abar * abar)
    n = units.shape[0]
    n_piv = int(math.ceil(cfg.pivot_frac * n - 1e-9)) if cfg.pivot_frac > 0 else 0
    order = np.lexsort((np.arange(n), -units))  # longest half-life first, ties low index
    if len(cfg.bits_choices) == 1 and n_piv == 0:
        b = np.full(n, cfg.bits_choices[0], dtype=np.int64)
    else:
        b = allocate_bits(w, cfg.bits_choices, cfg.avg_bits, n_piv, order)
    if cfg.variant == GDN:
        out = np.repeat(b[:, None], cfg.dk, axis=1)
    else:
        out = b.reshape(cfg.heads, cfg.dk)
    return out.astype(np.uint8)


def query_gains(cfg: Config) -> np.ndarray:
    """Per (head, key row) query gains, float64 [H, dk], applied before the
    normalisation of q: ones when cfg.q_gain_sigma is 0, else LogNormal(0, sigma),
    so that key rows weigh differently in the readout."""
    if cfg.q_gain_sigma <= 0:
        return np.ones((cfg.heads, cfg.dk))
    key = derive_key(cfg.table_seed, S_Q_GAIN)
    z = normal(key, np.arange(cfg.heads * cfg.dk))
    return np.exp(cfg.q_gain_sigma * z).reshape(cfg.heads, cfg.dk)


def outlier_gains(cfg: Config):
    """(k_gain [H, dk], v_gain [H, dv]) float64; ones when the config has no outliers."""
    kg = np.ones((cfg.heads, cfg.dk))
    vg = np.ones((cfg.heads, cfg.dv))
    if cfg.outlier_frac <= 0:
        return kg, vg
    nk = int(math.ceil(cfg.outlier_frac * cfg.dk - 1e-9))
    nv = int(math.ceil(cfg.outlier_frac * cfg.dv - 1e-9))
    for h in range(cfg.heads):
        uk = uniform01(derive_key(cfg.table_seed, S_OUT_K, h), np.arange(cfg.dk))
        uv = uniform01(derive_key(cfg.table_seed, S_OUT_V, h), np.arange(cfg.dv))
        kg[h, np.argsort(uk, kind="stable")[:nk]] = cfg.outlier_gain
        vg[h, np.argsort(uv, kind="stable")[:nv]] = cfg.outlier_gain
    return kg, vg


# ----------------------------------------------------------------------------
# per-step inputs
# ----------------------------------------------------------------------------

def step_inputs(cfg: Config, t: int, requests=None):
    """Inputs of decode step t for the given requests (default: all).

    Returns a dict of float32 arrays: q, k [R, H, dk]; v [R, H, dv];
    beta [R, H]; alpha [R, H] (GDN) or [R, H, dk] (KDA).  Step indices below
    zero are the warm-up steps that build the initial state.
    """
    req = np.arange(cfg.batch) if requests is None else np.asarray(requests, dtype=np.int64)
    R, H = req.shape[0], cfg.heads
    bb, hh = np.meshgrid(req, np.arange(H), indexing="ij")
    kg, vg = outlier_gains(cfg)

    def field(stream, n):
        key = derive_key(cfg.input_seed, stream, bb[..., None], hh[..., None], t)
        return normal(key, np.arange(n)[None, None, :])

    k = field(S_K, cfg.dk) * kg[None]
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    q = field(S_Q, cfg.dk)
    if cfg.q_gain_sigma > 0:
        q = q * query_gains(cfg)[None]
    q = q / np.linalg.norm(q, axis=-1, keepdims=True)
    v = field(S_V, cfg.dv) * vg[None]
    zb = normal(derive_key(cfg.input_seed, S_BETA, bb, hh, t), np.zeros_like(bb))
    beta = 1.0 / (1.0 + np.exp(-zb))
    a = gates(cfg)
    alpha = np.broadcast_to(a[None], (R,) + a.shape)
    return {
        "q": q.astype(np.float32), "k": k.astype(np.float32), "v": v.astype(np.float32),
        "beta": beta.astype(np.float32), "alpha": np.ascontiguousarray(alpha, dtype=np.float32),
    }


# Calibration rollouts: requests and steps of their own (counter ranges no
# serving step or request uses), the same generators otherwise.
CALIB_REQUEST0 = 1 << 20
CALIB_STEP0 = 1 << 20


def calibration_requests(batch: int) -> np.ndarray:
    return CALIB_REQUEST0 + np.arange(batch)


def calibration_inputs(cfg: Config, tau: int, batch: int):
    """Inputs of calibration step tau (0, 1, ...) for `batch` calibration requests."""
    return step_inputs(cfg, CALIB_STEP0 + tau, calibration_requests(batch))


def parity_requests(cfg: Config):
    """Requests the oracle follows on large batches: {0, 1, B/2, B-1}."""
    B = cfg.batch
    return sorted(set([0, min(1, B - 1), B // 2, B - 1]))


# ----------------------------------------------------------------------------
# packed pool layout (format arithmetic only)
# ----------------------------------------------------------------------------

GROUP_ROWS, GROUP_COLS, SLAB_COLS = 16, 4, 16


def storage_rows(bits_head: np.ndarray) -> np.ndarray:
    """key_of[s]: the key row stored as storage row s.  Key order when the head
    has one width; otherwise the key rows sorted by width (widest first, ties
    by key index), the j-th stored as row 16 (j % RG) + j // RG (RG = dk/16),
    so that every row group holds rows of the same widths."""
    bits_head = np.asarray(bits_head)
    dk = bits_head.shape[0]
    if np.all(bits_head == bits_head[0]):
        return np.arange(dk)
    rg = dk // GROUP_ROWS
    order = np.lexsort((np.arange(dk), -bits_head.astype(np.int64)))
    key_of = np.empty(dk, dtype=np.int64)
    j = np.arange(dk)
    key_of[GROUP_ROWS * (j % rg) + j // rg] = order
    return key_of


def position_widths(bits_head: np.ndarray) -> np.ndarray:
    """F[p], p < 16: the field width of row position p (storage row 16 g + p of
    every row group g), the widest row at that position over the groups."""
    bits_head = np.asarray(bits_head)
    dk = bits_head.shape[0]
    sb = bits_head[storage_rows(bits_head)].astype(np.int64)
    return sb.reshape(dk // GROUP_ROWS, GROUP_ROWS).max(axis=0)


def stream_words(bits: np.ndarray) -> np.ndarray:
    """32-bit words per stream of each head, [H]: ceil(4 sum_p F[p] / 32)."""
    H, dk = bits.shape
    out = np.zeros(H, dtype=np.int64)
    for h in range(H):
        out[h] = (GROUP_COLS * int(position_widths(bits[h]).sum()) + 31) // 32
    return out


def head_item_bytes(bits: np.ndarray, dv: int) -> np.ndarray:
    """Bytes of one packed (request, head) item: r[dk] f32 | c[dv] f32 | slabs,
    dv/16 slabs of (dk/16) * 4 interleaved streams of stream_words words each."""
    dk = bits.shape[1]
    n_streams = (dk // GROUP_ROWS) * GROUP_COLS
    return 4 * dk + 4 * dv + 4 * n_streams * (dv // SLAB_COLS) * stream_words(bits)


def item_offsets(bits: np.ndarray, dv: int, batch: int) -> np.ndarray:
    """Byte offset of every item (b, h) in the pool, shape [B, H]; plus total."""
    sz = head_item_bytes(bits, dv)
    per_req = int(sz.sum())
    pre = np.concatenate([[0], np.cumsum(sz)[:-1]])
    offs = np.arange(batch, dtype=np.int64)[:, None] * per_req + pre[None, :]
    return offs, per_req * batch
