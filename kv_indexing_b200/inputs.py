"""Seeded synthetic inputs for the LSA indexer / top-k / sparse-attention path.

This module only *draws* inputs. It holds none of the method's arithmetic: no
scores, no selection, no pooling, no attention. Both the CUDA path (through the
tests and ``bench.py``) and the CPU oracle consume the arrays it returns, so the
two sides always see identical bytes.

Element encodings used throughout:

* bf16 tensors are ``numpy.uint16`` arrays of raw bfloat16 bit patterns,
  produced from float32 draws by round-to-nearest-even on the 16 dropped bits.
* FP8 tensors are ``numpy.uint8`` arrays of OCP E4M3 ("e4m3fn") codes with a
  float32 scale per row (per key token, per query head).

Workload shapes follow the LSA pages: the LongCat Sparse Attention paper
(arXiv 2608.01662 summary page: streaming sink + window taking half of a
2048-entry budget, page size / recall for Hierarchical Indexing, 1M-token
contexts) and the DSA Lightning Indexer article (top-k 2048, MLA-style
latent KV). Needles stand in for the pages' suggested needle-in-a-haystack
probing (the release-news page, "Actionable Advice"); no benchmark item is
reproduced.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

# ---------------------------------------------------------------------------
# Workload descriptions
# ---------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: indexer, budget, hierarchy and attention shapes."""

    name: str
    B: int            # sequences
    L: int            # cached tokens per sequence (all sequences full)
    T: int            # queries per sequence, at positions L-T .. L-1
    H: int            # indexer heads
    d: int            # indexer head dim
    k: int            # token budget
    sink: int         # attention-sink prefix size
    window: int       # local sliding-window size
    needle_frac: float = 0.0   # planted needles as a fraction of L (per sequence)
    needles: int = 0           # or an absolute count per sequence
    P: int = 0                 # page size (0 = flat indexing)
    M: int = 0                 # recalled pages
    n_layers: int = 1          # cross-layer group size
    Hq: int = 128              # attention query heads
    d_qk: int = 576            # attention q/k dim
    d_v: int = 512             # attention v dim
    mla: bool = True           # V = first d_v columns of the latent K row
    scale: float = 1.0 / math.sqrt(576.0)
    fp8: bool = False          # also provide FP8-e4m3 indexer keys / queries
    m: int = 0                 # > 0: index compressed entries of m tokens (budget, sink, window in entries)

    @property
    def n_needles(self) -> int:
        if self.needles:
            return self.needles
        return int(round(self.needle_frac * self.L))


WORKLOADS: Dict[str, Workload] = {
    # Tiny correctness case: one sequence, last 64 positions as causal queries.
    "tiny_l2k": Workload(
        name="tiny_l2k", B=1, L=2048, T=64, H=4, d=64, k=256, sink=64, window=64,
        needles=16, Hq=8, d_qk=64, d_v=64, mla=False, scale=1.0 / 8.0),
    # Flat decode: 8 sequences of 128K tokens, one query each.
    "flat_decode_128k": Workload(
        name="flat_decode_128k", B=8, L=131072, T=1, H=64, d=128, k=2048, sink=64,
        window=960, needle_frac=0.01),
    # Flat prefill chunk: T=4096 causal queries at the end of a 64K sequence.
    "prefill_64k": Workload(
        name="prefill_64k", B=1, L=65536, T=4096, H=64, d=128, k=2048, sink=64,
        window=960, fp8=True),
    # Hierarchical decode at 1M tokens.
    "hier_decode_1m": Workload(
        name="hier_decode_1m", B=2, L=1048576, T=1, H=64, d=128, k=2048, sink=64,
        window=960, needle_frac=0.01, P=64, M=256),
    # Flat decode at 1M tokens: the hierarchical workload's inputs with the
    # hierarchy off (same seed => identical indexer inputs and needles).
    "flat_decode_1m": Workload(
        name="flat_decode_1m", B=2, L=1048576, T=1, H=64, d=128, k=2048, sink=64,
        window=960, needle_frac=0.01),
    # Cross-layer group: two layers share one indexer pass.
    "cli_group_256k": Workload(
        name="cli_group_256k", B=4, L=262144, T=1, H=64, d=128, k=2048, sink=64,
        window=960, needle_frac=0.01, P=64, M=256, n_layers=2),
    # The same group with flat indexing (hierarchy off).
    "cli_group_256k_flat": Workload(
        name="cli_group_256k_flat", B=4, L=262144, T=1, H=64, d=128, k=2048, sink=64,
        window=960, needle_frac=0.01, n_layers=2),
    # Compressed-entry decode: 1M tokens as 262144 entries of 4 tokens; 2048
    # entries chosen (16 sink + 240 window entries, the token budget's 64 / 960
    # in entries); attention over the chosen compressed latent entries.
    "compressed_decode_1m": Workload(
        name="compressed_decode_1m", B=4, L=1048576, T=1, H=64, d=128, k=2048, sink=16,
        window=240, needle_frac=0.01, m=4, fp8=True),
}


def scaled(w: Workload, **changes) -> Workload:
    """Return a copy of ``w`` with some fields replaced (for reduced-size cases)."""
    return dataclasses.replace(w, **changes)


# ---------------------------------------------------------------------------
# Element encoders (input preparation only)
# ---------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even.

    Inputs drawn here are finite normals, so no NaN/overflow handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact)."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


_E4M3_MAX = 448.0


def f32_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> OCP E4M3 codes, round to nearest even, saturating at +-448.

    E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent field 15 with
    mantissa 7 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.
    Field 0 encodes subnormals m/8 * 2^-6.
    """
    x = np.asarray(x, dtype=np.float64)
    sign = (x < 0) | ((x == 0) & np.signbit(x))
    a = np.minimum(np.abs(x), _E4M3_MAX)
    out = np.zeros(a.shape, dtype=np.int64)
    normal = a >= 2.0 ** -6
    # normals: a = (1 + m/8) * 2^e
    mant, exp = np.frexp(np.where(normal, a, 1.0))   # a = mant * 2^exp, mant in [0.5,1)
    e = exp - 1
    frac = mant * 2.0 - 1.0                           # in [0, 1)
    q = np.rint(frac * 8.0).astype(np.int64)          # ties to even
    carry = q == 8
    q = np.where(carry, 0, q)
    e = np.where(carry, e + 1, e)
    over = e > 8
    code_n = ((e + 7) << 3) | q
    code_n = np.where(over | (code_n > 0x7E), 0x7E, code_n)
    # subnormals: a = q/8 * 2^-6 = q * 2^-9
    qs = np.rint(a * 2.0 ** 9).astype(np.int64)       # 0..8 ; 8 -> min normal 0x08
    out = np.where(normal, code_n, qs)
    out = out | np.where(sign, 0x80, 0)
    return out.astype(np.uint8)


def quantize_e4m3_rows(x: np.ndarray, chunk_rows: int = 1 << 14) -> tuple:
    """Quantise along the last axis: scale = amax / 448, codes = e4m3(x / scale).

    Rows that are entirely zero get scale 1. Returns (codes uint8, scale float32).
    Rows are encoded chunk_rows at a time, so a 1M-token latent cache needs no
    more than a few hundred MB of temporaries; every row is independent.
    """
    x = np.asarray(x, dtype=np.float32)
    flat = x.reshape(-1, x.shape[-1])
    codes = np.empty(flat.shape, dtype=np.uint8)
    scale = np.empty(flat.shape[0], dtype=np.float32)
    for r0 in range(0, flat.shape[0], chunk_rows):
        blk = flat[r0:r0 + chunk_rows]
        amax = np.max(np.abs(blk), axis=-1)
        sc = np.where(amax > 0, amax / np.float32(_E4M3_MAX), np.float32(1.0)).astype(np.float32)
        codes[r0:r0 + chunk_rows] = f32_to_e4m3_bits(blk / sc[:, None])
        scale[r0:r0 + chunk_rows] = sc
    return codes.reshape(x.shape), scale.reshape(x.shape[:-1])


# ---------------------------------------------------------------------------
# Draws
# ---------------------------------------------------------------------------

# Independent sub-streams per tensor so each can be drawn alone.
_STREAM = {"q": 1, "w": 2, "k": 3, "needle": 4, "qa": 5, "kv": 6, "v": 7}


def _rng(seed: int, stream: str, extra: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), _STREAM[stream], int(extra)])


def normal_bf16(shape, rng: np.random.Generator, chunk: int = 1 << 26) -> np.ndarray:
    """N(0,1) draws rounded to bf16 bit patterns, generated in chunks."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        out[lo:hi] = f32_to_bf16_bits(rng.standard_normal(hi - lo, dtype=np.float32))
    return out.reshape(shape)


def positions(L: int, T: int) -> np.ndarray:
    """Absolute position of each of the T queries of a length-L sequence."""
    return np.arange(L - T, L, dtype=np.int64)


def entry_workload(w: Workload) -> Workload:
    """The workload seen over compressed entries: L // m entries, no compression."""
    return dataclasses.replace(w, L=w.L // w.m, m=0)


def make_compressed_inputs(w: Workload, seed: int) -> dict:
    """Indexer inputs over compressed entries of ``w.m`` tokens.

    The pages name no compressor, so the entry keys are drawn like token keys
    (N(0,1) bf16, with needles planted in the entries of the dynamic region; see
    make_indexer_inputs), as ``entry_keys`` [B, L/m, d] (plus e4m3 codes and
    per-entry scales when ``w.fp8``). seq_len counts tokens (L).
    """
    x = make_indexer_inputs(entry_workload(w), seed)
    x["entry_keys"] = x.pop("k_idx")
    if "k_idx_fp8" in x:
        x["entry_keys_fp8"] = x.pop("k_idx_fp8")
    x["seq_len"] = np.full((w.B,), w.L, dtype=np.int32)
    return x


def make_indexer_inputs(w: Workload, seed: int, with_needles: bool = True) -> dict:
    """Indexer inputs: q_idx [B,T,H,d] bf16, w [B,T,H] f32, k_idx [B,L,d] bf16.

    Needles: per sequence, ``w.n_needles`` keys are overwritten with a copy of
    a random query head's indexer vector plus N(0, 0.1) noise. For each needle a
    query t and head h are drawn uniformly, and its position uniformly (without
    replacement) from that query's dynamic region [sink, pos(t) - window].
    """
    B, T, H, d, L = w.B, w.T, w.H, w.d, w.L
    q = normal_bf16((B, T, H, d), _rng(seed, "q"))
    wt = _rng(seed, "w").random((B, T, H), dtype=np.float32)
    k = normal_bf16((B, L, d), _rng(seed, "k"))
    pos = positions(L, T)
    needle_pos = np.zeros((B, 0), dtype=np.int64)
    if with_needles and w.n_needles > 0:
        rng = _rng(seed, "needle")
        allpos = []
        qf = bf16_bits_to_f32(q)
        for b in range(B):
            taken = set()
            ts = rng.integers(0, T, size=w.n_needles)
            hs = rng.integers(0, H, size=w.n_needles)
            noise = rng.standard_normal((w.n_needles, d), dtype=np.float32) * np.float32(0.1)
            plist = []
            for i in range(w.n_needles):
                lo, hi = w.sink, int(pos[ts[i]]) - w.window   # inclusive range
                if hi < lo:
                    continue
                for _ in range(64):
                    s = int(rng.integers(lo, hi + 1))
                    if s not in taken:
                        break
                else:
                    continue
                taken.add(s)
                plist.append(s)
                k[b, s] = f32_to_bf16_bits(qf[b, ts[i], hs[i]] + noise[i])
            allpos.append(plist)
        width = max(len(p) for p in allpos)
        needle_pos = np.full((B, width), -1, dtype=np.int64)
        for b, p in enumerate(allpos):
            needle_pos[b, :len(p)] = p
    out = {
        "q_idx": q, "w": wt, "k_idx": k,
        "seq_len": np.full((B,), L, dtype=np.int32),
        "needle_pos": needle_pos,
    }
    if w.fp8:
        kf = bf16_bits_to_f32(k)
        k8, ks = quantize_e4m3_rows(kf)
        q8, qs = quantize_e4m3_rows(bf16_bits_to_f32(q))
        out.update({"k_idx_fp8": k8, "k_scale": ks, "q_idx_fp8": q8, "q_scale": qs})
    return out


def make_attn_inputs(w: Workload, seed: int, layer: int = 0) -> dict:
    """Attention inputs for one layer.

    MLA (``w.mla``): qa [B,T,Hq,d_qk] bf16 and one latent row per token
    kv [B,L,d_qk] bf16; V is the first d_v columns of that row.
    Otherwise separate k [B,L,d_qk] and v [B,L,d_v] bf16 arrays.
    """
    B, T, L = w.B, w.T, w.L
    qa = normal_bf16((B, T, w.Hq, w.d_qk), _rng(seed, "qa", layer))
    out = {"qa": qa}
    if w.mla:
        out["kv"] = normal_bf16((B, L, w.d_qk), _rng(seed, "kv", layer))
    else:
        out["k"] = normal_bf16((B, L, w.d_qk), _rng(seed, "kv", layer))
        out["v"] = normal_bf16((B, L, w.d_v), _rng(seed, "v", layer))
    return out


def needle_pages(needle_pos: np.ndarray, P: int) -> np.ndarray:
    """Page ids holding needles (for recall diagnostics)."""
    return np.where(needle_pos >= 0, needle_pos // P, -1)
