"""Plain CPU oracle of the QSA (Qwen Sparse Attention) decode hot path.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference leg may import or call this module. The product path
(the CUDA library and its Python binding) never imports it and shares no code
with it; the only module both sides use is `synth` (seeded inputs, no method
arithmetic).

Everything is float64 numpy, written for a reader to check against the pages by
eye: no blocking, fusion or reordering beyond the definitions below. A library
matmul serves as the dot-product step.

Sources (web pages; cited below by short name and section):
  Part 10  = "第10回 EVO-X2（Ryzen AI Max+ 395 / 128GB）+ Qwen3.8-Flash-Next用の
             llama.cpp改造で長コンテキストのTGを高速化した話" (qiita, ariera)
     §QSA indexer         : section "QSAとQSA indexerについて", subsection "QSA indexer"
     §COMMON-004          : section "incremental pooled-key cache（COMMON-004）"
     §FA-scaling          : section "なぜFlash Attentionがcontext長に比例していたのか"
     §COMMON-005          : section "selected QSA K/V gather（COMMON-005）"
     §COMMON-006          : section "block-domain top-k（COMMON-006）実装は見送り"

What the method computes (Part 10 §QSA indexer, §COMMON-004..006):
  1. indexer keys are summarised per 4-token micro-block: mean pool -> RMS norm ->
     RoPE at the block position; completed summaries are cached per layer and only
     new blocks are computed (COMMON-004);
  2. the current query is scored against every completed block; the top-k blocks
     covering indexer_top_k tokens are chosen, plus the still-open tail block
     (at most 2048 + 4 - 1 = 2051 cells);
  3. only those K/V cells are gathered (COMMON-005) and
  4. ordinary (GQA) softmax attention runs over them.

Readings taken where the pages are silent (each one is listed in the design notes):
  R1 score_b = sum_h w_h * ReLU(q~_h . p_b) / sqrt(d_idx)  (the pages give no formula);
     one pooled key per block is shared by all indexer heads.
  R2 RoPE is the NeoX half-split rotation over all d dims: pair (i, i + d/2),
     theta_i = base^(-2i/d), base 10000; z_i = x_i + j*x_{i+d/2} is multiplied by
     exp(j * pos * theta_i). Switches for the other readings: rope_dims = R < d rotates
     only the first R dims (pairs (i, i + R/2), theta_i = base^(-2i/R)) and passes the
     rest through; rope_interleaved pairs (2i, 2i + 1) instead (GPT-J style).
  R3 the position of block b is its first token, pos(b) = 4b; the query sits at
     position n-1 (n = context length including the current token). Switches:
     pos(b) = stride*b + offset, query position floor(stride*(n-1)/4); stride 1 puts
     both in the block domain (pos(b) = b, query at the index of its own block).
  R4 RMS norm r = m / sqrt(mean(m^2) + eps) * g with eps 1e-6, unit gain unless a
     gain vector is given.
  R5 pooled summaries are stored as f16 (round to nearest even), like the cache.
  R6 top-k ties go to the lower block index; if B <= K every block is selected; the
     selected blocks are returned in ascending order.
  R7 the tail is the n mod 4 tokens of the open block; a block that has just
     completed is scored like any other, not force-included.
  R8 attention: scale 1/sqrt(D), query head i uses KV head floor(i / (Hq/Hkv)), no
     extra mask, sink, gate or softcap.
  R11 verifying T drafted tokens at once is T single-token steps: query t (token n-T+t)
     sees the blocks completed within its first n-T+t+1 tokens and its own open tail; a
     rollback drops rejected tokens and the summaries of blocks they completed (Part 10
     §COMMON-004: speculative writes must not corrupt the cached range).
  R12 FP8 K/V cache (optional): per (token, KV head) row, scale = amax/448 and e4m3 codes
     of x * 448/amax (nearest-even, saturating); attention reads code * scale.
  R13 8-bit pooled keys (optional): each f16 summary p_b (R5) is stored as e4m3 codes with
     one f32 scale, by the R12 rule applied to the row; the indexer scores code * scale.

Also stated here: the sharded (context-parallel) form of one step, whose local top-K
candidates, merged selection and (o, lse) partials reproduce the single-device step.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BLOCK = 4  # micro-block size = compression ratio 4 (Part 10 §QSA indexer)


@dataclass(frozen=True)
class QsaShape:
    """Layer shapes the oracle needs (its own copy; it imports nothing from the product)."""

    d_idx: int
    n_idx_heads: int
    top_k_tokens: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    rope_dims: int = 0             # rotary dims R; 0 = all d_idx (reading R2)
    rope_interleaved: bool = False  # pairs (2i, 2i+1) instead of (i, i+R/2) (reading R2)
    rope_pos_stride: int = 4       # pos(b) = stride*b + offset (reading R3)
    rope_pos_offset: int = 0

    @property
    def k_blocks(self) -> int:
        # indexer_top_k tokens / compression ratio 4 (Part 10 §FA-scaling)
        return self.top_k_tokens // BLOCK

    @property
    def rotary_dims(self) -> int:
        return self.rope_dims or self.d_idx

    @classmethod
    def of(cls, wl, **rope) -> "QsaShape":
        return cls(wl.d_idx, wl.n_idx_heads, wl.top_k_tokens, wl.n_q_heads, wl.n_kv_heads,
                   wl.head_dim, wl.rope_base, wl.rms_eps, **rope)


def to_f16(x) -> np.ndarray:
    """Round float64 values to f16, nearest-even, directly from double (reading R5)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16)


# ---------------------------------------------------------------------------
# Step 1: pooled summaries (Part 10 §QSA indexer: average pooling -> RMS norm -> RoPE)
# ---------------------------------------------------------------------------

def rope_frequencies(dim: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/dim), i < dim/2, dim = the rotary dims (reading R2)."""
    i = np.arange(dim // 2, dtype=np.float64)
    return base ** (-2.0 * i / dim)


def rope_pairs(d: int, rope_dims: int = 0, interleaved: bool = False):
    """The rotation pairs (a_i, b_i), i < R/2, of a d-wide vector (reading R2).

    NeoX half-split: (i, i + R/2); interleaved (GPT-J): (2i, 2i + 1). Dims >= R are
    in no pair. R = rope_dims, or d when rope_dims is 0.
    """
    r = rope_dims or d
    if r % 2 or not 0 < r <= d:
        raise ValueError("rotary dims must be even and within the vector")
    i = np.arange(r // 2)
    return (2 * i, 2 * i + 1) if interleaved else (i, i + r // 2)


def rope(x, pos, base: float, rope_dims: int = 0, interleaved: bool = False) -> np.ndarray:
    """RoPE of the last axis of x at position(s) pos (reading R2).

    x has shape [..., d]; pos is a scalar or broadcasts against x[..., 0]. Pair i,
    (x_a, x_b) = (x[a_i], x[b_i]), is read as the complex number x_a + j*x_b and
    multiplied by exp(j * pos * theta_i); dims in no pair are copied unchanged.
    """
    x = np.asarray(x, dtype=np.float64)
    a, b = rope_pairs(x.shape[-1], rope_dims, interleaved)
    angle = np.multiply.outer(np.asarray(pos, dtype=np.float64), rope_frequencies(2 * a.size, base))
    c, s = np.cos(angle), np.sin(angle)
    xa, xb = x[..., a], x[..., b]
    out = x.copy()
    out[..., a] = xa * c - xb * s
    out[..., b] = xa * s + xb * c
    return out


def shape_rope(x, pos, shape: "QsaShape") -> np.ndarray:
    """rope() with the layer's rotary switches."""
    return rope(x, pos, shape.rope_base, shape.rope_dims, shape.rope_interleaved)


def mean_pool(raw_block) -> np.ndarray:
    """Average of the 4 indexer keys of a micro-block: [..., 4, d] -> [..., d]."""
    raw = np.asarray(raw_block, dtype=np.float64)
    return raw.sum(axis=-2) / BLOCK


def rms_normalize(m, eps: float, gain=None) -> np.ndarray:
    """r = m / sqrt(mean(m^2) + eps) * g over the last axis (reading R4)."""
    m = np.asarray(m, dtype=np.float64)
    r = m / np.sqrt(np.mean(m * m, axis=-1, keepdims=True) + eps)
    return r if gain is None else r * np.asarray(gain, dtype=np.float64)


def block_position(b, stride: int = BLOCK, offset: int = 0):
    """Position of micro-block b: stride*b + offset; by default its first token 4b (reading R3)."""
    return stride * np.asarray(b) + offset


def query_position(n: int, stride: int = BLOCK) -> int:
    """Position of the current token n-1 on the block-position scale: floor(stride*(n-1)/4) (R3)."""
    return (stride * (n - 1)) // BLOCK


def pooled_summaries(raw_idx, first_block: int, last_block: int, shape: QsaShape,
                     gain=None) -> np.ndarray:
    """f16 summaries p_b of blocks [first_block, last_block) from the raw indexer keys."""
    d = shape.d_idx
    blocks = np.arange(first_block, last_block)
    raw = np.asarray(raw_idx[BLOCK * first_block:BLOCK * last_block]).reshape(-1, BLOCK, d)
    m = mean_pool(raw)
    r = rms_normalize(m, shape.rms_eps, gain)
    p = shape_rope(r, block_position(blocks, shape.rope_pos_stride, shape.rope_pos_offset), shape)
    return to_f16(p)


def pooled_cache_full(raw_idx, n: int, shape: QsaShape, gain=None) -> np.ndarray:
    """The old per-step path: every completed block recomputed (Part 10 §COMMON-004, 従来)."""
    return pooled_summaries(raw_idx, 0, n // BLOCK, shape, gain)


class PooledKeyCache:
    """Persistent per-layer pooled-key cache, updated incrementally (Part 10 §COMMON-004).

    Only blocks that completed (or were invalidated) since the last update are
    computed; rows below `n_pooled` are reused as they are.
    """

    def __init__(self, max_blocks: int, d_idx: int):
        self.rows = np.zeros((max_blocks, d_idx), dtype=np.float16)
        self.n_pooled = 0

    def update(self, raw_idx, n: int, shape: QsaShape, gain=None) -> int:
        b_done = n // BLOCK
        new = max(0, b_done - self.n_pooled)
        if new:
            self.rows[self.n_pooled:b_done] = pooled_summaries(raw_idx, self.n_pooled, b_done,
                                                               shape, gain)
            self.n_pooled = b_done
        return new

    def invalidate(self, from_block: int) -> None:
        """State load / sequence edit: rows from `from_block` on are no longer trusted."""
        self.n_pooled = min(self.n_pooled, max(0, from_block))


# ---------------------------------------------------------------------------
# Step 2: indexer scores and block-domain top-k (Part 10 §QSA indexer, §COMMON-006)
# ---------------------------------------------------------------------------

def indexer_query(q_idx, n: int, shape: QsaShape) -> np.ndarray:
    """q~_h = RoPE(q_h, n-1): the current token's indexer query (readings R2, R3)."""
    return shape_rope(np.asarray(q_idx, dtype=np.float64), query_position(n, shape.rope_pos_stride), shape)


def block_scores(pooled, q_idx, w, n: int, shape: QsaShape) -> np.ndarray:
    """s_b = sum_h w_h * ReLU(q~_h . p_b) / sqrt(d_idx) for every completed block b < n/4 (R1)."""
    b_done = n // BLOCK
    p = np.asarray(pooled[:b_done], dtype=np.float64)             # [B, d]
    q = indexer_query(q_idx, n, shape)                             # [H, d]
    dots = p @ q.T                                                 # [B, H]
    return (np.maximum(dots, 0.0) @ np.asarray(w, dtype=np.float64)) / np.sqrt(shape.d_idx)


def topk_blocks(scores, k_blocks: int) -> np.ndarray:
    """The k_blocks highest-scoring blocks, ties to the lower index, ascending (R6)."""
    s = np.asarray(scores, dtype=np.float64)
    if not np.all(np.isfinite(s)):
        raise ValueError("indexer scores must be finite")
    order = np.lexsort((np.arange(s.size), -s))   # by score descending, then index ascending
    return np.sort(order[:min(k_blocks, s.size)]).astype(np.int64)


def expand_cells(sel_blocks, n: int) -> np.ndarray:
    """Selected blocks -> their 4 cells each, then the open tail [4B, n) (Part 10 §COMMON-006, R7)."""
    sel = np.asarray(sel_blocks, dtype=np.int64)
    cells = (BLOCK * sel[:, None] + np.arange(BLOCK)[None, :]).reshape(-1)
    tail = np.arange(BLOCK * (n // BLOCK), n, dtype=np.int64)
    return np.concatenate([cells, tail])


# ---------------------------------------------------------------------------
# Step 3+4: selected K/V gather and GQA attention (Part 10 §COMMON-005, reading R8)
# ---------------------------------------------------------------------------

def sparse_attention(q, k_cache, v_cache, cells, shape: QsaShape) -> np.ndarray:
    """o_i = sum_c softmax_c(q_i . K[c, g] / sqrt(D)) V[c, g], g = i // (Hq/Hkv), over `cells`."""
    q = np.asarray(q, dtype=np.float64)
    cells = np.asarray(cells, dtype=np.int64)
    group = shape.n_q_heads // shape.n_kv_heads
    out = np.zeros((shape.n_q_heads, shape.head_dim), dtype=np.float64)
    for i in range(shape.n_q_heads):
        g = i // group
        kc = np.asarray(k_cache[cells, g], dtype=np.float64)     # gathered rows [n_c, D]
        vc = np.asarray(v_cache[cells, g], dtype=np.float64)
        logits = kc @ q[i] / np.sqrt(shape.head_dim)
        e = np.exp(logits - logits.max())
        out[i] = (e @ vc) / e.sum()
    return out


# ---------------------------------------------------------------------------
# Context-parallel form of one decode step (the pages run one GPU; this is the sharded form).
# The context of one layer is split into contiguous, block-aligned shards; the last
# shard holds the open tail. Each shard scores its own completed blocks (the query at
# the global position n-1, the blocks at their global positions), keeps its local top-K
# as (score, global block) candidates, and after an exchange every shard takes the global
# top-K of all candidates with the same rule. Each shard attends over its selected cells
# and returns (o, lse) per head; the exact merge is o = sum_r exp(lse_r - LSE) o_r with
# LSE = log sum_r exp(lse_r). Any block of the global top-K is in its shard's local top-K
# (fewer than K blocks beat it anywhere), and candidates listed shard by shard in
# ascending block order keep "ties to the lower block" intact, so the result equals the
# single-device step.
# ---------------------------------------------------------------------------

def shard_candidates(pooled_shard, first_block: int, q_idx, w, n: int, shape: QsaShape):
    """Local top-K of one shard: (scores, global block ids), ascending by block.
    pooled_shard holds the summaries of global blocks first_block, first_block+1, ...
    (completed ones only)."""
    q = indexer_query(q_idx, n, shape)
    p = np.asarray(pooled_shard, dtype=np.float64)
    s = (np.maximum(p @ q.T, 0.0) @ np.asarray(w, dtype=np.float64)) / np.sqrt(shape.d_idx)
    local = topk_blocks(s, shape.k_blocks) if len(s) else np.zeros(0, np.int64)
    return s[local], local + first_block


def merge_candidates(cand_scores, cand_blocks, k_blocks: int) -> np.ndarray:
    """Global top-K from the shards' candidates listed shard by shard (block order)."""
    scores = np.concatenate(cand_scores) if cand_scores else np.zeros(0)
    blocks = np.concatenate(cand_blocks) if cand_blocks else np.zeros(0, np.int64)
    pick = topk_blocks(scores, k_blocks) if len(scores) else np.zeros(0, np.int64)
    return blocks[pick]


def attention_partial(q, k_cache, v_cache, cells, shape: QsaShape):
    """(o, lse) per query head over `cells`: o normalised, lse = log sum_c exp(logit_c);
    an empty cell set gives o = 0 and lse = -inf."""
    q = np.asarray(q, dtype=np.float64)
    cells = np.asarray(cells, dtype=np.int64)
    group = shape.n_q_heads // shape.n_kv_heads
    o = np.zeros((shape.n_q_heads, shape.head_dim))
    lse = np.full(shape.n_q_heads, -np.inf)
    if len(cells) == 0:
        return o, lse
    for i in range(shape.n_q_heads):
        g = i // group
        kc = np.asarray(k_cache[cells, g], dtype=np.float64)
        vc = np.asarray(v_cache[cells, g], dtype=np.float64)
        logits = kc @ q[i] / np.sqrt(shape.head_dim)
        m = logits.max()
        e = np.exp(logits - m)
        o[i] = (e @ vc) / e.sum()
        lse[i] = m + np.log(e.sum())
    return o, lse


def merge_partials(partials):
    """Exact merge of per-shard (o, lse) into the attention over the union of the cells."""
    lse = np.stack([p[1] for p in partials])                   # [G, Hq]
    top = lse.max(axis=0)
    safe = np.where(np.isfinite(top), top, 0.0)
    wts = np.where(np.isfinite(lse), np.exp(lse - safe), 0.0)  # [G, Hq]
    den = wts.sum(axis=0)
    o = sum(wts[r][:, None] * partials[r][0] for r in range(len(partials)))
    return np.where(den[:, None] > 0, o / np.where(den > 0, den, 1.0)[:, None], 0.0)


# ---------------------------------------------------------------------------
# FP8 K/V cache. The Qwen3.8-Flash-Next parameter-tuning post on EVO-X2 (section
# "KV cacheをQ8_0にしてみる") tried an 8-bit K/V cache and gives no layout.
# Reading R12: one f32 scale per (token, KV head) row, scale = amax / 448, codes =
# e4m3(x * (448 / amax)) with round-to-nearest-even and saturation to +-448; an all-zero
# row gets scale 1 and zero codes. Attention runs over code * scale.
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """Value of an e4m3 byte: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent 0 is subnormal (m * 2^-9); S.1111.111 is NaN (no infinities)."""
    code = int(code)
    sign = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_encode(x) -> np.ndarray:
    """Round float32 values to e4m3 bytes: nearest representable value, ties to the even
    mantissa, magnitudes above 448 saturate to 448, the sign bit kept for zero results
    (the values here are finite)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    mag = np.abs(x)
    # quantum of the binade of |x| (2^(e-3)), with the subnormal quantum 2^-9 below 2^-6
    e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    e = np.maximum(e, -6.0)
    quantum = 2.0 ** (e - 3)
    k = np.round(mag / quantum)          # numpy rounds halves to even
    r = np.minimum(k * quantum, E4M3_MAX)
    # encode r (exactly representable) into sign/exponent/mantissa bits
    out = np.zeros(x.shape, dtype=np.uint8)
    nz = r > 0
    er = np.floor(np.log2(np.where(nz, r, 1.0)))
    sub = nz & (er < -6)
    norm = nz & ~sub
    m_sub = np.where(sub, r / 2.0 ** -9, 0).astype(np.int64)
    exp_n = np.where(norm, er + 7, 0).astype(np.int64)
    m_n = np.where(norm, (r / 2.0 ** np.where(norm, er, 0) - 1.0) * 8.0, 0).astype(np.int64)
    bits = np.where(sub, m_sub, (exp_n << 3) | m_n)
    out[...] = np.where(np.signbit(x), 0x80, 0) | bits   # -0 and negatives that round to 0 keep the sign
    return out


def quantize_kv_rows(rows):
    """[..., D] f16 rows -> (e4m3 codes [..., D] uint8, scales [...] f32), reading R12.
    The scale and the multiplier are single f32 operations, like the library's."""
    x = np.asarray(rows, dtype=np.float16).astype(np.float32)
    amax = np.max(np.abs(x), axis=-1)
    zero = amax == 0
    safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
    scale = np.where(zero, np.float32(1.0), safe / np.float32(E4M3_MAX)).astype(np.float32)
    mult = np.where(zero, np.float32(0.0), np.float32(E4M3_MAX) / safe).astype(np.float32)
    codes = e4m3_encode((x * mult[..., None]).astype(np.float32))
    return codes, scale


_E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)])


def pooled_fp8_rows(pooled_f16):
    """8-bit pooled keys (R13): the f16 summaries [B, d] as e4m3 codes [B, d] and one f32
    scale per row [B], by the R12 rule."""
    return quantize_kv_rows(np.asarray(pooled_f16, np.float16))


def dequantize_kv_rows(codes, scales) -> np.ndarray:
    """code * scale in float64."""
    return _E4M3_TABLE[np.asarray(codes)] * np.asarray(scales, dtype=np.float64)[..., None]


# ---------------------------------------------------------------------------
# One layer, step by step (mirrors the library's calls)
# ---------------------------------------------------------------------------

class OracleLayer:
    """One QSA layer's caches and the decode-step calls, in plain numpy."""

    def __init__(self, shape: QsaShape, max_ctx: int, gain=None, kv_fp8: bool = False, pooled_fp8: bool = False):
        self.shape = shape
        self.max_ctx = max_ctx
        self.gain = gain
        self.kv_fp8 = kv_fp8
        self.pooled_fp8 = pooled_fp8
        kv_shape = (max_ctx, shape.n_kv_heads, shape.head_dim)
        # attention reads self.k / self.v: the f16 rows, or code * scale (reading R12)
        self.k = np.zeros(kv_shape, dtype=np.float64 if kv_fp8 else np.float16)
        self.v = np.zeros_like(self.k)
        if kv_fp8:
            self.k_codes = np.zeros(kv_shape, dtype=np.uint8)
            self.v_codes = np.zeros(kv_shape, dtype=np.uint8)
            self.kv_scales = np.zeros((max_ctx, shape.n_kv_heads, 2), dtype=np.float32)
        self.idx = np.zeros((max_ctx, shape.d_idx), dtype=np.float16)
        self.pooled = PooledKeyCache(max_ctx // BLOCK, shape.d_idx)
        self.n = 0

    def append_tokens(self, k, v, idx) -> None:
        k = np.asarray(k, np.float16).reshape(-1, self.shape.n_kv_heads, self.shape.head_dim)
        m = k.shape[0]
        if self.n + m > self.max_ctx:
            raise ValueError("context capacity exceeded")
        v = np.asarray(v, np.float16).reshape(k.shape)
        if self.kv_fp8:
            for rows, codes, which, deq in ((k, self.k_codes, 0, self.k), (v, self.v_codes, 1, self.v)):
                c, sc = quantize_kv_rows(rows)
                codes[self.n:self.n + m] = c
                self.kv_scales[self.n:self.n + m, :, which] = sc
                deq[self.n:self.n + m] = dequantize_kv_rows(c, sc)
        else:
            self.k[self.n:self.n + m] = k
            self.v[self.n:self.n + m] = v
        self.idx[self.n:self.n + m] = np.asarray(idx, np.float16).reshape(m, self.shape.d_idx)
        self.n += m

    def update_pooled_cache(self) -> int:
        return self.pooled.update(self.idx, self.n, self.shape, self.gain)

    @property
    def scored_rows(self) -> np.ndarray:
        """What the indexer scores: the f16 summaries, or with 8-bit pooled keys their
        e4m3 codes * scale (R13)."""
        if not self.pooled_fp8:
            return self.pooled.rows
        codes, scales = pooled_fp8_rows(self.pooled.rows)
        return dequantize_kv_rows(codes, scales)

    def scores(self, q_idx, w) -> np.ndarray:
        if self.pooled.n_pooled != self.n // BLOCK:
            raise ValueError("pooled cache is stale")
        return block_scores(self.scored_rows, q_idx, w, self.n, self.shape)

    def index_topk(self, q_idx, w):
        s = self.scores(q_idx, w)
        return topk_blocks(s, self.shape.k_blocks), s

    def gather_cells(self, sel_blocks) -> np.ndarray:
        return expand_cells(sel_blocks, self.n)

    def attend(self, q, cells) -> np.ndarray:
        return sparse_attention(q, self.k, self.v, cells, self.shape)

    def rollback(self, n_keep: int) -> None:
        """Drop the tokens at positions >= n_keep (rejected speculative tokens). Summaries of
        blocks those tokens completed are no longer trusted (Part 10 §COMMON-004: dirty
        speculative writes must not corrupt the cached range)."""
        self.n = min(self.n, max(0, n_keep))
        self.pooled.invalidate(self.n // BLOCK)

    def multi_query_step(self, k, v, idx, q_idx, w, q):
        """Verify T tokens at once (speculative / multi-token decode): append all T, bring the
        pooled cache up to date, then query t (token n-T+t) selects and attends over the
        context it can see, n_t = n-T+t+1 tokens: the blocks completed within n_t and its own
        open tail. k, v: [T, Hkv, D]; idx: [T, d]; q_idx: [T, H, d]; w: [T, H]; q: [T, Hq, D]."""
        T = len(k)
        self.append_tokens(k, v, idx)
        self.update_pooled_cache()
        outs = []
        for t in range(T):
            n_t = self.n - T + t + 1
            s = block_scores(self.scored_rows, q_idx[t], w[t], n_t, self.shape)
            sel = topk_blocks(s, self.shape.k_blocks)
            cells = expand_cells(sel, n_t)
            outs.append({"sel": sel, "scores": s, "cells": cells, "out": self.attend(q[t], cells)})
        return outs

    def decode_step(self, k, v, idx, q_idx, w, q):
        """append -> incremental pooled update -> scores + top-k -> cells -> attention."""
        self.append_tokens(k[None], v[None], idx[None])
        self.update_pooled_cache()
        sel, s = self.index_topk(q_idx, w)
        cells = self.gather_cells(sel)
        return {"sel": sel, "scores": s, "cells": cells, "out": self.attend(q, cells)}
