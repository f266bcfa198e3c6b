"""Plain CPU oracle for SageAttention-style quantized attention (forward).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import or run this module.
It shares no code, constant table or helper with the CUDA library.

What it computes, stage by stage, for one (sequence, query head) with its KV head:

1. K smoothing: subtract K's per-channel mean over tokens
   (glossary page "SageAttention(セージアテンション)", 概要 and 主な特徴・仕組み;
   heatdrop review "2–5× attention speedups without the accuracy apology tour",
   The interesting bit: outlier smoothing).
2. Per-block INT8 quantization of Q and smoothed K with scale max|x|/127
   (vibecrowd repo page "thu-ml--sageattention", How it works: INT8 for QK^T).
3. S = Q8 K8^T in exact integers (same page).
4. Dequantize, scale by 1/sqrt(d), online softmax over KV blocks
   (glossary page, 主な特徴・仕組み: FlashAttention-compatible usage).
5. P and V in FP8 e4m3, V with per-channel scales; PV accumulated per KV
   block, then added into the running output: two-level accumulation
   (vibecrowd page, How it works; heatdrop review, Key highlights).

Everything after the integer scores is done in float64.

Readings where the pages are silent (each is listed in the design doc):

* Q blocks are 128 tokens x d, K blocks are 64 tokens x d, per (sequence, head);
  the last block of a sequence may be short (its max ignores absent tokens).
* mu = fp32(fp64 sum over tokens / n); k_s = fp32(k - mu).
* s = fp32(a / 127), r = fp32(127 / a), x8 = clamp(rint_even(fp32(x * r)), -127, 127);
  a block with a == 0 gets s = 0 and all-zero codes.
* V: per-channel vmax over the sequence; sv = fp32(vmax / 448),
  v8 = e4m3_satfinite_rne(fp32(v * fp32(448 / vmax))); vmax == 0 -> sv = 0, codes 0.
* Online-softmax block T = 128 keys.  P8 = e4m3(448 * exp(x - m')) with m' the
  running max after the block; the running sum l adds the unquantized exp values.
* Output o = O * sv / (448 * l); lse = m + ln(l) (natural log of sum exp(x)).
* GQA: query head h reads KV head h // (Hq / Hkv).  Varlen: every packed
  sequence is an independent problem (its own mean, blocks and causal diagonal).
* Causal (equal query and key lengths): key j is masked for query i when j > i.

Parity of every function here is pinned by ``tests/test_oracle_pins.py``:
brute force on tiny inputs, closed forms, invariants and the OCP FP8 value table.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "BLKQ", "BLKK", "KV_TILE", "P_SCALE", "E4M3_MAX",
    "round_binary", "e4m3_round", "e4m3_encode", "e4m3_decode",
    "k_channel_mean", "smooth_k", "quantize_int8_blocks", "quantize_v_e4m3",
    "integer_scores", "online_softmax_pv", "attention_head", "sage_attention",
    "reference_attention", "attention_weights",
]

BLKQ = 128        # tokens per Q quantization block
BLKK = 64         # tokens per K quantization block
KV_TILE = 128     # keys per online-softmax block
E4M3_MAX = 448.0  # largest finite OCP E4M3 value: S.1111.110 = 1.75 * 2^8
P_SCALE = 448.0   # P (<= 1) is stored as e4m3(448 * P)


# --------------------------------------------------------------------------
# Exact rounding into small binary floating-point formats
# --------------------------------------------------------------------------

def round_binary(x, p: int, emin: int, max_finite: float | None = None) -> np.ndarray:
    """Round float64 values to the nearest value of a binary format, ties to even.

    ``p`` is the significand width including the implicit bit, ``emin`` the
    exponent of the smallest normal number (its value is 2**emin); below it the
    spacing stays 2**(emin - p + 1) (gradual underflow).  With ``max_finite``
    set, magnitudes beyond it saturate to it (the "satfinite" behaviour).
    The scaling by powers of two is exact, so np.rint (ties-to-even) is the only
    rounding step.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                     # x = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e - 1, emin)            # exponent of the leading bit, clamped
    quantum = np.ldexp(1.0, e - (p - 1))   # spacing of representable values there
    y = np.rint(x / quantum) * quantum
    if max_finite is not None:
        y = np.clip(y, -max_finite, max_finite)
    return y


def e4m3_round(x) -> np.ndarray:
    """OCP FP8 E4M3 value nearest to x (ties to even), saturating to +-448."""
    return round_binary(x, p=4, emin=-6, max_finite=E4M3_MAX)


def e4m3_decode(codes) -> np.ndarray:
    """Value of each OCP E4M3 byte: sign, 4-bit exponent (bias 7), 3-bit mantissa.

    Exponent field 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; there is
    no infinity.
    """
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    mf = c & 0x7
    mag = np.where(ef == 0, mf / 8.0 * 2.0 ** -6, (1.0 + mf / 8.0) * np.exp2(ef - 7.0))
    mag = np.where((ef == 0xF) & (mf == 0x7), np.nan, mag)
    return sign * mag


def e4m3_encode(values) -> np.ndarray:
    """Byte code of values that are already exactly representable in E4M3."""
    v = np.asarray(values, dtype=np.float64)
    sign = (np.signbit(v)).astype(np.int64) << 7
    a = np.abs(v)
    _, e = np.frexp(a)
    e = e - 1
    normal = a >= 2.0 ** -6
    ef = np.where(normal, e + 7, 0)
    mf = np.where(normal, np.rint((a / np.exp2(np.where(normal, e, 0)) - 1.0) * 8.0),
                  np.rint(a / 2.0 ** -9))
    code = sign | (ef.astype(np.int64) << 3) | mf.astype(np.int64)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------
# Quantization stages (integer / IEEE fp32 arithmetic, bit-exact by definition)
# --------------------------------------------------------------------------

def k_channel_mean(k: np.ndarray) -> np.ndarray:
    """mu[c] = fp32( (sum over tokens of k[t, c], in fp64) / n ) for k of shape (n, d)."""
    n = k.shape[0]
    s = np.sum(np.asarray(k, dtype=np.float64), axis=0)
    return (s / np.float64(n)).astype(np.float32)


def smooth_k(k: np.ndarray, mu: np.ndarray) -> np.ndarray:
    """k_s = fp32(k - mu), one IEEE fp32 subtraction per element."""
    return np.asarray(k, dtype=np.float32) - np.asarray(mu, dtype=np.float32)[None, :]


def quantize_int8_blocks(x: np.ndarray, blk: int):
    """Per-block symmetric INT8 quantization of x (n, d) in blocks of ``blk`` tokens.

    Returns (codes int8 of shape (ceil(n/blk)*blk, d) with zero padding rows,
    scales float32 of shape (ceil(n/blk),)).  Dequantized value = code * scale.
    """
    x = np.asarray(x, dtype=np.float32)
    n, d = x.shape
    nblk = -(-n // blk)
    codes = np.zeros((nblk * blk, d), dtype=np.int8)
    scales = np.zeros(nblk, dtype=np.float32)
    f127 = np.float32(127.0)
    for b in range(nblk):
        rows = x[b * blk:min(n, (b + 1) * blk)]
        a = np.max(np.abs(rows)).astype(np.float32)
        if a == 0:
            continue                        # s = 0 and all codes 0
        s = np.float32(a / f127)
        r = np.float32(f127 / a)
        y = (rows * r).astype(np.float32)   # one fp32 rounding
        codes[b * blk:b * blk + rows.shape[0]] = np.clip(np.rint(y), -127, 127).astype(np.int8)
        scales[b] = s
    return codes, scales


def quantize_v_e4m3(v: np.ndarray):
    """Per-channel FP8 E4M3 quantization of v (n, d).

    Returns (codes uint8 (n, d), sv float32 (d,)); dequantized = e4m3_decode(code) * sv.
    """
    v = np.asarray(v, dtype=np.float32)
    vmax = np.max(np.abs(v), axis=0).astype(np.float32)
    f448 = np.float32(E4M3_MAX)
    nz = vmax > 0
    safe = np.where(nz, vmax, np.float32(1.0))
    sv = np.where(nz, (safe / f448).astype(np.float32), np.float32(0.0)).astype(np.float32)
    r = np.where(nz, (f448 / safe).astype(np.float32), np.float32(0.0)).astype(np.float32)
    y = (v * r[None, :]).astype(np.float32)       # one fp32 rounding
    vals = e4m3_round(y.astype(np.float64))       # exact rounding of that fp32 value
    return e4m3_encode(vals), sv


def integer_scores(q8: np.ndarray, k8: np.ndarray) -> np.ndarray:
    """S[i, j] = sum_c q8[i, c] * k8[j, c], exact (int64 accumulation, returned as int32)."""
    s = np.asarray(q8, dtype=np.int64) @ np.asarray(k8, dtype=np.int64).T
    return s.astype(np.int32)


# --------------------------------------------------------------------------
# fp64 stages: dequantization, online softmax, two-level PV accumulation
# --------------------------------------------------------------------------

def online_softmax_pv(x_rows: np.ndarray, vvals: np.ndarray, sv: np.ndarray,
                      quantize_p: bool = True):
    """Online softmax over KV blocks of KV_TILE keys with two-level PV accumulation.

    x_rows: (r, n_kv) float64 logits, already dequantized and scaled, with masked
    entries set to -inf.  vvals: (n_kv, d) float64 V values (e4m3 values when
    quantized).  sv: (d,) per-channel V scales (ones when not quantized).
    Returns (out (r, d), lse (r,)).
    """
    r, n_kv = x_rows.shape
    d = vvals.shape[1]
    m = np.full(r, -np.inf)
    l = np.zeros(r)
    o = np.zeros((r, d))
    for t0 in range(0, n_kv, KV_TILE):
        x = x_rows[:, t0:t0 + KV_TILE]
        m_new = np.maximum(m, np.max(x, axis=1))
        # rows whose keys so far are all masked keep m = -inf: nothing to add
        live = np.isfinite(m_new)
        m_safe = np.where(live, m_new, 0.0)
        p = np.where(live[:, None], np.exp(x - m_safe[:, None]), 0.0)
        alpha = np.where(np.isfinite(m), np.exp(m - m_safe), 0.0)
        l = l * alpha + np.sum(p, axis=1)
        p8 = e4m3_round(P_SCALE * p) if quantize_p else P_SCALE * p
        pv_blk = p8 @ vvals[t0:t0 + KV_TILE]          # first level: one KV block
        o = o * alpha[:, None] + pv_blk                # second level: running output
        m = np.where(live, m_new, m)
    out = o * sv[None, :] / (P_SCALE * l[:, None])
    lse = m + np.log(l)
    return out, lse


def attention_head(q, k, v, *, causal: bool = False, sm_scale: float | None = None,
                   rows=None, quantize: bool = True, smooth: bool = True) -> dict:
    """Quantized attention for one (sequence, query head) with its KV head.

    q: (n, d), k, v: (n_kv, d), float32 holding the input values.  ``rows`` picks a
    subset of query rows (all by default); every row is computed independently.
    ``quantize=False`` replaces every quantizer by the identity (fp64 values,
    P unrounded), which reduces the method to exact softmax attention.
    """
    q = np.asarray(q, dtype=np.float32)
    k = np.asarray(k, dtype=np.float32)
    v = np.asarray(v, dtype=np.float32)
    n, d = q.shape
    n_kv = k.shape[0]
    if causal and n != n_kv:
        raise ValueError("causal attention needs equal query and key lengths")
    scale = (1.0 / math.sqrt(d)) if sm_scale is None else float(sm_scale)
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)

    mu = k_channel_mean(k) if smooth else np.zeros(d, dtype=np.float32)
    res = {"k_mean": mu}
    if quantize:
        ks = smooth_k(k, mu)
        q8, sq = quantize_int8_blocks(q, BLKQ)
        k8, sk = quantize_int8_blocks(ks, BLKK)
        v8, sv = quantize_v_e4m3(v)
        s_int = integer_scores(q8[rows], k8[:n_kv])
        row_scale = sq[rows // BLKQ].astype(np.float64)
        col_scale = sk[np.arange(n_kv) // BLKK].astype(np.float64)
        x = s_int.astype(np.float64) * row_scale[:, None] * col_scale[None, :] * scale
        vvals = e4m3_decode(v8)
        svv = sv.astype(np.float64)
        res.update(q8=q8, q_scale=sq, k8=k8, k_scale=sk, v8=v8, v_scale=sv, s_int=s_int)
    else:
        ks = np.asarray(k, dtype=np.float64) - mu.astype(np.float64)[None, :]
        x = (q[rows].astype(np.float64) @ ks.T) * scale
        vvals = v.astype(np.float64)
        svv = np.ones(d)
    if causal:
        x = np.where(np.arange(n_kv)[None, :] > rows[:, None], -np.inf, x)
    out, lse = online_softmax_pv(x, vvals, svv, quantize_p=quantize)
    res.update(out=out, lse=lse, rows=rows)
    return res


def attention_weights(q, k, *, causal=False, sm_scale=None, quantize=True, smooth=True):
    """Normalized attention weights the oracle applies (tiny inputs; for pins).

    Key j of row i weighs exp(x_ij - m_i) / l_i with the final row max m_i and
    sum l_i; with quantization on, x is the dequantized logit.
    """
    q = np.asarray(q, dtype=np.float32)
    k = np.asarray(k, dtype=np.float32)
    n, d = q.shape
    scale = (1.0 / math.sqrt(d)) if sm_scale is None else float(sm_scale)
    mu = k_channel_mean(k) if smooth else np.zeros(d, dtype=np.float32)
    if quantize:
        q8, sq = quantize_int8_blocks(q, BLKQ)
        k8, sk = quantize_int8_blocks(smooth_k(k, mu), BLKK)
        s_int = integer_scores(q8[:n], k8[:k.shape[0]]).astype(np.float64)
        x = s_int * sq[np.arange(n) // BLKQ, None] * sk[None, np.arange(k.shape[0]) // BLKK] * scale
    else:
        x = (q.astype(np.float64) @ (k.astype(np.float64) - mu.astype(np.float64)).T) * scale
    if causal:
        x = np.where(np.arange(k.shape[0])[None, :] > np.arange(n)[:, None], -np.inf, x)
    m = np.max(x, axis=1, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=1, keepdims=True)


def sage_attention(q, k, v, *, causal=False, sm_scale=None, cu_seqlens=None,
                   quantize=True, smooth=True) -> np.ndarray:
    """Whole-batch quantized attention in float64.

    Dense: q (B,Hq,N,d), k, v (B,Hkv,N,d) -> out (B,Hq,N,d).
    Varlen: q (T,Hq,d), k, v (T,Hkv,d) packed, with cu_seqlens -> out (T,Hq,d).
    """
    if cu_seqlens is None:
        B, Hq, N, d = q.shape
        g = Hq // k.shape[1]
        out = np.zeros((B, Hq, N, d))
        for b in range(B):
            for h in range(Hq):
                out[b, h] = attention_head(q[b, h], k[b, h // g], v[b, h // g], causal=causal,
                                           sm_scale=sm_scale, quantize=quantize,
                                           smooth=smooth)["out"]
        return out
    T, Hq, d = q.shape
    g = Hq // k.shape[1]
    out = np.zeros((T, Hq, d))
    for s0, s1 in zip(cu_seqlens[:-1], cu_seqlens[1:]):
        for h in range(Hq):
            out[s0:s1, h] = attention_head(q[s0:s1, h], k[s0:s1, h // g], v[s0:s1, h // g],
                                           causal=causal, sm_scale=sm_scale, quantize=quantize,
                                           smooth=smooth)["out"]
    return out


def reference_attention(q, k, v, *, causal=False, sm_scale=None) -> np.ndarray:
    """Full-precision attention softmax(q k^T * scale) v in float64 for one head (n, d)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    scale = (1.0 / math.sqrt(q.shape[1])) if sm_scale is None else float(sm_scale)
    x = (q @ k.T) * scale
    if causal:
        x = np.where(np.arange(k.shape[0])[None, :] > np.arange(q.shape[0])[:, None], -np.inf, x)
    x = x - np.max(x, axis=1, keepdims=True)
    p = np.exp(x)
    return (p @ v) / np.sum(p, axis=1, keepdims=True)
