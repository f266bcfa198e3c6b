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

Everything after the integer scores is done in float64: ``attention_head`` is
that all-fp64 definition and the reference every GPU parity check compares with.
``attention_head_fp32_logits`` is a second, diagnostic path: it forms the logits,
the running max and the exponent argument t with the fp32 operations the kernel
uses, and then takes 2^t correctly rounded to fp32 (an fp64 exp2 followed by one
rounding), so it shows how much of a difference comes from fp32 logits alone.
Neither path contains any approximation of the exponential.

Readings where the pages are silent:

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
* 16-bit PV option (vibecrowd page, How it works: "FP16/FP8 for PV"): with
  ``pv="fp16"`` or ``pv="bf16"`` V keeps its input values (no V quantization, sv = 1)
  and P~ is rounded to that 16-bit type with scale 1; the output is O / l.
* GQA: query head h reads KV head h // (Hq / Hkv).  Varlen: every packed
  sequence is an independent problem (its own mean, blocks and causal diagonal).
* Causal (equal query and key lengths): key j is masked for query i when j > i.
* "Per-thread quantization" (heatdrop review, The interesting bit) is read as a Q
  scale per token and a K scale per 32-token block (qblk = 1, kblk = 32), an option
  next to the per-block default.

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
    "PV_FORMATS", "round_pv", "p_scale",
    "LOG2E_F32", "fma_f32", "exp2_rn_f32", "kernel_scale_log2",
    "online_softmax_pv_fp32_decision", "attention_head_fp32_logits",
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


# P (and, for the 16-bit option, V) formats of the PV product
PV_FORMATS = ("e4m3", "fp16", "bf16")


def p_scale(pv: str) -> float:
    """Static scale of P~ (<= 1) before rounding: 448 fills e4m3; 16-bit types take P~ as is."""
    if pv not in PV_FORMATS:
        raise ValueError(f"pv must be one of {PV_FORMATS}, got {pv!r}")
    return P_SCALE if pv == "e4m3" else 1.0


def round_pv(x, pv: str) -> np.ndarray:
    """Round P values to the PV operand format (e4m3 satfinite, fp16 or bf16; RNE)."""
    if pv == "e4m3":
        return e4m3_round(x)
    if pv == "fp16":
        return round_binary(x, p=11, emin=-14)
    if pv == "bf16":
        return round_binary(x, p=8, emin=-126)
    raise ValueError(f"pv must be one of {PV_FORMATS}, got {pv!r}")


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
                      quantize_p: bool = True, pv: str = "e4m3"):
    """Online softmax over KV blocks of KV_TILE keys with two-level PV accumulation.

    x_rows: (r, n_kv) float64 logits, already dequantized and scaled, with masked
    entries set to -inf.  vvals: (n_kv, d) float64 V values (e4m3 values when
    quantized, the input values for a 16-bit ``pv``).  sv: (d,) per-channel V
    scales (ones when V is not quantized).  ``pv`` names the format P is rounded
    to (``round_pv``) at its static scale (``p_scale``).
    Returns (out (r, d), lse (r,)).
    """
    r, n_kv = x_rows.shape
    d = vvals.shape[1]
    ps = p_scale(pv)
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
        pq = round_pv(ps * p, pv) if quantize_p else ps * p
        pv_blk = pq @ vvals[t0:t0 + KV_TILE]           # first level: one KV block
        o = o * alpha[:, None] + pv_blk                # second level: running output
        m = np.where(live, m_new, m)
    out = o * sv[None, :] / (ps * l[:, None])
    lse = m + np.log(l)
    return out, lse


def attention_head(q, k, v, *, causal: bool = False, sm_scale: float | None = None,
                   rows=None, quantize: bool = True, smooth: bool = True,
                   qblk: int = BLKQ, kblk: int = BLKK, pv: str = "e4m3") -> dict:
    """Quantized attention for one (sequence, query head) with its KV head.

    q: (n, d), k, v: (n_kv, d), float32 holding the input values.  ``rows`` picks a
    subset of query rows (all by default); every row is computed independently.
    ``quantize=False`` replaces every quantizer by the identity (fp64 values,
    P unrounded), which reduces the method to exact softmax attention.  qblk / kblk
    are the INT8 scale blocks of Q and K in tokens (128 / 64 as the method states;
    1 / 32 for the per-thread granularity).  ``pv`` is the PV format: "e4m3" (the
    method: e4m3 P and per-channel e4m3 V) or "fp16" / "bf16" (P rounded to that
    type, V at its input values).
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
        q8, sq = quantize_int8_blocks(q, qblk)
        k8, sk = quantize_int8_blocks(ks, kblk)
        s_int = integer_scores(q8[rows], k8[:n_kv])
        row_scale = sq[rows // qblk].astype(np.float64)
        col_scale = sk[np.arange(n_kv) // kblk].astype(np.float64)
        x = s_int.astype(np.float64) * row_scale[:, None] * col_scale[None, :] * scale
        res.update(q8=q8, q_scale=sq, k8=k8, k_scale=sk, s_int=s_int)
        if pv == "e4m3":
            v8, sv = quantize_v_e4m3(v)
            vvals = e4m3_decode(v8)
            svv = sv.astype(np.float64)
            res.update(v8=v8, v_scale=sv)
        else:
            p_scale(pv)                                 # validates the format name
            vvals = v.astype(np.float64)
            svv = np.ones(d)
    else:
        ks = np.asarray(k, dtype=np.float64) - mu.astype(np.float64)[None, :]
        x = (q[rows].astype(np.float64) @ ks.T) * scale
        vvals = v.astype(np.float64)
        svv = np.ones(d)
    if causal:
        x = np.where(np.arange(n_kv)[None, :] > rows[:, None], -np.inf, x)
    out, lse = online_softmax_pv(x, vvals, svv, quantize_p=quantize, pv=pv)
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
                   quantize=True, smooth=True, qblk: int = BLKQ, kblk: int = BLKK,
                   pv: str = "e4m3") -> np.ndarray:
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
                                           smooth=smooth, qblk=qblk, kblk=kblk, pv=pv)["out"]
        return out
    T, Hq, d = q.shape
    g = Hq // k.shape[1]
    out = np.zeros((T, Hq, d))
    for s0, s1 in zip(cu_seqlens[:-1], cu_seqlens[1:]):
        for h in range(Hq):
            out[s0:s1, h] = attention_head(q[s0:s1, h], k[s0:s1, h // g], v[s0:s1, h // g],
                                           causal=causal, sm_scale=sm_scale, quantize=quantize,
                                           smooth=smooth, qblk=qblk, kblk=kblk, pv=pv)["out"]
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


# --------------------------------------------------------------------------
# fp32 logits with a correctly rounded exponential (diagnostic path)
# --------------------------------------------------------------------------
# The kernel forms the logits in fp32: u = S * ck in the log2 domain with
# ck = fp32(fp32(q_scale * k_scale) * fp32(sm_scale * log2 e)), the running max m'
# as the fp32 max over K blocks of (largest score * block factor), and the exponent
# argument t = fma(S, ck, log2(P scale) - m').  This path takes exactly those fp32
# steps and then 2^t correctly rounded to fp32; everything else (the running sum l,
# the rescale factors, PV and the output) is fp64, as in ``attention_head``.

LOG2E_F32 = np.float32(1.4426950408889634)


def fma_f32(a, b, c) -> np.ndarray:
    """fp32 fused multiply-add a*b + c with a single round-to-nearest-even.

    a*b of two fp32 values is exact in fp64; TwoSum gives the fp64 sum s and
    its exact error e; rounding s to fp32 is then correct unless s sits exactly
    on an fp32 midpoint, where the sign of e decides the direction.
    """
    a = np.asarray(a, dtype=np.float32).astype(np.float64)
    b = np.asarray(b, dtype=np.float32).astype(np.float64)
    c = np.asarray(c, dtype=np.float32).astype(np.float64)
    p = a * b
    s = p + c
    bb = s - p
    e = (p - (s - bb)) + (c - bb)
    r = s.astype(np.float32)
    r64 = r.astype(np.float64)
    up = np.nextafter(r, np.float32(np.inf))
    dn = np.nextafter(r, np.float32(-np.inf))
    # s exactly halfway between r and a neighbour: the exact sum s + e decides
    tie_up = (s > r64) & (s - r64 == (up.astype(np.float64) - r64) / 2) & (e > 0)
    tie_dn = (s < r64) & (r64 - s == (r64 - dn.astype(np.float64)) / 2) & (e < 0)
    r = np.where(tie_up, up, np.where(tie_dn, dn, r))
    return r.astype(np.float32)


def exp2_rn_f32(t) -> np.ndarray:
    """2^t for fp32 t, rounded once to fp32 (round to nearest even).

    np.exp2 in float64 is accurate to about one fp64 ulp, 2^-29 of an fp32 ulp, so
    the single rounding to fp32 is the correctly rounded result except for
    arguments whose exact power lies within that distance of an fp32 midpoint.
    """
    with np.errstate(over="ignore"):          # 2^t beyond the fp32 range rounds to inf
        return np.exp2(np.asarray(t, dtype=np.float32).astype(np.float64)).astype(np.float32)


def kernel_scale_log2(d: int, sm_scale: float | None = None) -> np.float32:
    """sm_scale * log2(e) as the kernel forms it in fp32 (default 1/sqrt(d))."""
    s = (np.float32(1.0) / np.sqrt(np.float32(d))) if sm_scale is None else np.float32(sm_scale)
    return np.float32(s * LOG2E_F32)


def online_softmax_pv_fp32_decision(s_int, sq_rows, sk_blocks, scale_log2, valid, vvals, sv,
                                    quantize_p: bool = True, kblk: int = BLKK,
                                    pv: str = "e4m3"):
    """Online softmax with fp32 logits and running max and an exact fp32 2^t.

    s_int: (r, n_kv) exact scores; sq_rows: (r,) float32 Q scales; sk_blocks:
    float32 K scales per kblk-key block; scale_log2: float32 sm_scale*log2(e);
    valid: (r, n_kv) bool key mask; vvals (n_kv, d) and sv (d,) as in
    online_softmax_pv; ``pv`` the PV format.  The running max m' is the fp32 max
    of fp32 products of each K block's largest score with that block's factor.
    Returns (out, lse).
    """
    r, n_kv = s_int.shape
    d = vvals.shape[1]
    ps = p_scale(pv)
    log2_ps = np.float32(math.log2(ps))
    per_tile = KV_TILE // kblk
    nblk = per_tile * (-(-n_kv // KV_TILE))
    skb = np.zeros(nblk, dtype=np.float32)
    skb[:len(sk_blocks)] = sk_blocks
    sq_rows = np.asarray(sq_rows, dtype=np.float32)
    m32 = np.full(r, -np.inf, dtype=np.float32)
    l = np.zeros(r)
    o = np.zeros((r, d))
    for j, t0 in enumerate(range(0, n_kv, KV_TILE)):
        cols = np.arange(t0, min(n_kv, t0 + KV_TILE))
        S = s_int[:, cols].astype(np.int64)
        ok = valid[:, cols]
        blk = (cols - t0) // kblk                                                  # K block in tile
        ck = np.stack([((sq_rows * skb[per_tile * j + h]).astype(np.float32) * scale_log2).astype(np.float32)
                       for h in range(per_tile)], axis=1)                          # (r, per_tile)
        mt = np.full(r, -np.inf, dtype=np.float32)
        for h in range(per_tile):
            sel = blk == h
            if not np.any(sel):
                continue
            Sh = np.where(ok[:, sel], S[:, sel], np.iinfo(np.int64).min)
            imax = Sh.max(axis=1)
            has = imax != np.iinfo(np.int64).min
            prod = (imax.astype(np.float32) * ck[:, h]).astype(np.float32)
            mt = np.maximum(mt, np.where(has, prod, np.float32(-np.inf)))
        m_new = np.maximum(m32, mt)
        nbias = (log2_ps - m_new).astype(np.float32)
        tt = fma_f32(S.astype(np.float32), ck[:, blk], nbias[:, None])
        p = np.where(ok, exp2_rn_f32(tt).astype(np.float64), 0.0)                   # ps * P~
        pq = round_pv(p, pv) if quantize_p else p
        alpha = np.where(np.isfinite(m32), np.exp2(m32.astype(np.float64) - m_new.astype(np.float64)), 0.0)
        l = l * alpha + np.sum(p, axis=1)
        o = o * alpha[:, None] + pq @ vvals[cols]
        m32 = m_new
    out = o * sv[None, :] / l[:, None]
    lse = m32.astype(np.float64) * math.log(2.0) + np.log(l / ps)
    return out, lse


def attention_head_fp32_logits(q, k, v, *, causal=False, sm_scale=None, rows=None,
                               quantize_p: bool = True, qblk: int = BLKQ,
                               kblk: int = BLKK, pv: str = "e4m3") -> dict:
    """attention_head with fp32 logits, fp32 running max and a correctly rounded 2^t.

    Quantization of Q, K, V and the integer scores are the same exact stages as
    attention_head; p = P scale * P~ is fp32(2^t) with t from the kernel's fp32
    logit steps, P = round_pv(p), and the row sum l (of the unrounded p), the
    rescale factors, PV and the output are fp64.
    """
    q = np.asarray(q, dtype=np.float32)
    k = np.asarray(k, dtype=np.float32)
    v = np.asarray(v, dtype=np.float32)
    n, d = q.shape
    n_kv = k.shape[0]
    if causal and n != n_kv:
        raise ValueError("causal attention needs equal query and key lengths")
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    mu = k_channel_mean(k)
    q8, sq = quantize_int8_blocks(q, qblk)
    k8, sk = quantize_int8_blocks(smooth_k(k, mu), kblk)
    s_int = integer_scores(q8[rows], k8[:n_kv])
    valid = np.ones((len(rows), n_kv), dtype=bool)
    if causal:
        valid = np.arange(n_kv)[None, :] <= rows[:, None]
    res = dict(rows=rows, k_mean=mu, q8=q8, q_scale=sq, k8=k8, k_scale=sk, s_int=s_int)
    if pv == "e4m3":
        v8, sv = quantize_v_e4m3(v)
        vvals, svv = e4m3_decode(v8), sv.astype(np.float64)
        res.update(v8=v8, v_scale=sv)
    else:
        vvals, svv = v.astype(np.float64), np.ones(d)
    out, lse = online_softmax_pv_fp32_decision(
        s_int, sq[rows // qblk], sk, kernel_scale_log2(d, sm_scale), valid, vvals, svv,
        quantize_p=quantize_p, kblk=kblk, pv=pv)
    res.update(out=out, lse=lse)
    return res
