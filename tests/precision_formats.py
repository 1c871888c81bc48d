"""Oracle-side precision experiment: which low-precision operand formats keep the
sparse attention within the parity tolerance?

The tensor cores offer block-scaled FP4 products (kind::mxf4nvf4: both operands
E2M1 with an E4M3 scale per 16 elements along K) and FP8 products.  The main KV
is already NVFP4-like (E2M1 + E4M3 per 16 channels, agentnet.co.il, "דיפסיק
משיקה את V4.1-פלאש ...", section "קוונטיזציה ופריסה: FP4 ו-DRAM במקום SSD"),
so Q.K^T could run block-scaled if the query were quantised too; P.V cannot
(the value scales vary along the output channels, not along K = rows).  This
module reruns the oracle's attention with the query or the softmax weights
rounded to such formats and measures the output error against the
exact-softmax fp64 output, under the parity bound max|d| <= 1e-2 max|o| + 1e-3.

Variants (each ends with the bf16 rounding of the output, as a kernel would):
  exact      fp64 weights
  p_f16      weights rounded to f16 (the attention kernel's P and denominator)
  p_bf16     weights rounded to bf16
  p_fp8      weights scaled by 448 and rounded to E4M3
  q_fp8      query rounded to E4M3 with one fp32 scale per head (amax / 448)
  q_nvfp4    query rounded with the cache's own codec (E2M1 + E4M3 per 16)
  q_nvfp4_g  the same after dividing by a per-head fp32 scale amax / (6 x 448)
  q_fp8_p_fp8  both roundings together

Run as a script to print the table for the 64K decode sample:
    python -m tests.precision_formats
"""
from __future__ import annotations

import numpy as np

from oracle import attention as oattn
from oracle import codec as ocodec
from oracle import formats as ofmt
from oracle import idxk_fp8 as ofp8
from oracle import indexer as oidx

E4M3_MAX = 448.0


def _bf16_round(x: np.ndarray) -> np.ndarray:
    return ofmt.bf16_to_f64(ofmt.f32_to_bf16(np.asarray(x, dtype=np.float32)))


def _f16_round(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float16).astype(np.float64)


def _e4m3_round(x: np.ndarray) -> np.ndarray:
    return ofmt.E4M3_VALUES[ofp8.e4m3_code(np.asarray(x, dtype=np.float32)).astype(np.int64)]


def q_fp8(q: np.ndarray) -> np.ndarray:
    """E4M3 codes with one fp32 scale per head (amax / 448)."""
    s = (np.abs(q).max(axis=1, keepdims=True) / E4M3_MAX).astype(np.float32).astype(np.float64)
    s = np.where(s == 0, 1.0, s)
    return _e4m3_round(q / s) * s


def q_nvfp4(q: np.ndarray, global_scale: bool) -> np.ndarray:
    """E2M1 codes with an E4M3 scale per 16 channels (the cache's codec), with or
    without a per-head fp32 scale that maps the head's amax to 6 x 448."""
    g = np.ones((q.shape[0], 1))
    if global_scale:
        g = np.abs(q).max(axis=1, keepdims=True) / (6.0 * E4M3_MAX)
        g = np.where(g == 0, 1.0, g)
    codes, scales = ocodec.quantize_rows(q / g)
    return ocodec.dequantize(codes, scales) * g


def attend_variant(q: np.ndarray, rows: np.ndarray, p_round=None) -> np.ndarray:
    """Softmax attention of q [H,512] (fp64 values) over rows [T,512]; the
    weights exp(s - max) may be rounded (the denominator sums the rounded
    weights); the output is rounded to bf16."""
    s = q @ rows.T
    p = np.exp(s - s.max(axis=1, keepdims=True))
    if p_round is not None:
        p = p_round(p)
    o = (p @ rows) / p.sum(axis=1, keepdims=True)
    return _bf16_round(o)


VARIANTS = {
    "exact": (lambda q: q, None),
    "p_f16": (lambda q: q, lambda p: _f16_round(p * 4096.0) / 4096.0),
    "p_bf16": (lambda q: q, _bf16_round),
    "p_fp8": (lambda q: q, lambda p: _e4m3_round(p * E4M3_MAX) / E4M3_MAX),
    "q_fp8": (q_fp8, None),
    "q_nvfp4": (lambda q: q_nvfp4(q, False), None),
    "q_nvfp4_g": (lambda q: q_nvfp4(q, True), None),
    "q_fp8_p_fp8": (q_fp8, lambda p: _e4m3_round(p * E4M3_MAX) / E4M3_MAX),
}


def error_ratios(q_bits: np.ndarray, rows: np.ndarray) -> dict[str, float]:
    """max|variant - exact| / (1e-2 max|exact| + 1e-3) per variant (exact: the
    fp64 oracle output, not rounded)."""
    ref = oattn.attend(q_bits, rows)
    bound = 1e-2 * float(np.abs(ref).max()) + 1e-3
    q = ofmt.bf16_to_f64(q_bits)
    out = {}
    for name, (qf, pf) in VARIANTS.items():
        got = attend_variant(qf(q), rows, pf)
        out[name] = float(np.abs(got - ref).max()) / bound
    return out


def decode_sample(seqs=(0, 1, 2, 3), layers=(0, 1), length: int | None = None):
    """(q bits [H,512], attended rows [T,512]) of the 64K decode workload: the
    Full layer's index set of each sampled sequence, queries of the given
    layers (a Reuse layer attends over the same rows with its own query)."""
    import workload as wl
    w = wl.workload(1)
    L = length or w.lengths[0]
    for s in seqs:
        keys = wl.idxk_rows(w.seed, s, 0, L)
        _, idx, _ = oidx.full_indexer(wl.idxq_rows(w.seed, 0, s), keys, L)
        pos = oattn.attended_positions(idx, L)
        c, sc = ocodec.unpack_rows(ocodec.encode_bf16_rows(wl.kv_rows(w.seed, s, 0, L)[pos]))
        rows = ocodec.dequantize(c, sc)
        for layer in layers:
            yield wl.q_rows(w.seed, layer, s, w.heads), rows


def table(sample) -> dict[str, float]:
    """Worst error ratio of each variant over a sample."""
    worst: dict[str, float] = {}
    for q_bits, rows in sample:
        for k, v in error_ratios(q_bits, rows).items():
            worst[k] = max(worst.get(k, 0.0), v)
    return worst


if __name__ == "__main__":
    for k, v in table(decode_sample()).items():
        print(f"{k:12s} worst error / bound = {v:.3f}  {'pass' if v <= 1 else 'FAIL'}")
