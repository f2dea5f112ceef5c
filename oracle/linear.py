"""fp64 definitions of the QLoRA linear layer forward and backward.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Row-vector convention: W is [N, K] (out x in), X [M, K], A [K, r], B [r, N],
s = alpha / r.  "QLoRA" (ozercemkelahmet.com), How it works, Step 5 writes the
column form y = dequant(W) x + (alpha/r) B (A x); for token rows x^T this is
Y = X deq(W)^T + s (X A') B' with A' = A, B' = B in [K, r] / [r, N] layout.
Step 6: gradients flow through the dequantized weights into the adapters only;
no gradient for W.
"""
from __future__ import annotations

import numpy as np

from .nf4 import bf16_to_f32, f64_to_bf16_rn


def as_f64(bits_or_f) -> np.ndarray:
    a = np.asarray(bits_or_f)
    if a.dtype == np.uint16:
        return bf16_to_f32(a).astype(np.float64).reshape(a.shape)
    return a.astype(np.float64)


def forward(X, Wd, A, B, s: float):
    """XA = X A;  Y = X Wd^T + s XA B.  All fp64; inputs may be bf16 bits."""
    X, Wd, A, B = (as_f64(t) for t in (X, Wd, A, B))
    XA = X @ A
    Y = X @ Wd.T + s * (XA @ B)
    return Y, XA


def backward(dY, X, Wd, A, B, s: float, XA=None):
    """G = dY B^T;  dX = dY Wd + s G A^T;  dA = s X^T G;  dB = s XA^T dY."""
    dY, X, Wd, A, B = (as_f64(t) for t in (dY, X, Wd, A, B))
    if XA is None:
        XA = X @ A
    else:
        XA = np.asarray(XA, np.float64)
    G = dY @ B.T
    dX = dY @ Wd + s * (G @ A.T)
    dA = s * (X.T @ G)
    dB = s * (XA.T @ dY)
    return dict(G=G, dX=dX, dA=dA, dB=dB)


def lora_products(dY, X, A, B, s: float):
    """The rank-r quantities that need no W: XA = X A, G = dY B^T,
    dA = s X^T G, dB = s XA^T dY (fp64)."""
    dY, X, A, B = (as_f64(t) for t in (dY, X, A, B))
    XA = X @ A
    G = dY @ B.T
    return dict(XA=XA, G=G, dA=s * (X.T @ G), dB=s * (XA.T @ dY))


def forward_rows(X, Wd, A, B, s: float, rows):
    """Y restricted to the given token rows (for sampled checks at full size)."""
    rows = np.asarray(rows)
    Y, XA = forward(as_f64(X)[rows], Wd, A, B, s)
    return Y, XA


def backward_rows_dx(dY, Wd, A, B, s: float, rows):
    """dX restricted to the given token rows."""
    dY = as_f64(dY)[np.asarray(rows)]
    Wd, A, B = (as_f64(t) for t in (Wd, A, B))
    G = dY @ B.T
    return dY @ Wd + s * (G @ A.T)


def merge_weight(W_base, A, B, s: float) -> np.ndarray:
    """The adapter folded into a 16-bit weight for serving ("QLoRA",
    ozercemkelahmet.com, How it works, Step 8 and section "Merging after QLoRA";
    its FAQ on merging): W_merged = W_base + s (A B)^T, stored in bf16.

    W_base [N, K] is the 16-bit original or the dequantized NF4 weight (the
    pages prefer the original and allow the dequantized copy), as bf16 bits;
    A [K, r], B [r, N] bf16 bits.  The sum is exact in fp64 up to its own
    rounding and is rounded once to bf16 (nearest, ties to even).  With this,
    Y = X W_merged^T equals the adapted forward up to that rounding.
    Returns bf16 bits [N, K].
    """
    Wb, A, B = (as_f64(t) for t in (W_base, A, B))
    return f64_to_bf16_rn(Wb + s * (A @ B).T)


def dropout_input(X, keep, p: float) -> np.ndarray:
    """Inverted dropout of the adapter input: X * keep / (1 - p), fp64.  `keep` is
    the 0/1 mask (drawn by the caller, Bernoulli(1 - p) per element); the frozen
    path still sees the undropped X."""
    return as_f64(X) * (np.asarray(keep, np.float64) / (1.0 - p))


def forward_dropout(X, Wd, A, B, s: float, keep, p: float):
    """Y = X Wd^T + s (drop(X) A) B with drop the inverted dropout above: the
    adapter input dropout of a LoRA configuration ("QLoRA", ozercemkelahmet.com,
    "A code example with common libraries", lora_dropout)."""
    Xd = dropout_input(X, keep, p)
    XA = Xd @ as_f64(A)
    Y = as_f64(X) @ as_f64(Wd).T + s * (XA @ as_f64(B))
    return Y, XA


def backward_dropout(dY, X, Wd, A, B, s: float, keep, p: float, XA=None):
    """Gradients of forward_dropout for a fixed mask: G = dY B^T;
    dX = dY Wd + s (G A^T) * keep / (1 - p);  dA = s drop(X)^T G;
    dB = s XA^T dY with XA = drop(X) A."""
    dY, Wd, A, B = (as_f64(t) for t in (dY, Wd, A, B))
    Xd = dropout_input(X, keep, p)
    XA = Xd @ A if XA is None else np.asarray(XA, np.float64)
    G = dY @ B.T
    dX = dY @ Wd + s * (G @ A.T) * (np.asarray(keep, np.float64) / (1.0 - p))
    return dict(G=G, dX=dX, dA=s * (Xd.T @ G), dB=s * (XA.T @ dY))


def accumulate_grads(acc: dict | None, grads: dict) -> dict:
    """Gradient accumulation over micro-batches ("QLoRA", ozercemkelahmet.com,
    "Training arguments", gradient_accumulation_steps; "Reading the memory
    profile": smaller micro-batches with more accumulation steps keep the
    effective batch): dA and dB are summed over the micro-batches before the
    optimizer step."""
    if acc is None:
        return {k: np.array(grads[k], np.float64) for k in ("dA", "dB")}
    return {k: acc[k] + grads[k] for k in ("dA", "dB")}


def rel_fro(got, ref) -> float:
    """||got - ref||_F / ||ref||_F."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))
