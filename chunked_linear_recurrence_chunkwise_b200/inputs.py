"""Seeded synthetic inputs for the chunkwise linear-recurrence layer.

This module draws random tensors and nothing else: it holds none of the
layer's arithmetic, so the CUDA path and the fp64 oracle can both consume its
output without sharing any code of the method.

The pages measure on trained models and The Pile ("Sequence Accumulation and
Beyond", Experimental setup); none of that is needed here because the cost of
the layer depends only on shapes.  The workloads below stand in for those runs
with seeded Gaussian draws of the stated shapes and value distributions.

Recipe (every workload):
  * One ``numpy`` PCG64 stream per (tensor, block of 4096 tokens), seeded by
    ``SeedSequence([seed, tensor_id, block])``, so any token range can be
    regenerated on its own and the full tensor is the concatenation.
  * Tensors, in this order of ``tensor_id``: q, k, v, gate source, beta source,
    dO.  Each is drawn in float32 C order over ``[B, block, H, d]`` (``[B,
    block, H]`` for the gate/beta sources).
  * Transforms of the draws that define the input distribution (not the
    method): L2 normalisation of each (token, head) vector, logsigmoid /
    softplus / sigmoid of the gate and beta sources.
  * bf16 workloads round q, k, v and dO to bf16 (round to nearest even); the
    float32 arrays returned here hold exactly those bf16 values, so the oracle
    sees the same numbers as the kernels.  g and beta stay float32.
  * The nonuniform cut draws ``p ~ Dirichlet(1_n)`` from
    ``SeedSequence([seed, 99])`` and gives sub-sequence i
    ``64 * (1 + floor((T/64 - n) p_i))`` tokens; leftover 64-token units go to
    the largest fractional parts (ties to the lower index).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

BLOCK = 4096


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    variant: str          # "la" (linear attention), "gla" (scalar-gated LA), "gdn" (gated delta rule)
    B: int
    T: int
    H: int
    d: int
    dtype: str            # "f32" or "bf16" (I/O dtype of q, k, v, o and the gradients)
    n_sub: int
    cut: str              # "uniform" or "dirichlet"
    backward: bool
    seed: int
    q_norm: bool          # q L2-normalised per (token, head)
    k_norm: bool
    chunk: int = 64

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def has_g(self) -> bool:
        return self.variant in ("gla", "gdn")

    @property
    def has_beta(self) -> bool:
        return self.variant == "gdn"


WORKLOADS = {
    w.name: w
    for w in [
        Workload("linear_attention_fp32_h2_t1k", "la", 1, 1024, 2, 64, "f32", 4, "uniform",
                 False, 0, False, True),
        Workload("gated_linear_attention_bf16_b2_h16_t32k", "gla", 2, 32768, 16, 128, "bf16", 8,
                 "uniform", True, 1, False, True),
        Workload("gated_deltanet_bf16_h32_t64k", "gdn", 1, 65536, 32, 128, "bf16", 16, "uniform",
                 True, 2, True, True),
        Workload("gated_deltanet_bf16_h16_t256k_dirichlet12", "gdn", 1, 262144, 16, 128, "bf16",
                 12, "dirichlet", True, 3, True, True),
        Workload("gated_deltanet_bf16_h64_t256k", "gdn", 1, 262144, 64, 128, "bf16", 16, "uniform",
                 True, 4, True, True),
    ]
}

# The workload the throughput metric is quoted on.
BENCH_WORKLOAD = "gated_deltanet_bf16_h32_t64k"

_TENSOR_ID = {"q": 0, "k": 1, "v": 2, "gate": 3, "beta": 4, "dO": 5}


def _rng(seed: int, tid: int, block: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, tid, block]))


def _to_bf16_values(a: np.ndarray) -> np.ndarray:
    import torch  # plumbing only: RNE rounding to bf16

    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(torch.float32).numpy()


def _l2n(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / n).astype(np.float32)


def _draw(w: Workload, name: str, t0: int, t1: int, heads=None) -> np.ndarray:
    """Draw tensor ``name`` for tokens [t0, t1) (and optionally a head subset)."""
    tid = _TENSOR_ID[name]
    per_tok = name in ("gate", "beta")
    parts = []
    b0 = t0 // BLOCK
    b1 = (t1 + BLOCK - 1) // BLOCK
    for blk in range(b0, b1):
        bs = blk * BLOCK
        be = min(bs + BLOCK, w.T)
        L = be - bs
        shape = (w.B, L, w.H) if per_tok else (w.B, L, w.H, w.d)
        x = _rng(w.seed, tid, blk).standard_normal(shape, dtype=np.float32)
        lo = max(t0, bs) - bs
        hi = min(t1, be) - bs
        x = x[:, lo:hi]
        if heads is not None:
            x = x[:, :, heads]
        parts.append(x)
    if not parts:
        shape = (w.B, 0, w.H if heads is None else len(heads)) + (() if per_tok else (w.d,))
        return np.zeros(shape, np.float32)
    return np.ascontiguousarray(np.concatenate(parts, axis=1))


def generate(w: Workload, t0: int = 0, t1: int | None = None, heads=None,
             with_grad: bool | None = None) -> dict:
    """Inputs of workload ``w`` for tokens [t0, t1) as float32 numpy arrays.

    Keys: q, k, v, g (None unless gated), beta (None unless delta rule), dO
    (None for forward-only workloads unless ``with_grad``).  ``heads`` selects
    a subset of heads (the draw is the same as for the full tensor).
    """
    if t1 is None:
        t1 = w.T
    bf16 = w.dtype == "bf16"
    out = {}
    q = _draw(w, "q", t0, t1, heads)
    k = _draw(w, "k", t0, t1, heads)
    v = _draw(w, "v", t0, t1, heads)
    if w.q_norm:
        q = _l2n(q)
    if w.k_norm:
        k = _l2n(k)
    out["q"], out["k"], out["v"] = q, k, v
    out["g"] = None
    out["beta"] = None
    if w.variant == "gla":
        x = _draw(w, "gate", t0, t1, heads).astype(np.float64)
        out["g"] = (-np.logaddexp(0.0, -(x + 2.0))).astype(np.float32)  # logsigmoid(N(2,1))
    elif w.variant == "gdn":
        x = _draw(w, "gate", t0, t1, heads).astype(np.float64)
        out["g"] = (-0.1 * np.logaddexp(0.0, x)).astype(np.float32)      # -0.1 softplus(N(0,1))
        y = _draw(w, "beta", t0, t1, heads).astype(np.float64)
        out["beta"] = (1.0 / (1.0 + np.exp(-y))).astype(np.float32)      # sigmoid(N(0,1))
    grad = w.backward if with_grad is None else with_grad
    out["dO"] = _draw(w, "dO", t0, t1, heads) if grad else None
    if bf16:
        for key in ("q", "k", "v", "dO"):
            if out[key] is not None:
                out[key] = _to_bf16_values(out[key])
    return out


def sub_lengths(w: Workload) -> list:
    """Sub-sequence lengths of workload ``w`` (sum = T)."""
    if w.cut == "uniform":
        base = w.T // w.n_sub
        lens = [base] * w.n_sub
        lens[-1] += w.T - base * w.n_sub
        return lens
    units = w.T // 64
    n = w.n_sub
    p = np.random.default_rng(np.random.SeedSequence([w.seed, 99])).dirichlet(np.ones(n))
    share = (units - n) * p
    base = np.floor(share).astype(np.int64)
    left = (units - n) - int(base.sum())
    frac = share - base
    order = sorted(range(n), key=lambda i: (-frac[i], i))
    for i in order[:left]:
        base[i] += 1
    lens = [int(64 * (1 + b)) for b in base]
    lens[-1] += w.T - 64 * units  # T not a multiple of 64: the tail goes to the last piece
    assert sum(lens) == w.T and min(lens) >= 1
    return lens


def random_state(w: Workload, seed_tag: int, scale: float = 0.1, B=None, H=None) -> np.ndarray:
    """N(0, scale^2) boundary state [B, H, d, d] for tests that want a nonzero S_in/dS_out."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    r = np.random.default_rng(np.random.SeedSequence([w.seed, 1000 + seed_tag]))
    return (scale * r.standard_normal((B, H, w.d, w.d))).astype(np.float32)


def n_chunks(T: int, chunk: int = 64) -> int:
    return math.ceil(T / chunk)


def iter_blocks(w: Workload, heads=None, with_grad: bool | None = None, threads: int | None = None):
    """Yields ``(t0, t1, arrays)`` for consecutive 4096-token blocks of workload ``w``.

    Blocks are drawn in a thread pool (numpy releases the GIL while drawing)
    and yielded in order; concatenating them gives ``generate(w)``.
    """
    import os
    from concurrent.futures import ThreadPoolExecutor

    nblk = (w.T + BLOCK - 1) // BLOCK
    threads = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        futs = {}
        ahead = 2 * threads

        def submit(i):
            t0, t1 = i * BLOCK, min(w.T, (i + 1) * BLOCK)
            futs[i] = ex.submit(generate, w, t0, t1, heads, with_grad)

        for i in range(min(nblk, ahead)):
            submit(i)
        for i in range(nblk):
            arrays = futs.pop(i).result()
            if i + ahead < nblk:
                submit(i + ahead)
            yield i * BLOCK, min(w.T, (i + 1) * BLOCK), arrays


def to_torch(w: Workload, device="cpu", heads=None, with_grad: bool | None = None, pin=False,
             keep_heads=None):
    """Workload inputs as torch tensors (q, k, v, dO in the workload dtype; g, beta float32).

    Filled block by block, so the host never holds more than a few blocks in
    float32.  ``pin`` allocates page-locked host memory (``device='cpu'``).
    ``keep_heads`` (list of (b, h)) also returns, under key "kept", a list of
    float32 numpy dicts with the full sequence of those (batch, head) pairs,
    taken from the same draw (single-head arrays shaped [1, T, 1, ...]).
    """
    import torch

    H = w.H if heads is None else len(heads)
    io = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    grad = w.backward if with_grad is None else with_grad
    shapes = {"q": (w.B, w.T, H, w.d), "k": (w.B, w.T, H, w.d), "v": (w.B, w.T, H, w.d)}
    if w.has_g:
        shapes["g"] = (w.B, w.T, H)
    if w.has_beta:
        shapes["beta"] = (w.B, w.T, H)
    if grad:
        shapes["dO"] = (w.B, w.T, H, w.d)
    out = {}
    for key, shp in shapes.items():
        dt = torch.float32 if key in ("g", "beta") else io
        if pin:
            out[key] = torch.empty(shp, dtype=dt, pin_memory=True)
        else:
            out[key] = torch.empty(shp, dtype=dt, device=device)
    kept = None if keep_heads is None else [{key: [] for key in shapes} for _ in keep_heads]
    for t0, t1, arr in iter_blocks(w, heads, grad):
        for key in shapes:
            src = torch.from_numpy(arr[key])
            out[key][:, t0:t1].copy_(src.to(out[key].dtype))
            if kept is not None:
                for i, (b, h) in enumerate(keep_heads):
                    kept[i][key].append(arr[key][b:b + 1, :, h:h + 1].copy())
    for key in ("g", "beta", "dO"):
        out.setdefault(key, None)
    if kept is not None:
        out["kept"] = []
        for d in kept:
            full = {key: np.concatenate(parts, axis=1) for key, parts in d.items()}
            for key in ("g", "beta", "dO"):
                full.setdefault(key, None)
            out["kept"].append(full)
    return out
