"""Seeded synthetic workloads for the IndexMem hot path.

This module only *draws* inputs: hidden states, the frozen model's Q/K/V
projections of them, random-init weights and decode-step inputs. It holds none
of the method's arithmetic (no indexer, selection, memory or attention math),
so both the CUDA path and the CPU oracle may take their inputs from it.

Recipe (shapes follow the workload table of the hot path; values are synthetic
because the pages' suites -- RULER, Needle-in-a-Haystack, LongBench -- and the
trained weights are not available):

* hidden states X ~ N(0, 1); token 0 scaled 4x (attention sink); 1% of the
  tokens, drawn per sequence, scaled 3x (heavy hitters, 3x key norm because the
  projections are linear);
* weights ~ N(0, 1/fan_in): the frozen model's W_q, W_k, W_v, the indexer's
  W_Iq, W_Ik, w_Ig, and the memory's W_phi, w_gate;
* Q = X W_q, K = X W_k, V = X W_v, computed once here and rounded to the
  workload's dtype: they are inputs of the path, not part of it;
* decode steps draw fresh hidden states and project them the same way;
* optional "needles": keys planted with cosine 0.8 to a later decode query.

Everything is drawn from one seeded ``torch.Generator`` on the requested
device, so a given (workload, seed, device) always yields the same tensors.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class LayerShape:
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    idx_dim: int
    mem_r: int
    lam: float
    dtype: str  # "fp32" or "bf16"

    @property
    def idx_heads(self) -> int:
        # The indexer down-projects each attention query head: one indexer
        # head per query head.
        return self.n_q_heads

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    batch: int
    L: int
    budgets: Tuple[int, ...]
    n_decode: int
    seed: int
    prefill_chunk: Optional[int] = None   # query-range size for chunked prefill
    needles: int = 0
    n_layers: int = 1
    mem_chunk: int = 512

    @property
    def budget(self) -> int:
        return self.budgets[-1]


TINY = LayerShape(hidden=512, n_q_heads=8, n_kv_heads=2, head_dim=64,
                  idx_dim=32, mem_r=32, lam=0.99, dtype="fp32")
LLAMA8B = LayerShape(hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
                     idx_dim=64, mem_r=64, lam=0.995, dtype="bf16")

WORKLOADS: Dict[str, Workload] = {
    # tiny single layer, fp32
    "c0": Workload("c0", TINY, batch=1, L=1024, budgets=(128,), n_decode=16, seed=0),
    # Llama-3.1-8B-shaped layer, 90% eviction
    "c1": Workload("c1", LLAMA8B, batch=1, L=4096, budgets=(410,), n_decode=256, seed=1),
    # same layer, batch 4 at 16K context, budget sweep
    "c2": Workload("c2", LLAMA8B, batch=4, L=16384, budgets=(128, 256, 512, 1024),
                   n_decode=512, seed=2),
    # one 128K sequence, chunked prefill, planted needles
    "c3": Workload("c3", LLAMA8B, batch=1, L=131072, budgets=(13107,), n_decode=1024,
                   seed=3, prefill_chunk=8192, needles=64),
    # 36-layer decode stress (Qwen3-8B-like layer shapes)
    "c4": Workload("c4", LLAMA8B, batch=64, L=32768, budgets=(2048,), n_decode=128,
                   seed=4, n_layers=36),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(g, shape, device, std=1.0):
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std


def make_weights(shape: LayerShape, seed: int, device="cpu") -> Dict[str, torch.Tensor]:
    """Random-init weights of one layer: the frozen model's projections and the
    method's slow weights. Shapes:

    W_q [H, Hq*d], W_k / W_v [H, Hkv*d]       (frozen model, dtype)
    W_iq [Hq, d, d_I], W_ik [H, d_I], w_ig [H, Hq]   (indexer, dtype)
    W_phi [r, d], w_gate [Hq, d]                     (memory, fp32)
    """
    g = _gen(device, 1_000_003 * (seed + 1))
    H, Hq, Hkv, d = shape.hidden, shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    dI, r = shape.idx_dim, shape.mem_r
    dt = shape.torch_dtype
    w = {
        "W_q": _randn(g, (H, Hq * d), device, 1 / math.sqrt(H)).to(dt),
        "W_k": _randn(g, (H, Hkv * d), device, 1 / math.sqrt(H)).to(dt),
        "W_v": _randn(g, (H, Hkv * d), device, 1 / math.sqrt(H)).to(dt),
        "W_iq": _randn(g, (Hq, d, dI), device, 1 / math.sqrt(d)).to(dt),
        "W_ik": _randn(g, (H, dI), device, 1 / math.sqrt(H)).to(dt),
        "w_ig": _randn(g, (H, Hq), device, 1 / math.sqrt(H)).to(dt),
        "W_phi": _randn(g, (r, d), device, 1 / math.sqrt(d)),
        "w_gate": _randn(g, (Hq, d), device, 1 / math.sqrt(d)),
    }
    return {k: v.contiguous() for k, v in w.items()}


def _project(x: torch.Tensor, W: torch.Tensor, heads: int, d: int, row_block: int = 8192):
    """x [..., H] (dtype) @ W [H, heads*d] -> [..., heads, d] rounded to dtype.
    Computed in fp32 on CPU (bf16 matmul on CPU is slow), native dtype on GPU."""
    lead = x.shape[:-1]
    x2 = x.reshape(-1, x.shape[-1])
    out = torch.empty(x2.shape[0], W.shape[1], dtype=x.dtype, device=x.device)
    for i in range(0, x2.shape[0], row_block):
        xb = x2[i:i + row_block]
        if x.device.type == "cpu":
            out[i:i + row_block] = (xb.float() @ W.float()).to(x.dtype)
        else:
            out[i:i + row_block] = (xb @ W).to(x.dtype)
    return out.reshape(*lead, heads, d)


def make_hidden(shape: LayerShape, batch: int, L: int, seed: int, device="cpu") -> torch.Tensor:
    """X [b, L, H]: N(0,1), token 0 x4, 1% heavy hitters x3 (drawn per sequence)."""
    g = _gen(device, 2_000_029 * (seed + 1))
    X = torch.randn(batch, L, shape.hidden, generator=g, device=device, dtype=torch.float32)
    X[:, 0] *= 4.0
    n_heavy = max(1, L // 100)
    for bi in range(batch):
        picks = torch.randperm(L - 1, generator=g, device=device)[:n_heavy] + 1
        X[bi, picks] *= 3.0
    return X.to(shape.torch_dtype).contiguous()


def make_layer_inputs(wl: Workload, weights, seed: Optional[int] = None, device="cpu",
                      L: Optional[int] = None, batch: Optional[int] = None):
    """X [b,L,H], Q [b,L,Hq,d], K/V [b,L,Hkv,d] in the workload dtype."""
    s = wl.shape
    seed = wl.seed if seed is None else seed
    L = wl.L if L is None else L
    batch = wl.batch if batch is None else batch
    X = make_hidden(s, batch, L, seed, device)
    Q = _project(X, weights["W_q"], s.n_q_heads, s.head_dim)
    K = _project(X, weights["W_k"], s.n_kv_heads, s.head_dim)
    V = _project(X, weights["W_v"], s.n_kv_heads, s.head_dim)
    return {"X": X, "Q": Q.contiguous(), "K": K.contiguous(), "V": V.contiguous()}


def make_decode_inputs(wl: Workload, weights, n_steps: int, seed: Optional[int] = None,
                       device="cpu", batch: Optional[int] = None):
    """Per decode step: the new token's hidden state x [n,b,H] and its
    projections q [n,b,Hq,d], k_new / v_new [n,b,Hkv,d] (workload dtype)."""
    s = wl.shape
    seed = wl.seed if seed is None else seed
    batch = wl.batch if batch is None else batch
    g = _gen(device, 3_000_017 * (seed + 1))
    x = torch.randn(n_steps, batch, s.hidden, generator=g, device=device,
                    dtype=torch.float32).to(s.torch_dtype)
    q = _project(x, weights["W_q"], s.n_q_heads, s.head_dim)
    k = _project(x, weights["W_k"], s.n_kv_heads, s.head_dim)
    v = _project(x, weights["W_v"], s.n_kv_heads, s.head_dim)
    return {"x": x.contiguous(), "q": q.contiguous(), "k_new": k.contiguous(),
            "v_new": v.contiguous()}


def plant_needles(wl: Workload, K: torch.Tensor, q_dec: torch.Tensor, n_needles: int,
                  seed: Optional[int] = None, cosine: float = 0.8):
    """Plant keys that align with later decode queries (in place on K).

    For each needle position p (uniform in [0, L)) a decode step is drawn; for
    every KV head the key at p keeps its norm but takes the direction
    cosine*q_dir + sqrt(1-cosine^2)*u, where q_dir is the unit query of the
    group's first query head at that step and u a random unit vector
    orthogonal to it. Returns the positions (sorted) and their decode steps.
    """
    s = wl.shape
    seed = wl.seed if seed is None else seed
    dev = K.device
    g = _gen(dev, 4_000_037 * (seed + 1))
    b, L = K.shape[0], K.shape[1]
    group = s.n_q_heads // s.n_kv_heads
    pos = torch.randint(0, L, (n_needles,), generator=g, device=dev)
    steps = torch.randint(0, q_dec.shape[0], (n_needles,), generator=g, device=dev)
    sin = math.sqrt(1.0 - cosine * cosine)
    for i in range(n_needles):
        p, st = int(pos[i]), int(steps[i])
        for bi in range(b):
            for kv in range(s.n_kv_heads):
                qd = q_dec[st, bi, kv * group].float()
                qd = qd / qd.norm()
                u = torch.randn(s.head_dim, generator=g, device=dev)
                u = u - (u @ qd) * qd
                u = u / u.norm()
                kn = K[bi, p, kv].float().norm()
                K[bi, p, kv] = (kn * (cosine * qd + sin * u)).to(K.dtype)
    order = torch.argsort(pos)
    return pos[order], steps[order]


def make_index_subset(batch: int, L: int, n: int, seed: int, device="cpu") -> torch.Tensor:
    """Per sequence, n distinct positions of [0, L) drawn uniformly, ascending
    (int32 [batch, n]) -- a synthetic evicted set."""
    g = _gen(device, 5_000_011 * (seed + 1))
    rows = []
    for _ in range(batch):
        p = torch.randperm(L, generator=g, device=device)[:n]
        rows.append(torch.sort(p).values)
    return torch.stack(rows).to(torch.int32).contiguous()


def make_memory_state(shape: LayerShape, batch: int, seed: int, device="cpu"):
    """A synthetic memory state: M [b,Hkv,r,d] and b [b,Hkv,r], fp32, N(0,1)."""
    g = _gen(device, 6_000_023 * (seed + 1))
    M = torch.randn(batch, shape.n_kv_heads, shape.mem_r, shape.head_dim, generator=g,
                    device=device, dtype=torch.float32)
    b = torch.randn(batch, shape.n_kv_heads, shape.mem_r, generator=g, device=device,
                    dtype=torch.float32)
    return M.contiguous(), b.contiguous()
