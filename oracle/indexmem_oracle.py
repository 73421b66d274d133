"""CPU oracle for the IndexMem hot path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct NumPy float64 restatement of what the path
computes. Only the test-suite, the package's ``smoke()`` check and the
benchmark's CPU-baseline leg may import it; the product path never does, and
the CUDA library shares no code with it.

Sources, cited by page title and section:

* [IM-sum]  "IndexMem: learned KV-cache eviction with latent memory",
            technical summary (gist.science; Japanese and Italian versions
            share the section numbering): §1 Problem, §2.A Learnable indexer,
            §2.B Latent memory, §4 Experimental results.
* [IM-abs]  "IndexMem: Learned KV-Cache Eviction with Latent Memory for
            Long-Context LLM Inference", arXiv abstract.

The pages give the structure but not every formula. Where they are silent the
oracle takes the plainest reading (RMS QK-norm with eps 1e-6 and no scale;
per-query sigmoid head gate from the hidden state; causal running max with the
diagonal; ties to the lower position; phi(k) = W_phi k shared by keys and
queries; readout denominator b.phi(q) + 1e-6; scale 1/sqrt(d)).

Parity status: every function below is pinned by a not-gpu test against a
closed form, a library routine, a hand-worked example or brute force (see
tests/test_oracle_*.py). The end-to-end tie to the pages' accuracy claims is
parity unpinned: the pages print no worked example and no reference outputs.

Everything is float64; inputs are upcast from whatever dtype the CUDA path
consumed (the same rounded values).
"""

from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

RMS_EPS = 1e-6       # QK-norm epsilon
READOUT_EPS = 1e-6   # memory readout epsilon


def f64(a) -> np.ndarray:
    """Upcast a numpy array or a CPU torch tensor (any float dtype) to float64."""
    if hasattr(a, "detach"):
        a = a.detach().float().cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


# ---------------------------------------------------------------------------
# Indexer  ([IM-sum] §2.A "Architecture": MQA-style module, queries projected
# to a low dimension, one shared key derived from the hidden state, QK-norm,
# learnable head gating)
# ---------------------------------------------------------------------------

def rms_normalize(x: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """QK-norm: x / sqrt(mean(x^2) + eps) over the last axis, no scale."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def indexer_features(X, Q, W_iq, W_ik, w_ig):
    """Indexer query, key and head gate.

    X [b,L,H], Q [b,L,Hq,d], W_iq [Hq,d,dI], W_ik [H,dI], w_ig [H,Hq] ->
      qhat [b,L,Hq,dI]  RMS-normalised per-head down-projected queries
      khat [b,L,dI]     RMS-normalised shared key
      gate [b,L,Hq]     sigmoid head gate of each query token
    """
    X, Q, W_iq, W_ik, w_ig = map(f64, (X, Q, W_iq, W_ik, w_ig))
    # per head h: qI[b, l, h, :] = Q[b, l, h, :] @ W_iq[h]  (batched matmul over heads)
    qI = np.matmul(Q.transpose(0, 2, 1, 3), W_iq[None]).transpose(0, 2, 1, 3)
    kI = X @ W_ik
    gate = sigmoid(X @ w_ig)
    return rms_normalize(qI), rms_normalize(kI), gate


def score_block(qhat_s, gate_s, khat_t, d_idx: int) -> np.ndarray:
    """A[s,t] for a set of queries s and keys t of one sequence ([IM-sum] §2.A
    "Function": a dense query-to-key score matrix, A[s,t] = importance of key t
    for query s). Computed per head, then gated and summed over heads:

      A[s,t] = sum_h gate[s,h] * (qhat[s,h] . khat[t]) / sqrt(dI)

    qhat_s [S,Hq,dI], gate_s [S,Hq], khat_t [T,dI] -> A [S,T].
    """
    S, Hq, dI = qhat_s.shape
    per_head = (qhat_s.reshape(S * Hq, dI) @ khat_t.T).reshape(S, Hq, -1)  # [S,Hq,T]
    return np.einsum("sh,sht->st", gate_s, per_head) / math.sqrt(d_idx)


def pooled_importance(qhat, khat, gate, q_begin: int = 0, q_end: Optional[int] = None,
                      prev: Optional[np.ndarray] = None, keys: Optional[np.ndarray] = None,
                      key_block: int = 128) -> np.ndarray:
    """Per-key importance pooled by a running max over the causal queries
    ([IM-sum] §2.A "Training": pooled per-key importance, aggregated by a running
    maximum computed in a streaming way so the L x L matrix is never formed).

      I[t] = max( prev[t], max_{s in [max(t, q_begin), q_end)} A[s,t] )

    prev = -inf for keys first seen in this query range (t >= q_begin), and for
    every key when ``prev`` is None. Keys t >= q_end have no query yet and keep
    prev. ``keys`` restricts the evaluation to a subset (returned in that order).
    qhat [b,L,Hq,dI], khat [b,L,dI], gate [b,L,Hq] -> I [b, L or len(keys)].
    """
    b, L = khat.shape[:2]
    dI = khat.shape[-1]
    q_end = L if q_end is None else q_end
    keys = np.arange(L) if keys is None else np.asarray(keys)
    out = np.full((b, len(keys)), -np.inf)
    if prev is not None:
        prev = f64(prev)
        old = keys < q_begin
        out[:, old] = prev[:, keys[old]]
    for bi in range(b):
        for j0 in range(0, len(keys), key_block):
            ks = keys[j0:j0 + key_block]
            ks = ks[ks < q_end]
            if len(ks) == 0:
                continue
            s0 = max(int(ks.min()), q_begin)
            A = score_block(qhat[bi, s0:q_end], gate[bi, s0:q_end], khat[bi, ks], dI)
            s_idx = np.arange(s0, q_end)[:, None]
            A = np.where(s_idx >= np.maximum(ks[None, :], q_begin), A, -np.inf)
            col = j0 + np.nonzero(keys[j0:j0 + key_block] < q_end)[0]
            out[bi, col] = np.maximum(out[bi, col], A.max(axis=0))
    return out


# ---------------------------------------------------------------------------
# Top-B retention  ([IM-sum] §1 "token eviction": keep the important tokens,
# discard the rest within a bounded budget; §4: 90% eviction)
# ---------------------------------------------------------------------------

def select_budget(I, B: int) -> Tuple[np.ndarray, np.ndarray]:
    """R = the B largest I (ties -> lower position, -0 == +0), E = the rest.
    Both returned in ascending position order. I [b,L] -> R [b,B], E [b,L-B]."""
    I = np.asarray(I)
    b, L = I.shape
    if not (0 <= B <= L):
        raise ValueError("budget out of range")
    R = np.empty((b, B), dtype=np.int64)
    E = np.empty((b, L - B), dtype=np.int64)
    for bi in range(b):
        score = I[bi].astype(np.float64) + 0.0   # + 0.0 maps -0 to +0
        if np.isnan(score).any():
            raise ValueError("NaN importance")
        order = np.lexsort((np.arange(L), -score))   # by -score, then position
        R[bi] = np.sort(order[:B])
        E[bi] = np.sort(order[B:])
    return R, E


def compact(K, V, R, cap: Optional[int] = None):
    """Retained cache: K_R[j] = K[R[j]], V_R[j] = V[R[j]] for all KV heads,
    in a buffer of ``cap`` rows (rows >= B left zero for decode appends).
    K, V [b,L,Hkv,d] -> K_R, V_R [b,cap,Hkv,d] (same dtype as the input)."""
    K, V = np.asarray(K), np.asarray(V)
    b, B = R.shape
    cap = B if cap is None else cap
    KR = np.zeros((b, cap) + K.shape[2:], dtype=K.dtype)
    VR = np.zeros_like(KR)
    for bi in range(b):
        KR[bi, :B] = K[bi, R[bi]]
        VR[bi, :B] = V[bi, R[bi]]
    return KR, VR


# ---------------------------------------------------------------------------
# Latent memory  ([IM-sum] §2.B "Mechanism": evicted tokens update online a
# fixed-size state matrix M and a stabiliser vector b by an outer-product
# accumulation with decay; a projection layer and gate read it)
# ---------------------------------------------------------------------------

def memory_update(K, V, E, W_phi, lam: float, M0=None, b0=None):
    """Sequential fast-weight update over the evicted tokens, in ascending
    position order, separately for every KV head:

      phi = W_phi k ;  M <- lam * M + phi v^T ;  b <- lam * b + phi

    K, V [b,L,Hkv,d]; E [b,n] evicted positions (ascending); W_phi [r,d];
    M0 [b,Hkv,r,d], b0 [b,Hkv,r] (zeros when None) -> (M, b) float64.
    """
    K, V, W_phi = f64(K), f64(V), f64(W_phi)
    E = np.asarray(E)
    b, _, Hkv, d = K.shape
    r = W_phi.shape[0]
    M = np.zeros((b, Hkv, r, d)) if M0 is None else f64(M0).copy()
    bs = np.zeros((b, Hkv, r)) if b0 is None else f64(b0).copy()
    rows = np.arange(b)
    for j in range(E.shape[1]):
        k = K[rows, E[:, j]]                       # [b,Hkv,d]
        v = V[rows, E[:, j]]
        phi = np.einsum("rd,bhd->bhr", W_phi, k)   # [b,Hkv,r]
        M = lam * M + phi[..., :, None] * v[..., None, :]
        bs = lam * bs + phi
    return M, bs


# ---------------------------------------------------------------------------
# Decode step  ([IM-sum] §2.B "Output": o = o_attn + g(q) * m(q), o_attn the
# standard attention over the retained tokens, m(q) the memory readout;
# [IM-abs]: residual readouts compensate the attention lost to eviction)
# ---------------------------------------------------------------------------

def decode_step(q, k_new, v_new, K_R, V_R, cache_len, M, bstab, W_phi, w_gate,
                gate_override: Optional[float] = None, eps: float = READOUT_EPS):
    """One decode step for every sequence.

    q [b,Hq,d]; k_new, v_new [b,Hkv,d] appended at row cache_len[b] of K_R/V_R
    [b,cap,Hkv,d] (updated in place, float64 copies are not written back);
    M [b,Hkv,r,d], bstab [b,Hkv,r]; W_phi [r,d]; w_gate [Hq,d].
    Returns (o [b,Hq,d] float64, new cache_len, o_attn, m, denominators).

      o_attn = softmax(q K^T / sqrt(d)) V  over the cache incl. the new row
      u = W_phi q ; m = M^T u / (b . u + eps) ; g = sigmoid(w_gate[h] . q)
      o = o_attn + g m
    Query head h reads KV head h // (Hq/Hkv).
    """
    q, k_new, v_new = f64(q), f64(k_new), f64(v_new)
    KR, VR = f64(K_R), f64(V_R)
    M, bstab, W_phi, w_gate = f64(M), f64(bstab), f64(W_phi), f64(w_gate)
    cache_len = np.asarray(cache_len).astype(np.int64)
    b, Hq, d = q.shape
    Hkv = k_new.shape[1]
    group = Hq // Hkv
    o = np.zeros((b, Hq, d))
    o_attn = np.zeros((b, Hq, d))
    mread = np.zeros((b, Hq, d))
    den = np.zeros((b, Hq))
    new_len = cache_len + 1
    for bi in range(b):
        n = int(cache_len[bi])
        Kc = np.concatenate([KR[bi, :n], k_new[bi][None]], axis=0)   # [n+1,Hkv,d]
        Vc = np.concatenate([VR[bi, :n], v_new[bi][None]], axis=0)
        for h in range(Hq):
            kv = h // group
            s = Kc[:, kv] @ q[bi, h] / math.sqrt(d)
            p = np.exp(s - s.max())
            p /= p.sum()
            o_attn[bi, h] = p @ Vc[:, kv]
            u = W_phi @ q[bi, h]
            den[bi, h] = bstab[bi, kv] @ u + eps
            mread[bi, h] = (M[bi, kv].T @ u) / den[bi, h]
            g = sigmoid(w_gate[h] @ q[bi, h]) if gate_override is None else gate_override
            o[bi, h] = o_attn[bi, h] + g * mread[bi, h]
    return o, new_len, o_attn, mread, den


def parameter_counts(hidden: int, n_q_heads: int, head_dim: int, idx_dim: int,
                     mem_r: int, n_layers: int) -> Tuple[int, int]:
    """Slow-weight parameter counts implied by the shapes the oracle uses:
    indexer = W_iq [Hq,d,dI] + W_ik [H,dI] + w_ig [H,Hq];
    memory  = W_phi [r,d] + w_gate [Hq,d]; both per layer, times n_layers."""
    idx = n_q_heads * head_dim * idx_dim + hidden * idx_dim + hidden * n_q_heads
    mem = mem_r * head_dim + n_q_heads * head_dim
    return idx * n_layers, mem * n_layers


def prefill_layer(X, Q, K, V, W_iq, W_ik, w_ig, W_phi, lam: float, B: int,
                  cap: Optional[int] = None, ranges=None):
    """The prefill side of the path for one layer, stage by stage:
    indexer features -> pooled importance (over the given query ranges, or all
    queries at once) -> top-B selection -> compaction -> memory update.
    Returns a dict with qhat, khat, gate, I, R, E, K_R, V_R, M, b."""
    qhat, khat, gate = indexer_features(X, Q, W_iq, W_ik, w_ig)
    L = khat.shape[1]
    I = None
    for (q0, q1) in (ranges or [(0, L)]):
        I = pooled_importance(qhat, khat, gate, q_begin=q0, q_end=q1, prev=I)
    R, E = select_budget(I, B)
    KR, VR = compact(np.asarray(K.float() if hasattr(K, "float") else K),
                     np.asarray(V.float() if hasattr(V, "float") else V), R, cap)
    M, bs = memory_update(K, V, E, W_phi, lam)
    return {"qhat": qhat, "khat": khat, "gate": gate, "I": I, "R": R, "E": E,
            "K_R": KR, "V_R": VR, "M": M, "b": bs}


def prefill_streaming(X, Q, K, V, W_iq, W_ik, w_ig, W_phi, lam: float, B: int, ranges):
    """Pre-eviction during chunked prefill ([IM-sum] §2.A: the indexer can evict
    before the whole prefix has been processed, keeping the cache bounded).

    The query ranges are processed in order (contiguous, from 0). Before range
    [q0, q1) the cache holds the retained set R (at most B positions) with
    their pooled importances. The candidates are R followed by the range's own
    keys; their importances are pooled over the range's queries (running max,
    causal within the range: I[t] = max(I_R[t], max_{s in [q0,q1)} A[s,t]) for
    t in R, max_{s in [t,q1)} A[s,t] for t in the range). If there are more
    than B candidates, the B most important stay (ties to the lower position)
    and the others are evicted into the memory in ascending position order,
    after everything evicted by earlier ranges.

    Returns a dict: R [b, min(B, L)] final retained positions (ascending), M, b
    (the memory), and ``chunks``: per range a dict with cand [b, n] candidate
    positions, I [b, n] their importances, R, E (positions, ascending)."""
    qhat, khat, gate = indexer_features(X, Q, W_iq, W_ik, w_ig)
    b, L = khat.shape[:2]
    R = [np.zeros(0, dtype=np.int64) for _ in range(b)]
    IR = [np.zeros(0) for _ in range(b)]
    M = bs = None
    chunks = []
    for (q0, q1) in ranges:
        rec = {"cand": [], "I": [], "R": [], "E": []}
        for bi in range(b):
            cand = np.concatenate([R[bi], np.arange(q0, q1)])
            prev = np.full((1, L), -np.inf)
            prev[0, R[bi]] = IR[bi]
            Ic = pooled_importance(qhat[bi:bi + 1], khat[bi:bi + 1], gate[bi:bi + 1],
                                   q_begin=q0, q_end=q1, prev=prev, keys=cand)[0]
            if len(cand) > B:
                ri, ei = select_budget(Ic[None], B)   # candidate order = position order
                R[bi], E, IR[bi] = cand[ri[0]], cand[ei[0]], Ic[ri[0]]
            else:
                R[bi], E, IR[bi] = cand, np.zeros(0, dtype=np.int64), Ic
            for k, v in (("cand", cand), ("I", Ic), ("R", R[bi]), ("E", E)):
                rec[k].append(v)
        for k in rec:
            rec[k] = np.stack(rec[k])
        if rec["E"].shape[1] > 0:
            M, bs = memory_update(K, V, rec["E"], W_phi, lam, M0=M, b0=bs)
        chunks.append(rec)
    if M is None:
        M, bs = memory_update(K, V, np.zeros((b, 0), dtype=np.int64), W_phi, lam)
    return {"R": np.stack(R), "M": M, "b": bs, "chunks": chunks}


def decode_step_online(x_new, q, k_new, v_new, K_R, V_R, khat_R, I_R, pos_R, next_pos, M, bstab,
                       W_iq, W_ik, w_ig, W_phi, w_gate, lam: float):
    """One decode step with online eviction at a fixed budget ([IM-sum] §2.B:
    the memory is updated online during inference as tokens leave the cache;
    §2.A: the indexer scores keys for the queries that arrive).

    The cache holds B = K_R.shape[1] - 1 tokens in slots [0, B) (any order):
    keys/values K_R, V_R [b, B+1, Hkv, d] (slot B free), indexer keys khat_R
    [b, B+1, dI], importances I_R [b, B+1], positions pos_R [b, B+1].
    x_new [b, H] is the new token's hidden state, q [b, Hq, d] its query,
    k_new, v_new [b, Hkv, d]; next_pos [b] its position.

      1. o = decode_step over slots [0, B) + the new token (memory before
         this step's eviction);
      2. the new token's indexer query q~ and key k^ (indexer_features of the
         token); I_t <- max(I_t, q~ . k^_t) for the cached tokens, and the new
         token's importance is its own score q~ . k^_new;
      3. the least important of the B + 1 leaves (ties: the higher position
         leaves, so that ties keep lower positions); M <- lam M + phi(k) v^T,
         b <- lam b + phi(k) with its key and value;
      4. the new token takes the freed slot (nothing moves if it left itself).

    Returns (o, evicted position [b], new state dict with K_R, V_R, khat_R,
    I_R, pos_R, M, b) -- float64 copies."""
    x_new, q = f64(x_new), f64(q)
    k_new, v_new = f64(k_new), f64(v_new)
    KR, VR = f64(K_R).copy(), f64(V_R).copy()
    khR, IR = f64(khat_R).copy(), f64(I_R).copy()
    posR = np.asarray(pos_R).astype(np.int64).copy()
    M, bs = f64(M).copy(), f64(bstab).copy()
    W_phi = f64(W_phi)
    b = q.shape[0]
    B = KR.shape[1] - 1
    o, _, _, _, _ = decode_step(q, k_new, v_new, KR[:, :B], VR[:, :B], np.full(b, B), M, bs,
                                W_phi, w_gate)
    qhat, khat, gate = indexer_features(x_new[:, None], q[:, None], W_iq, W_ik, w_ig)
    dI = khat.shape[-1]
    q_t = np.einsum("bh,bhd->bd", gate[:, 0], qhat[:, 0]) / math.sqrt(dI)   # q~ [b, dI]
    evicted = np.zeros(b, dtype=np.int64)
    for bi in range(b):
        IR[bi, :B] = np.maximum(IR[bi, :B], khR[bi, :B] @ q_t[bi])
        khR[bi, B] = khat[bi, 0]
        IR[bi, B] = khat[bi, 0] @ q_t[bi]
        KR[bi, B], VR[bi, B] = k_new[bi], v_new[bi]
        posR[bi, B] = int(next_pos[bi])
        # lowest importance leaves; among equal ones the highest position
        e = min(range(B + 1), key=lambda j: (IR[bi, j] + 0.0, -posR[bi, j]))
        evicted[bi] = posR[bi, e]
        k, v = KR[bi, e], VR[bi, e]                      # [Hkv, d]
        phi = k @ W_phi.T                                # [Hkv, r]
        M[bi] = lam * M[bi] + phi[:, :, None] * v[:, None, :]
        bs[bi] = lam * bs[bi] + phi
        if e != B:
            for arr in (KR, VR, khR, IR, posR):
                arr[bi, e] = arr[bi, B]
    state = {"K_R": KR, "V_R": VR, "khat_R": khR, "I_R": IR, "pos_R": posR, "M": M, "b": bs}
    return o, evicted, state


def importance_at_keys(X, Q, W_iq, W_ik, w_ig, keys, q_end: Optional[int] = None,
                       s_block: int = 4096) -> np.ndarray:
    """Pooled importance I[t] = max_{s in [t, q_end)} A[s,t] for a few keys t of
    ONE sequence, streaming the queries in blocks so that long contexts fit in
    host memory (each A[s,t] is still computed per head by the definition of
    ``score_block``). X [L,H], Q [L,Hq,d] (one sequence); keys ascending or not.
    Equals ``pooled_importance`` over the full query range at those keys."""
    X = np.asarray(X) if not hasattr(X, "detach") else X
    L = X.shape[0]
    q_end = L if q_end is None else q_end
    keys = np.asarray(keys)
    W_iq, W_ik, w_ig = f64(W_iq), f64(W_ik), f64(w_ig)
    dI = W_ik.shape[1]
    # keys' own features
    _, khat_all, _ = indexer_features(X[None, keys], Q[None, keys], W_iq, W_ik, w_ig)
    khat = khat_all[0]
    out = np.full(len(keys), -np.inf)
    s_min = int(keys.min())
    for s0 in range(s_min, q_end, s_block):
        s1 = min(q_end, s0 + s_block)
        qhat, _, gate = indexer_features(X[None, s0:s1], Q[None, s0:s1], W_iq, W_ik, w_ig)
        A = score_block(qhat[0], gate[0], khat, dI)                 # [S, T]
        s_idx = np.arange(s0, s1)[:, None]
        A = np.where(s_idx >= keys[None, :], A, -np.inf)
        out = np.maximum(out, A.max(axis=0))
    return out
