"""One IndexMem layer on the GPU: owns the library context and the caller-side
buffers (allocated with torch), and calls the C ABI through ``binding``.

Plumbing only -- every step of the path runs in libindexmem.so's kernels.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import binding as B_


@dataclasses.dataclass
class PrefillState:
    running_max: torch.Tensor     # [b, L] fp32
    idx_retained: torch.Tensor    # [b, B] int32
    idx_evicted: torch.Tensor     # [b, L-B] int32
    K_ret: torch.Tensor           # [b, cap, Hkv, d]
    V_ret: torch.Tensor
    cache_len: torch.Tensor       # [b] int32
    M: torch.Tensor               # [b, Hkv, r, d] fp32 (moment readout: S^T, r = d)
    bstab: torch.Tensor           # [b, Hkv, r] fp32 (moment readout: s_k)
    s_v: Optional[torch.Tensor] = None   # [b, Hkv, d] fp32, moment readout only
    n_e: Optional[torch.Tensor] = None   # [b] fp32, moment readout only


@dataclasses.dataclass
class OnlineState:
    """Decode-time online eviction: per cache slot the indexer key, the
    importance and the position; the next token's position; the position
    evicted by the last step."""
    khat_ret: torch.Tensor        # [b, cap, 64] bf16
    I_ret: torch.Tensor           # [b, cap] fp32
    pos_ret: torch.Tensor         # [b, cap] int32
    next_pos: torch.Tensor        # [b] int32
    evicted: torch.Tensor         # [b] int32


class IndexMemLayer:
    """Context for one layer. ``weights`` holds device tensors W_iq [Hq,d,dI],
    W_ik [H,dI], w_ig [H,Hq] (model dtype), W_phi [r,d], w_gate [Hq,d] (fp32).

    readout="gated" is IndexMem's memory readout; readout="moment" keeps
    MomentKV's moment statistics instead (r = d, no decay; W_phi and w_gate
    are not used): update_memory then accumulates them and decode mixes the
    retained attention with their estimate of the evicted attention."""

    def __init__(self, hidden, n_q_heads, n_kv_heads, head_dim, idx_dim, mem_r, lam, dtype,
                 weights, gate_override: Optional[float] = None, eps: float = 1e-6,
                 readout: str = "gated"):
        if readout not in ("gated", "moment"):
            raise ValueError("readout must be 'gated' or 'moment'")
        self.moment = readout == "moment"
        if self.moment:
            mem_r, lam = head_dim, 1.0
        self.dims = dict(hidden=hidden, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads,
                         head_dim=head_dim, idx_dim=idx_dim, mem_r=mem_r)
        self.lam = lam
        self.torch_dtype = dtype
        self.code = B_.BF16 if dtype == torch.bfloat16 else B_.FP32
        cfg = B_.make_config(hidden, n_q_heads, n_kv_heads, head_dim, idx_dim, mem_r, lam,
                             self.code, eps=eps, gate_override=gate_override,
                             readout=B_.READOUT_MOMENT if self.moment else B_.READOUT_GATED)
        self.ctx = B_.init(cfg, weights["W_iq"], weights["W_ik"], weights["w_ig"],
                           None if self.moment else weights["W_phi"],
                           None if self.moment else weights["w_gate"])
        self._ws = None
        self._ws_key = None

    @classmethod
    def from_shape(cls, shape, weights, gate_override=None, readout: str = "gated"):
        return cls(shape.hidden, shape.n_q_heads, shape.n_kv_heads, shape.head_dim,
                   shape.idx_dim, shape.mem_r, shape.lam, shape.torch_dtype, weights,
                   gate_override=gate_override, readout=readout)

    def close(self):
        if self.ctx:
            B_.destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- buffers ---------------------------------------------------------------
    def workspace(self, batch: int, L: int, B: int, device) -> torch.Tensor:
        key = (batch, L, B)
        if self._ws is None or self._ws_key != key:
            n = B_.workspace_size(self.ctx, batch, L, B)
            self._ws = torch.zeros(n, dtype=torch.uint8, device=device)   # zero-filled once
            self._ws_key = key
        return self._ws

    def workspace_evict(self, batch: int, L: int, B: int, chunk: int, device) -> torch.Tensor:
        """Workspace for pre-eviction (also serves decode)."""
        key = ("evict", batch, L, B, chunk)
        if self._ws is None or self._ws_key != key:
            n = B_.workspace_size_evict(self.ctx, batch, L, B, chunk)
            self._ws = torch.zeros(n, dtype=torch.uint8, device=device)
            self._ws_key = key
        return self._ws

    def new_state(self, batch: int, L: int, B: int, cap: int, device) -> PrefillState:
        d, Hkv, r = self.dims["head_dim"], self.dims["n_kv_heads"], self.dims["mem_r"]
        return PrefillState(
            running_max=torch.empty(batch, L, dtype=torch.float32, device=device),
            idx_retained=torch.empty(batch, B, dtype=torch.int32, device=device),
            idx_evicted=torch.empty(batch, max(L - B, 1), dtype=torch.int32, device=device),
            K_ret=torch.zeros(batch, cap, Hkv, d, dtype=self.torch_dtype, device=device),
            V_ret=torch.zeros(batch, cap, Hkv, d, dtype=self.torch_dtype, device=device),
            cache_len=torch.full((batch,), B, dtype=torch.int32, device=device),
            M=torch.zeros(batch, Hkv, r, d, dtype=torch.float32, device=device),
            bstab=torch.zeros(batch, Hkv, r, dtype=torch.float32, device=device),
            s_v=(torch.zeros(batch, Hkv, d, dtype=torch.float32, device=device)
                 if self.moment else None),
            n_e=torch.zeros(batch, dtype=torch.float32, device=device) if self.moment else None)

    # -- the path --------------------------------------------------------------
    def score_and_evict(self, X, Q, K, V, st: PrefillState, B: int, q_ranges=None,
                        stream=None):
        batch, L = X.shape[0], X.shape[1]
        ws = self.workspace(batch, L, B, X.device)
        ranges = q_ranges or [(0, L)]
        for i, (q0, q1) in enumerate(ranges):
            last = i == len(ranges) - 1
            B_.score_and_evict(self.ctx, batch, L, B, X, Q, K, V, st.running_max, q0, q1,
                               1 if last else 0, st.idx_retained,
                               st.idx_evicted if B < L else None, st.K_ret, st.V_ret,
                               st.K_ret.shape[1], ws, stream)

    def prefill_evict(self, X, Q, K, V, st: PrefillState, B: int, chunk: int,
                      mem_chunk: int = 512, stream=None, record: bool = False):
        """Chunked prefill with pre-eviction after every query range of
        ``chunk`` tokens: the cache never holds more than B tokens and the
        evicted ones enter the memory as they leave. Fills st.idx_retained
        (first min(B, L) entries), st.K_ret/V_ret, st.M, st.bstab.
        record=True returns per range the candidates' importances, the
        retained and the evicted positions (copies, for inspection)."""
        batch, L = X.shape[0], X.shape[1]
        ws = self.workspace_evict(batch, L, B, chunk, X.device)
        ev = torch.empty(batch * chunk, dtype=torch.int32, device=X.device)
        cand = (torch.empty(batch, B + chunk, dtype=torch.float32, device=X.device)
                if record else None)
        recs = []
        for q0 in range(0, L, chunk):
            q1 = min(L, q0 + chunk)
            B_.prefill_evict_chunk(self.ctx, batch, L, B, chunk, X, Q, K, V, q0, q1,
                                   st.idx_retained, ev, cand, st.M, st.bstab, mem_chunk,
                                   q1 == L, st.K_ret, st.V_ret, st.K_ret.shape[1], ws, stream)
            if record:
                B_.join(self.ctx, stream)   # the range's selection runs on a second stream
                n = min(B, q0) + (q1 - q0)
                n_ev = max(0, n - B)
                recs.append({"range": (q0, q1), "I": cand[:, :n].clone(),
                             "retained": st.idx_retained[:, :min(B, q1)].clone(),
                             "evicted": ev[:batch * n_ev].view(batch, n_ev).clone()})
        st.cache_len.fill_(min(B, L))
        return recs

    def update_memory(self, K, V, st: PrefillState, B: int, chunk: int = 512, stream=None):
        batch, L = K.shape[0], K.shape[1]
        ws = self.workspace(batch, L, B, K.device)
        idx = st.idx_evicted if B < L else None
        if self.moment:
            B_.update_moments(self.ctx, batch, L, K, V, idx, L - B, chunk, st.M, st.bstab, st.s_v,
                              st.n_e, ws, stream)
        else:
            B_.update_memory(self.ctx, batch, L, K, V, idx, L - B, chunk, st.M, st.bstab, ws,
                             stream)

    def invalidate_decode(self, batch: int, stream=None):
        """After writing a retained cache, its length or the memory state
        other than through this layer: the next decode step then loads
        nothing before its launch-dependency wait."""
        if self._ws is not None:
            B_.decode_invalidate(self.ctx, batch, self._ws, stream)

    def decode(self, q, k_new, v_new, st: PrefillState, out=None, B: Optional[int] = None,
               L: Optional[int] = None, stream=None):
        batch = q.shape[0]
        if self._ws is None:
            raise RuntimeError("decode needs the workspace of a prefill (or call workspace())")
        if out is None:
            out = torch.empty_like(q)
        if self.moment:
            B_.decode_moment(self.ctx, batch, q, k_new, v_new, st.K_ret, st.V_ret, st.cache_len,
                             st.K_ret.shape[1], st.M, st.bstab, st.s_v, st.n_e, out, self._ws,
                             stream)
        else:
            B_.decode(self.ctx, batch, q, k_new, v_new, st.K_ret, st.V_ret, st.cache_len,
                      st.K_ret.shape[1], st.M, st.bstab, out, self._ws, stream)
        return out

    def online_init(self, st: PrefillState, B: int, L: int, stream=None) -> OnlineState:
        """State for decode-time online eviction after a one-shot prefill of L
        tokens into st (same layer, same workspace); the cache has B tokens."""
        batch, cap = st.K_ret.shape[0], st.K_ret.shape[1]
        dev = st.K_ret.device
        on = OnlineState(
            khat_ret=torch.zeros(batch, cap, 64, dtype=torch.bfloat16, device=dev),
            I_ret=torch.zeros(batch, cap, dtype=torch.float32, device=dev),
            pos_ret=torch.zeros(batch, cap, dtype=torch.int32, device=dev),
            next_pos=torch.zeros(batch, dtype=torch.int32, device=dev),
            evicted=torch.zeros(batch, dtype=torch.int32, device=dev))
        B_.online_init(self.ctx, batch, L, B, st.running_max, st.idx_retained, self._ws,
                       on.khat_ret, on.I_ret, on.pos_ret, on.next_pos, cap, stream)
        return on

    def decode_online(self, x_new, q, k_new, v_new, st: PrefillState, on: OnlineState, B: int,
                      out=None, stream=None):
        """One decode step that keeps the cache at B tokens: the least
        important of the B + 1 leaves into the memory (on.evicted: its
        position)."""
        batch = q.shape[0]
        if out is None:
            out = torch.empty_like(q)
        B_.decode_online(self.ctx, batch, B, x_new, q, k_new, v_new, st.K_ret, st.V_ret,
                         on.khat_ret, on.I_ret, on.pos_ret, on.next_pos, st.cache_len,
                         st.K_ret.shape[1], st.M, st.bstab, out, on.evicted, self._ws, stream)
        return out

    def sync(self, stream=None):
        B_.sync(self.ctx, stream)
