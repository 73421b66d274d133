"""Pins of the oracle's decode step: torch's scaled_dot_product_attention in
float64 (textbook softmax attention), a hand-worked example, and the closed
forms of the memory readout.

Sources: "IndexMem" technical summary §2.B Output (o = o_attn + g(q) m(q), with
o_attn the standard attention over the retained tokens); "IndexMem: Learned
KV-Cache Eviction with Latent Memory for Long-Context LLM Inference" abstract
(residual readouts compensate for attention lost to eviction).
"""
import math

import numpy as np
import pytest
import torch

from oracle import indexmem_oracle as om


def _case(rng, b=2, cap=20, n=13, Hq=6, Hkv=2, d=8, r=5):
    q = rng.standard_normal((b, Hq, d))
    kn = rng.standard_normal((b, Hkv, d))
    vn = rng.standard_normal((b, Hkv, d))
    KR = np.zeros((b, cap, Hkv, d)); VR = np.zeros((b, cap, Hkv, d))
    KR[:, :n] = rng.standard_normal((b, n, Hkv, d))
    VR[:, :n] = rng.standard_normal((b, n, Hkv, d))
    M = rng.standard_normal((b, Hkv, r, d))
    bs = rng.standard_normal((b, Hkv, r))
    W = rng.standard_normal((r, d)) / math.sqrt(d)
    wg = rng.standard_normal((Hq, d)) / math.sqrt(d)
    lens = np.array([n, n - 4])[:b]
    return q, kn, vn, KR, VR, lens, M, bs, W, wg


def test_attention_part_equals_torch_sdpa_float64():
    """Gate forced to 0 -> plain softmax attention over cache + new row, GQA
    grouping h // (Hq/Hkv): equals torch's SDPA (scale 1/sqrt(d)) in float64."""
    rng = np.random.default_rng(20)
    q, kn, vn, KR, VR, lens, M, bs, W, wg = _case(rng)
    o, new_len, o_attn, _, _ = om.decode_step(q, kn, vn, KR, VR, lens, M, bs, W, wg,
                                              gate_override=0.0)
    assert list(new_len) == list(lens + 1)
    assert np.array_equal(o, o_attn)
    for bi in range(2):
        n = lens[bi]
        Kc = np.concatenate([KR[bi, :n], kn[bi][None]])
        Vc = np.concatenate([VR[bi, :n], vn[bi][None]])
        kt = torch.from_numpy(Kc).permute(1, 0, 2)[None].repeat_interleave(3, dim=1)
        vt = torch.from_numpy(Vc).permute(1, 0, 2)[None].repeat_interleave(3, dim=1)
        qt = torch.from_numpy(q[bi])[None, :, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0].numpy()
        assert np.allclose(o[bi], ref, rtol=1e-12, atol=1e-12)


def test_full_budget_is_full_attention_with_empty_memory():
    """B = L: nothing evicted, M = 0 and b = 0, so m = 0 and o = full attention."""
    rng = np.random.default_rng(21)
    b, L, Hkv, d, Hq = 1, 12, 2, 4, 4
    K = rng.standard_normal((b, L, Hkv, d)); V = rng.standard_normal((b, L, Hkv, d))
    R, E = om.select_budget(rng.standard_normal((b, L)), L)
    KR, VR = om.compact(K, V, R, cap=L + 1)
    W = rng.standard_normal((3, d))
    M, bs = om.memory_update(K, V, E, W, 0.9)
    assert not M.any() and not bs.any()
    q = rng.standard_normal((b, Hq, d)); kn = rng.standard_normal((b, Hkv, d))
    vn = rng.standard_normal((b, Hkv, d))
    o, _, o_attn, m, _ = om.decode_step(q, kn, vn, KR, VR, [L], M, bs, W,
                                        rng.standard_normal((Hq, d)))
    assert not m.any()
    assert np.array_equal(o, o_attn)
    Kc = np.concatenate([K[0], kn]); Vc = np.concatenate([V[0], vn])
    kt = torch.from_numpy(Kc).permute(1, 0, 2)[None].repeat_interleave(2, dim=1)
    vt = torch.from_numpy(Vc).permute(1, 0, 2)[None].repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[0])[None, :, None, :], kt, vt)[0, :, 0].numpy()
    assert np.allclose(o[0], ref, rtol=1e-12, atol=1e-12)


def test_decode_hand_worked_example():
    """d = 4 (scale 1/2), Hq = 2, Hkv = 1, one cached row plus the new row, r = 1.
    K_R[0] = (2,0,0,0), V_R[0] = (1,0,0,0); k_new = 0, v_new = (0,1,0,0).
    head 0: q = (ln 3,0,0,0) -> logits (ln 3, 0) -> p = (3/4, 1/4) -> o_attn = (3/4,1/4,0,0)
    head 1: q = 0 -> p = (1/2,1/2) -> o_attn = (1/2,1/2,0,0)
    W_phi = [[1,0,0,0]] -> u = q_0; M = [[0,0,2,0]], b = [1]:
      head 0: m = (0,0,2 ln3,0)/(ln3 + 1e-6); gate weights 0 -> g = 1/2
      head 1: u = 0 -> m = 0
    """
    l3 = math.log(3.0)
    q = np.array([[[l3, 0, 0, 0], [0, 0, 0, 0]]], dtype=np.float64)
    KR = np.zeros((1, 2, 1, 4)); VR = np.zeros((1, 2, 1, 4))
    KR[0, 0, 0] = [2, 0, 0, 0]; VR[0, 0, 0] = [1, 0, 0, 0]
    kn = np.zeros((1, 1, 4)); vn = np.array([[[0, 1, 0, 0]]], dtype=np.float64)
    M = np.array([[[[0, 0, 2, 0]]]], dtype=np.float64)
    bs = np.array([[[1.0]]])
    W = np.array([[1.0, 0, 0, 0]])
    wg = np.zeros((2, 4))
    o, new_len, o_attn, m, den = om.decode_step(q, kn, vn, KR, VR, [1], M, bs, W, wg)
    assert new_len[0] == 2
    assert np.allclose(o_attn[0, 0], [0.75, 0.25, 0, 0], atol=1e-15)
    assert np.allclose(o_attn[0, 1], [0.5, 0.5, 0, 0], atol=1e-15)
    m0 = 2 * l3 / (l3 + 1e-6)
    assert np.allclose(o[0, 0], [0.75, 0.25, 0.5 * m0, 0], atol=1e-15)
    assert np.allclose(o[0, 1], [0.5, 0.5, 0, 0], atol=1e-15)
    assert den[0, 1] == pytest.approx(1e-6)


def test_rank_one_memory_readout_closed_form():
    """One evicted token (k, v) from an empty state: M = phi(k) v^T, b = phi(k),
    so m(q) = v * s / (s + eps) with s = phi(k) . phi(q)."""
    rng = np.random.default_rng(22)
    d, r, Hq = 8, 5, 2
    k = rng.standard_normal(d); v = rng.standard_normal(d)
    K = np.zeros((1, 2, 1, d)); V = np.zeros((1, 2, 1, d))
    K[0, 1, 0] = k; V[0, 1, 0] = v
    W = rng.standard_normal((r, d))
    M, bs = om.memory_update(K, V, np.array([[1]]), W, 0.99)
    q = rng.standard_normal((1, Hq, d))
    KR = np.zeros((1, 1, 1, d)); VR = np.zeros((1, 1, 1, d))
    _, _, _, m, _ = om.decode_step(q, np.zeros((1, 1, d)), np.zeros((1, 1, d)), KR, VR, [0],
                                   M, bs, W, np.zeros((Hq, d)))
    for h in range(Hq):
        s = (W @ k) @ (W @ q[0, h])
        assert np.allclose(m[0, h], v * s / (s + 1e-6), rtol=1e-12)


def test_zero_memory_gives_plain_attention():
    rng = np.random.default_rng(23)
    q, kn, vn, KR, VR, lens, M, bs, W, wg = _case(rng)
    o, _, o_attn, m, _ = om.decode_step(q, kn, vn, KR, VR, lens, 0 * M, 0 * bs, W, wg)
    assert not m.any() and np.array_equal(o, o_attn)


def test_gate_is_sigmoid_of_query():
    """o - o_attn = g m with g = 1/(1+exp(-w_g . q)) per query head."""
    rng = np.random.default_rng(24)
    q, kn, vn, KR, VR, lens, M, bs, W, wg = _case(rng)
    o, _, o_attn, m, _ = om.decode_step(q, kn, vn, KR, VR, lens, M, bs, W, wg)
    g = torch.sigmoid(torch.einsum("hd,bhd->bh", torch.from_numpy(wg), torch.from_numpy(q))).numpy()
    assert np.allclose(o - o_attn, g[..., None] * m, rtol=1e-12, atol=1e-12)
