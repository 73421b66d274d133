"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare with the tolerances
the correctness criteria state:

  scores   |dI| <= 1e-2 * max(max|I_ref|, rms(I_ref))      per sequence
  indices  bit-exact (the oracle's top-B of the GPU's scores)
  cache    bit-exact gather
  memory   ||dM||_F / ||M_ref||_F <= 1e-3                   per (sequence, KV head)
  decode   |do| <= 1e-2 + 2e-2 |o_ref| elementwise; readouts whose denominator
           is ill-conditioned (|b.u| < 1e-4 ||b|| ||u||) are excluded (at most
           0.1% of them), their attention part is checked by a gate-0 run.

Where the GPU path takes a decision or produces a state that a later stage
consumes (the retained set from its scores, the memory state M, b that decode
reads), the oracle's later stage is run on the GPU's own decision or state,
and that decision or state is checked separately at its own tolerance.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from learned_kv_cache_indexmem_b200 import synth
from learned_kv_cache_indexmem_b200.layer import IndexMemLayer
from oracle import indexmem_oracle as om

SCORE_TOL = 1e-2
MEM_TOL = 1e-3
DEC_ATOL, DEC_RTOL = 1e-2, 2e-2
ILL_COND = 1e-4


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_scores(I_gpu, I_ref, what=""):
    I_gpu = np.asarray(I_gpu, dtype=np.float64)
    for bi in range(I_ref.shape[0]):
        ref = I_ref[bi]
        scale = max(np.abs(ref).max(), math.sqrt(np.mean(ref ** 2)))
        err = np.abs(I_gpu[bi] - ref).max()
        assert err <= SCORE_TOL * scale, "%s seq %d: score err %.3e > %.3e" % (
            what, bi, err, SCORE_TOL * scale)


def check_memory(M_gpu, b_gpu, M_ref, b_ref, what=""):
    M_gpu, b_gpu = np.asarray(M_gpu, np.float64), np.asarray(b_gpu, np.float64)
    for bi in range(M_ref.shape[0]):
        for h in range(M_ref.shape[1]):
            for g, r, name in ((M_gpu[bi, h], M_ref[bi, h], "M"), (b_gpu[bi, h], b_ref[bi, h], "b")):
                nr = np.linalg.norm(r)
                err = np.linalg.norm(g - r)
                assert err <= MEM_TOL * max(nr, 1e-30), "%s %s seq %d head %d: rel %.3e" % (
                    what, name, bi, h, err / max(nr, 1e-30))


def ill_conditioned(bstab, q, W_phi, group):
    """mask [b, Hq] of readouts whose denominator b.u cancels: |b.u| < 1e-4 |b||u|."""
    b_, Hq, d = q.shape
    u = np.einsum("rd,bhd->bhr", W_phi, q)
    bk = np.repeat(bstab, group, axis=1)                 # [b, Hq, r]
    dot = np.abs(np.sum(bk * u, -1))
    return dot < ILL_COND * np.linalg.norm(bk, axis=-1) * np.linalg.norm(u, axis=-1)


def check_decode(o_gpu, o_ref, mask_ill=None, what=""):
    o_gpu = np.asarray(o_gpu, np.float64)
    tol = DEC_ATOL + DEC_RTOL * np.abs(o_ref)
    bad = np.abs(o_gpu - o_ref) > tol
    if mask_ill is not None:
        frac = mask_ill.mean()
        assert frac <= 1e-3 or mask_ill.sum() <= 1, "%s: %.3f%% ill-conditioned readouts" % (
            what, 100 * frac)
        bad &= ~mask_ill[..., None]
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError("%s: %d decode mismatches, first at %s gpu=%g ref=%g" % (
            what, int(bad.sum()), tuple(idx), o_gpu[tuple(idx)], o_ref[tuple(idx)]))


class Case:
    """Seeded inputs of one workload (possibly shrunk), generated on `gen_device`
    and held on the GPU for the CUDA path and on the CPU for the oracle."""

    def __init__(self, wl: synth.Workload, device, L=None, batch=None, gen_device="cpu",
                 n_decode=None, seed=None):
        self.wl = wl
        self.shape = wl.shape
        self.L = wl.L if L is None else L
        self.batch = wl.batch if batch is None else batch
        self.n_decode = wl.n_decode if n_decode is None else n_decode
        self.seed = wl.seed if seed is None else seed
        w = synth.make_weights(wl.shape, self.seed, gen_device)
        inp = synth.make_layer_inputs(wl, w, self.seed, gen_device, L=self.L, batch=self.batch)
        dec = synth.make_decode_inputs(wl, w, self.n_decode, self.seed, gen_device, batch=self.batch)
        self.w_dev = {k: v.to(device) for k, v in w.items()}
        self.in_dev = {k: v.to(device) for k, v in inp.items()}
        self.dec_dev = {k: v.to(device) for k, v in dec.items()}
        self.w_cpu = {k: v.cpu() for k, v in w.items()}
        self.in_cpu = {k: v.cpu() for k, v in inp.items()}
        self.dec_cpu = {k: v.cpu() for k, v in dec.items()}
        self.device = device

    def layer(self, gate_override=None) -> IndexMemLayer:
        return IndexMemLayer.from_shape(self.shape, self.w_dev, gate_override=gate_override)

    def oracle_features(self):
        c = self.in_cpu
        w = self.w_cpu
        return om.indexer_features(c["X"], c["Q"], w["W_iq"], w["W_ik"], w["w_ig"])
