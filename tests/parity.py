"""Helpers for the GPU-vs-oracle parity tests (imported by tests only).

Tolerances (from the required match against the oracle):
  * bf16 outputs: max |err| <= 3e-2 and mean |err| <= 3e-3
  * lse: |err| <= 1e-3 (natural log)
  * FP8-KV outputs: max |err| <= 8e-2
  * indices: bit-exact, except candidates whose oracle score lies within 1e-3
    (relative) of the k-th largest oracle score
  * importance scores: relative error <= 2e-3 (exp of a logit difference whose
    fp32 error is ~1e-5; not a stated bar, derived from the arithmetic)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from workloads import bf16_bits

O_MAX, O_MEAN, LSE_TOL, FP8_MAX = 3e-2, 3e-3, 1e-3, 8e-2
SCORE_RTOL = 2e-3
TIE_BAND = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return O.bf16_to_f64(bf16_bits(t))
    return t.detach().to("cpu").double().numpy()


class LazyF64:
    """Read-only float64 view of a (device) tensor: only the slices the oracle
    asks for are copied to the host and decoded."""

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.shape = tuple(t.shape)

    def _conv(self, i):
        if isinstance(i, np.ndarray):
            return torch.from_numpy(i.astype(np.int64)).to(self.t.device)
        if isinstance(i, tuple):
            return tuple(self._conv(x) for x in i)
        return i

    def __getitem__(self, idx):
        return f64(self.t[self._conv(idx)])


def assert_close_out(got: np.ndarray, want: np.ndarray, max_tol=O_MAX, mean_tol=O_MEAN, what="o"):
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.isfinite(want).all() and np.isfinite(got).all(), what
    err = np.abs(got - want)
    assert err.max() <= max_tol, f"{what}: max abs err {err.max():.3e} > {max_tol}"
    assert err.mean() <= mean_tol, f"{what}: mean abs err {err.mean():.3e} > {mean_tol}"


def assert_close_lse(got: np.ndarray, want: np.ndarray, what="lse"):
    fin = np.isfinite(want)
    assert (np.isfinite(got) == fin).all(), f"{what}: finiteness differs"
    assert (got[~fin] == want[~fin]).all()
    if fin.any():
        err = np.abs(got[fin] - want[fin]).max()
        assert err <= LSE_TOL, f"{what}: max abs err {err:.3e} > {LSE_TOL}"


def assert_scores_close(got: np.ndarray, want: np.ndarray, tiles, what="scores"):
    for t in tiles:
        g, w = got[t], want[t]
        assert ((g == 0) == (w == 0)).all(), f"{what}: candidate pattern differs in tile {t}"
        nz = w > 0
        rel = np.abs(g[nz] - w[nz]) / w[nz]
        assert rel.max(initial=0) <= SCORE_RTOL, f"{what}: tile {t} rel err {rel.max():.3e}"


def assert_indices_match(idx_g, cnt_g, scores_o, idx_o, cnt_o, tiles, k):
    """Bit-exact except inside the oracle's tie band around the k-th score."""
    for t in tiles:
        for g in range(idx_o.shape[1]):
            co, cg = int(cnt_o[t, g]), int(cnt_g[t, g])
            assert co == cg, f"cnt differs at tile {t} head {g}: {cg} vs {co}"
            so = set(idx_o[t, g, :co].tolist())
            sg = set(idx_g[t, g, :cg].tolist())
            assert (idx_g[t, g, cg:] == -1).all()
            assert (np.diff(idx_g[t, g, :cg]) > 0).all(), "indices not ascending"
            if so == sg:
                continue
            sc = scores_o[t, g]
            kth = np.sort(sc[list(so)])[0] if so else 0.0
            for j in so ^ sg:
                assert abs(sc[j] - kth) <= TIE_BAND * kth, \
                    f"tile {t} head {g}: index {j} differs outside the tie band"


class GpuBlock:
    """Runs one hybrid block through the library's public block runner.

    The top-k runs as its own call on stored scores (the runner's default) so
    the scores can be checked against the oracle; the fused top-k
    (fuse_topk=True) is checked bit for bit against that path."""

    def __init__(self, w, inp, device="cuda", fused=True, fuse_topk=False):
        import hybrid_sparse_attention_tma_b200 as hs
        from hybrid_sparse_attention_tma_b200.block import HybridBlock, SparseLayerIn
        self.w = w
        self.inp = inp
        self.vl = hs.Varlen(w.cu_q(), w.cu_kv(), w.n_q_heads, w.n_kv_heads, w.head_dim, device=device)
        self.sel = hs.Sel(w.q_tile, w.block, w.topk, w.window, w.exclusive)
        self.block = HybridBlock(self.vl, w.q_tile, w.block, w.topk, w.window, w.swa_window, device=device,
                                 fused=fused, exclusive=w.exclusive, fuse_topk=fuse_topk)
        if self.block.decode and w.swa_window > 0:
            # decode reads each layer's own window cache as a ring of swa_window slots
            self.layers = [SparseLayerIn(L.q, *self.block.swa_rings(L.k_swa, L.v_swa), L.gamma) for L in inp.layers]
        else:
            self.layers = [SparseLayerIn(L.q, L.k_swa, L.v_swa, L.gamma) for L in inp.layers]

    def run(self, stream=None, fp8=False, intermediates=True):
        fp8_kv = None
        if fp8:
            fp8_kv = (self.inp.k_fp8, self.inp.v_fp8, self.inp.k_scale, self.inp.v_scale)
        return self.block.forward(self.inp.q, self.inp.k, self.inp.v, self.layers, stream=stream, keep_all=True,
                                  fp8_kv=fp8_kv, intermediates=intermediates)
