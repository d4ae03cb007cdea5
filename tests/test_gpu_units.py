"""GPU unit tests of single library calls, through the C ABI.

* hs_topk_select on scores drawn from a few levels, so that exact ties
  straddle the k-th place: the lower-index tie rule is the one place where
  several selections look plausible, so the result must equal the oracle's
  top-k bit for bit -- for rows staged in shared memory (<= 8192 candidates)
  and rows streamed from global memory (131073 candidates), at batch 1 and 64.
* hs_debug_exp2_poly: the FMA-pipe exponential that the softmax uses for one
  in four of its exponentials, against exact 2^x over the range the softmax
  feeds it, including the clamp at -125.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu


def _level_scores(shape, levels, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    lv = torch.tensor(levels, dtype=torch.float32, device="cuda")
    pick = torch.randint(0, len(levels), shape, generator=g, device="cuda")
    return lv[pick].contiguous()


TOPK_CASES = {
    # name: (ctx, new, Hkv, T, B, k, levels)
    # block level, staged rows: 32768 keys / 64 = 512 candidates at most
    "staged_block64_b1": ((0,), (32768,), 8, 64, 64, 16, [0.25, 0.5, 0.75, 1.0]),
    # block level, batch of 64 short sequences, some rows with fewer candidates than k
    "staged_block16_b64": (tuple(range(0, 64 * 37, 37)), (5,) * 64, 2, 4, 16, 8, [0.125, 0.5, 1.0]),
    # token level at the 8192-candidate staging limit (one row of exactly 8192)
    "staged_token_8192": ((8191 - 63,), (64,), 1, 64, 1, 1024, [0.0, 0.3, 0.6, 0.9]),
    # token level, decode rows: 64 sequences x 131073 candidates, streamed
    "streamed_decode_b64": ((131072,) * 64, (1,) * 64, 1, 1, 1, 1024, [0.1, 0.2, 0.4, 0.8]),
    # token level, one long sequence, tiles of 64, streamed
    "streamed_token_b1": ((131008,), (128,), 1, 64, 1, 1024, [0.5, 0.75, 1.0]),
    # window-exclusive candidates (start before the last query's window of 128), staged and streamed
    "excl_token_staged": ((4000, 100), (64, 64), 1, 64, 1, 1024, [0.25, 0.5, 1.0], 128),
    "excl_decode_streamed": ((131072,) * 8, (1,) * 8, 1, 1, 1, 1024, [0.1, 0.2, 0.4, 0.8], 128),
    "excl_block": ((0,), (4096,), 2, 64, 64, 8, [0.25, 0.5], 100),
}


@pytest.mark.parametrize("name", list(TOPK_CASES))
def test_topk_exact_ties_bit_exact(name):
    import hybrid_sparse_attention_tma_b200 as hs
    ctx, new, Hkv, T, B, k, levels = TOPK_CASES[name][:7]
    win = TOPK_CASES[name][7] if len(TOPK_CASES[name]) > 7 else 0  # window-exclusive cases
    kv = [c + n for c, n in zip(ctx, new)]
    cu_q = [0] + np.cumsum(new).tolist()
    cu_kv = [0] + np.cumsum(kv).tolist()
    vl = hs.Varlen(cu_q, cu_kv, Hkv, Hkv, 128, device="cuda")
    sel = hs.Sel(T, B, k, win, exclusive=win > 0)
    nblk = (max(kv) + B - 1) // B
    scores = _level_scores((vl.n_tiles(T), Hkv, nblk), levels, seed=len(name))
    idx, cnt = hs.topk_select(vl, sel, scores)
    torch.cuda.synchronize()
    sc = scores.cpu().double().numpy()
    idx_o, cnt_o = O.topk_select(sc, cu_q, cu_kv, T, B, k, w=win, exclusive=win > 0)
    assert np.array_equal(cnt.cpu().numpy(), cnt_o)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    # the case really exercises ties at the k-th place
    t0 = O.make_tiles(cu_q, cu_kv, T)[0]
    nc = O.n_candidates(t0, B, win, win > 0)
    if nc > k:
        row = np.sort(sc[0, 0, :nc])[::-1]
        assert row[k - 1] == row[k], "no tie straddles the k-th place"


def test_swa_ring_write_keeps_the_last_positions():
    """hs_swa_ring_write puts the row of position p at slot p mod R and, when a
    call brings more than R new tokens of a sequence, only the last R land
    (a prefill that builds the ring, then one decode token appended)."""
    import hybrid_sparse_attention_tma_b200 as hs
    R, hkv, d = 8, 2, 128
    cu_q, cu_kv = [0, 5, 25, 26], [0, 5, 25, 26]          # 5, 20 and 1 new tokens, no cache
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    k = torch.randn((26, hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((26, hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    kr = torch.zeros((3, R, hkv, d), dtype=torch.bfloat16, device="cuda")
    vr = torch.zeros_like(kr)
    vl = hs.Varlen(cu_q, cu_kv, 4, hkv, d)
    hs.swa_ring_write(vl, k, v, kr, vr)
    # one decode token per sequence at positions 5, 20, 1
    kn = torch.randn((3, hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    vn = torch.randn((3, hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    hs.swa_ring_write(hs.Varlen([0, 1, 2, 3], [0, 6, 27, 29], 4, hkv, d), kn, vn, kr, vr)
    torch.cuda.synchronize()
    ref_k = torch.zeros_like(kr).cpu()
    ref_v = torch.zeros_like(vr).cpu()
    kh, vh, knh, vnh = k.cpu(), v.cpu(), kn.cpu(), vn.cpu()
    for b, (a, e) in enumerate(zip(cu_q[:-1], cu_q[1:])):
        for p in range(max(0, (e - a) - R), e - a):
            ref_k[b, p % R], ref_v[b, p % R] = kh[a + p], vh[a + p]
        p = e - a  # the decode token
        ref_k[b, p % R], ref_v[b, p % R] = knh[b], vnh[b]
    assert torch.equal(kr.cpu().view(torch.int16), ref_k.view(torch.int16))
    assert torch.equal(vr.cpu().view(torch.int16), ref_v.view(torch.int16))


def test_kv_dequantize_bit_exact():
    """hs_kv_dequantize: bf16_rn(fp32(scale) * fp32(e4m3(code))) for every row,
    bit for bit against the same arithmetic by torch on the host (every code
    value appears, including subnormals and +-448)."""
    import hybrid_sparse_attention_tma_b200 as hs
    import workloads as W
    g = torch.Generator(device="cuda")
    g.manual_seed(4)
    x = torch.randn((3001, 2, 128), generator=g, device="cuda") * 3.0
    codes, scale = W.quantize_e4m3_per_token(x)
    codes = codes.clone()
    codes[0, 0] = torch.arange(128, dtype=torch.uint8, device="cuda")          # codes 0..127
    codes[0, 1] = torch.arange(128, 256, dtype=torch.uint8, device="cuda")     # codes 128..255
    codes[0, 1, 127] = 0x7E  # keep NaN codes (0x7F, 0xFF) out of the comparison
    codes[0, 0, 127] = 0x7E
    out = hs.kv_dequantize(codes, scale)
    torch.cuda.synchronize()
    ref = (codes.cpu().view(torch.float8_e4m3fn).float() * scale.cpu().unsqueeze(-1)).to(torch.bfloat16)
    assert torch.equal(out.cpu().view(torch.int16), ref.view(torch.int16))


def _exp2_poly(x: np.ndarray) -> np.ndarray:
    import hybrid_sparse_attention_tma_b200._lib as L
    lib = L.load()
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    yd = torch.empty_like(xd)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.hs_debug_exp2_poly(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(yd.data_ptr()), xd.numel(), s)
    assert st == L.HS_OK
    torch.cuda.synchronize()
    return yd.cpu().numpy().astype(np.float64)


def test_exp2_poly_relative_error_and_clamp():
    # the softmax feeds x = s * c - m with the lazily kept max m: x <= 8
    x = np.concatenate([
        np.linspace(-130.0, 8.0, 2_000_001),
        np.arange(-125, 9, dtype=np.float64),           # integers: f = 0
        np.arange(-125, 8, dtype=np.float64) + 0.5,     # f = +-1/2 edges of the reduction
        np.arange(-124, 9, dtype=np.float64) - 0.5,
        [0.0, -0.0, -125.0, -124.999, -125.001, -126.0, -200.0, -1e30],
    ]).astype(np.float32)
    y = _exp2_poly(x)
    xd = x.astype(np.float64)
    normal = xd >= -125.0
    exact = np.exp2(xd[normal])
    rel = np.abs(y[normal] - exact) / exact
    assert rel.max() <= 7.5e-5, f"max relative error {rel.max():.3e}"
    # below the clamp the result is the clamp's value, about 2^-125: zero for the softmax
    below = y[~normal]
    assert (below >= 0).all() and (below <= 2.0 ** -125 * (1 + 7.5e-5)).all()
    # at x = 0 the reduction is the identity (j = 0, f = 0)
    assert abs(_exp2_poly(np.zeros(2, dtype=np.float32))[0] - 1.0) <= 7.5e-5

