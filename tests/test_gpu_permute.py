"""GPU parity of the channel permutation search and the column gather
([Orin ch.7] 3.1 step 2 and 6.3) against the CPU oracle.

The search works on exact integers, so the bar is bit-exact: the same
permutation, the same number of exchanges and the same kept scores.  At the
full layer size, where the oracle's search would take too long, the result is
checked through properties that hold at any size: it is a permutation, its
kept score recomputed by the oracle equals the one reported, and (once the
search has stopped on its own) no sampled exchange raises the kept score.
"""
import time

import numpy as np
import pytest
import torch

from oracle import sp24_oracle as O
from structured_sparse_gemm_sp24_b200 import inputs as I
from structured_sparse_gemm_sp24_b200 import pipeline as P
from structured_sparse_gemm_sp24_b200 import sp24 as B

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    B.lib()
    assert B.sp24_device_status() == B.SP24_OK


def f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def run_gpu(w_bf16, n_keep, norms=None, max_swaps=1 << 20):
    nd = None if norms is None else torch.from_numpy(norms).cuda()
    perm, res = P.permute_search(w_bf16.cuda(), n_keep, nd, max_swaps)
    assert B.sp24_device_status() == B.SP24_OK
    return perm.cpu().numpy().astype(np.int64), res


def run_oracle(w_bf16, n_keep, norms=None, max_swaps=1 << 20):
    mode = O.MAGNITUDE if norms is None else O.WANDA
    q = O.permutation_scores(f64(w_bf16), mode, norms)
    return (q,) + O.permutation_search(q, n_keep, max_swaps)


# (N, K, n_keep, wanda, max_swaps): K = 100 and 132 leave ragged 64-channel
# gain tiles, N = 300 spans several 32-row stages and row slices.
CASES = [
    (37, 64, 2, False, None),
    (64, 100, 3, False, None),
    (130, 68, 2, True, None),
    (300, 132, 2, False, 6),
    (1, 16, 2, False, None),
    (50, 8, 3, False, None),
    (257, 40, 3, True, None),
]


@pytest.mark.parametrize("n,k,n_keep,wanda,max_swaps", CASES)
def test_search_matches_oracle(n, k, n_keep, wanda, max_swaps):
    seed = n * 1000 + k
    w = I.channel_scaled_bf16((n, k), 0.02, seed)
    norms = None
    if wanda:
        xc = I.normal_bf16((48, k), 1.0, seed + 2)
        norms = O.column_norms(f64(xc))
    limit = (1 << 20) if max_swaps is None else max_swaps
    q, perm_o, swaps_o, before_o, after_o = run_oracle(w, n_keep, norms, limit)
    perm_g, res = run_gpu(w, n_keep, norms, limit)
    assert (res["swaps"], res["kept_before"], res["kept_after"]) == (swaps_o, before_o, after_o)
    assert np.array_equal(perm_g, perm_o)
    if max_swaps is None:
        assert swaps_o > 0 or k == 4


@pytest.mark.parametrize("limit", [0, 1, 2, 3])
def test_search_stops_after_max_swaps(limit):
    w = I.channel_scaled_bf16((96, 48), 0.02, 77)
    q, perm_o, swaps_o, before_o, after_o = run_oracle(w, 2, None, limit)
    perm_g, res = run_gpu(w, 2, None, limit)
    assert res["swaps"] == swaps_o == limit
    assert (res["kept_before"], res["kept_after"]) == (before_o, after_o)
    assert np.array_equal(perm_g, perm_o)


def test_search_hand_examples():
    # the two worked cases of the oracle pins, through the CUDA path
    w = torch.tensor([[9, 9, 9, 9, 0, 0, 0, 0]], dtype=torch.bfloat16)
    perm, res = run_gpu(w, 2)
    assert perm.tolist() == [4, 5, 2, 3, 0, 1, 6, 7]
    assert res == {"swaps": 2, "kept_before": 2 * 2 ** 24, "kept_after": 4 * 2 ** 24}
    w = torch.tensor([[4, 3, 2, 1, 8, 7, 6, 5]], dtype=torch.bfloat16)
    perm, res = run_gpu(w, 3)
    assert perm.tolist() == [0, 1, 4, 3, 2, 5, 6, 7]
    assert res == {"swaps": 1, "kept_before": 30 * 2 ** 21, "kept_after": 33 * 2 ** 21}


@pytest.mark.parametrize("kind", ["one_group", "zeros", "constant", "nonfinite"])
def test_search_degenerate_inputs(kind):
    if kind == "one_group":
        w = I.normal_bf16((20, 4), 1.0, 3)
    elif kind == "zeros":
        w = torch.zeros((16, 32), dtype=torch.bfloat16)
    elif kind == "constant":
        w = torch.full((16, 32), -0.5, dtype=torch.bfloat16)
    else:
        w = I.channel_scaled_bf16((24, 32), 0.02, 9)
        w[3, 5] = float("nan")
        w[7, 20] = float("inf")
        w[9, 1] = float("-inf")
    q, perm_o, swaps_o, before_o, after_o = run_oracle(w, 2)
    perm_g, res = run_gpu(w, 2)
    assert np.array_equal(perm_g, perm_o)
    assert (res["swaps"], res["kept_before"], res["kept_after"]) == (swaps_o, before_o, after_o)
    if kind != "nonfinite":
        assert res["swaps"] == 0 and perm_g.tolist() == list(range(w.shape[1]))


@pytest.mark.parametrize("n,k,limit", [(3072, 768, None), (4096, 4096, 300)])
def test_search_full_size_properties(n, k, limit):
    w = I.channel_scaled_bf16((n, k), 0.02, 5)
    wd = w.cuda()
    cap = 64 * k if limit is None else limit   # bounds the run if the search never stopped
    P.permute_search(wd, 2, None, 1)          # warm-up (first-call set-up)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    perm_t, res = P.permute_search(wd, 2, None, cap)
    dt = time.perf_counter() - t0
    assert B.sp24_device_status() == B.SP24_OK
    perm = perm_t.cpu().numpy().astype(np.int64)
    print(f"\npermute_search {n}x{k}: {res['swaps']} swaps in {dt * 1e3:.1f} ms "
          f"({dt / max(res['swaps'], 1) * 1e6:.1f} us/swap); kept "
          f"{res['kept_before']} -> {res['kept_after']} "
          f"(+{100.0 * (res['kept_after'] / res['kept_before'] - 1):.3f} %)")
    assert sorted(perm.tolist()) == list(range(k))
    q = O.permutation_scores(f64(w), O.MAGNITUDE)
    assert res["kept_before"] == O.kept_score(q, np.arange(k), 2)
    assert res["kept_after"] == O.kept_score(q, perm, 2)
    assert res["kept_after"] - res["kept_before"] >= res["swaps"] > 0
    if limit is None:
        assert res["swaps"] < cap
        rng = np.random.default_rng(1)
        pos = np.argsort(perm)
        checked = 0
        while checked < 200:
            a, b = (int(v) for v in rng.integers(0, k, size=2))
            if pos[a] // 4 == pos[b] // 4:
                continue
            assert O.swap_gain(q, perm, a, b, 2) <= 0
            checked += 1
    else:
        assert res["swaps"] == limit


@pytest.mark.parametrize("dtype,rows,k", [(torch.bfloat16, 37, 100), (torch.int8, 64, 4096),
                                          (torch.float32, 5, 12), (torch.bfloat16, 4096, 768)])
def test_permute_columns_bit_exact(dtype, rows, k):
    g = torch.Generator().manual_seed(rows + k)
    if dtype == torch.int8:
        a = torch.randint(-128, 128, (rows, k), generator=g, dtype=torch.int8)
    else:
        a = torch.randn((rows, k), generator=g).to(dtype)
    perm = torch.randperm(k, generator=g).to(torch.int32)
    out = P.permute_columns(a.cuda(), perm.cuda()).cpu()
    assert B.sp24_device_status() == B.SP24_OK
    want = O.permute_columns(a.view(torch.uint8 if dtype == torch.int8 else
                                    (torch.int16 if dtype == torch.bfloat16 else torch.int32)
                                    ).numpy(), perm.numpy())
    got = out.view(torch.uint8 if dtype == torch.int8 else
                   (torch.int16 if dtype == torch.bfloat16 else torch.int32)).numpy()
    assert np.array_equal(got, want)


def test_permute_columns_bad_index_reports_and_zeroes():
    a = torch.ones((3, 8), dtype=torch.bfloat16, device="cuda")
    perm = torch.tensor([0, 1, 2, 3, 4, 5, 6, 8], dtype=torch.int32, device="cuda")
    out = P.permute_columns(a, perm)
    assert B.sp24_device_status() == B.SP24_ERR_INDEX
    assert B.sp24_device_status() == B.SP24_OK          # cleared
    assert (out[:, :7] == 1).all() and (out[:, 7] == 0).all()


def test_permuted_layer_prunes_and_multiplies_like_the_oracle():
    # search -> gather W and X -> prune -> compress -> GEMM; Y matches the
    # unpermuted product of the pruned weights, and the mask of the permuted
    # weights is the oracle's mask of the oracle's permuted weights.
    n, k, m = 128, 64, 96
    w = I.channel_scaled_bf16((n, k), 0.02, 21)
    x = I.normal_bf16((m, k), 1.0, 22)
    q, perm_o, *_ = run_oracle(w, 2)
    perm_g, _ = P.permute_search(w.cuda(), 2, None, 1 << 20)
    assert np.array_equal(perm_g.cpu().numpy(), perm_o)
    wp = P.permute_columns(w.cuda(), perm_g)
    xp = P.permute_columns(x.cuda(), perm_g)
    vals, meta, mask = P.prune_compress(wp, B.SP24_MAGNITUDE, want_mask=True)
    y = P.gemm(xp, vals, meta, n)
    assert B.sp24_device_status() == B.SP24_OK
    wpo = O.permute_columns(f64(w), perm_o)
    keep = O.prune(wpo, O.MAGNITUDE, 2)
    assert np.array_equal(O.unpack_mask(mask.cpu().numpy(), k), keep)
    xpo = O.permute_columns(f64(x), perm_o)
    wm = np.where(keep, wpo, 0.0)
    y_ref = xpo @ wm.T
    a_ref = np.abs(xpo) @ np.abs(wm).T
    assert (np.abs(f64(y) - y_ref) <= 8e-3 * a_ref).all()
    # the permuted layer keeps at least the kept magnitude of the plain one
    keep0 = O.prune(f64(w), O.MAGNITUDE, 2)
    assert np.abs(wpo)[keep].sum() >= np.abs(f64(w))[keep0].sum()
