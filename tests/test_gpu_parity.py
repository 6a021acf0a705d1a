"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bars: masks, metadata, int8 values, int32 accumulators, dequantised bf16 and
requantised int8 outputs are bit-exact; the bf16 GEMM satisfies, per element,
|y_gpu - y_ref| <= 8e-3 * sum_k |x_k * w_k| (y_ref and the bound in float64).
Inputs are the seeded workloads of structured_sparse_gemm_sp24_b200.inputs.
"""
import numpy as np
import pytest
import torch

from oracle import sp24_oracle as O
from structured_sparse_gemm_sp24_b200 import inputs as I
from structured_sparse_gemm_sp24_b200 import pipeline as P
from structured_sparse_gemm_sp24_b200 import sp24 as B
from tests import meta_layout as L

pytestmark = pytest.mark.gpu

TOL = 8e-3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    B.lib()
    assert B.sp24_device_status() == B.SP24_OK


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def keep_of(mask_dev: torch.Tensor, k: int) -> np.ndarray:
    return O.unpack_mask(mask_dev.cpu().numpy(), k)


def canon_meta(meta_dev, n, k, dtype):
    return L.decode(meta_dev.cpu().numpy(), n, k, dtype)


def assert_bf16_close(y_dev, y_ref, a_ref):
    y = f64(y_dev)
    d = np.abs(y - y_ref)
    ok = d <= TOL * a_ref
    if not ok.all():
        i = np.argwhere(~ok)[0]
        raise AssertionError(
            f"bf16 GEMM off at {tuple(i)}: gpu={y[tuple(i)]} ref={y_ref[tuple(i)]} "
            f"bound={TOL * a_ref[tuple(i)]} ({(~ok).sum()} of {ok.size} elements)")
    return float((d / np.where(a_ref > 0, a_ref, 1)).max())


def ok_status():
    assert B.sp24_device_status() == B.SP24_OK


# ------------------------------------------------------------------ a1
def test_colnorm_bert_calibration():
    w = I.bert_fc1()
    n = P.colnorm(w.Xc.cuda())
    assert np.array_equal(n.cpu().numpy(), O.column_norms(f64(w.Xc)))
    ok_status()


def test_colnorm_sums_in_token_order():
    xc = torch.zeros((33, 16), dtype=torch.bfloat16)
    xc[:32, 0] = 2.0 ** -27
    xc[32, 0] = 1.0
    xc[0, 8] = 1.0
    xc[1:, 8] = 2.0 ** -27
    n = P.colnorm(xc.cuda()).cpu().numpy()
    assert n[0] == 1.0 + 2.0 ** -50 and n[8] == 1.0
    assert np.array_equal(n, O.column_norms(f64(xc)))


# ------------------------------------------------------------------ a2/a3
PRUNE_SHAPES = [(64, 128, 1.0), (3072, 768, 0.02), (200, 136, 0.02), (1, 8, 1.0), (130, 264, 1.0)]


@pytest.mark.parametrize("n_keep", [2, 3])
@pytest.mark.parametrize("shape", PRUNE_SHAPES)
def test_prune_magnitude(shape, n_keep):
    n, k, sigma = shape
    w = I.normal_bf16((n, k), sigma, seed=11)
    mask = P.prune(w.cuda(), B.SP24_MAGNITUDE, n_keep)
    assert np.array_equal(keep_of(mask, k), O.prune(f64(w), O.MAGNITUDE, n_keep))
    ok_status()


def test_prune_ties_heavy():
    # a 5-value alphabet makes ties common; -0.0 and +0.0 both appear
    g = torch.Generator().manual_seed(5)
    w = (torch.randint(-2, 3, (257, 512), generator=g).float() * 0.5).to(torch.bfloat16)
    w[0, :4] = torch.tensor([0.0, -0.0, 0.0, -0.0])
    for n_keep in (2, 3):
        mask = P.prune(w.cuda(), B.SP24_MAGNITUDE, n_keep)
        assert np.array_equal(keep_of(mask, 512), O.prune(f64(w), O.MAGNITUDE, n_keep))


@pytest.mark.parametrize("n_keep", [2, 3])
def test_prune_wanda_bert(n_keep):
    w = I.bert_fc1()
    mask = P.prune(w.W.cuda(), B.SP24_WANDA, n_keep, Xc=w.Xc.cuda())
    ref = O.prune(f64(w.W), O.WANDA, n_keep, xc=f64(w.Xc))
    assert np.array_equal(keep_of(mask, w.K), ref)


@pytest.mark.parametrize("n,k,mc", [(130, 264, 37), (3072, 768, 128), (9000, 256, 128)])
def test_prune_wanda_norm_paths(n, k, mc):
    # small row-tiles x Mc: norms formed inside the prune kernel; large (the
    # last case: 71 row tiles x 128): separate column-norm kernel.  Either way
    # the mask matches and the workspace holds the norms afterwards.
    W = I.normal_bf16((n, k), 0.02, seed=91)
    Xc = I.normal_bf16((mc, k), 1.0, seed=92)
    out = torch.empty((n, k // 8), dtype=torch.uint8, device="cuda")
    ws = torch.full((B.sp24_prune_workspace_bytes(k, B.SP24_WANDA),), 0xAB, dtype=torch.uint8,
                    device="cuda")
    B.sp24_prune(W.cuda(), Xc.cuda(), B.SP24_WANDA, 2, None, out, ws)
    ok_status()
    assert np.array_equal(keep_of(out, k), O.prune(f64(W), O.WANDA, 2, xc=f64(Xc)))
    norms = ws[: 8 * k].view(torch.float64).cpu().numpy()
    assert np.array_equal(norms, O.column_norms(f64(Xc)))


def test_progressive_bert():
    w = I.bert_fc1()
    Wd, Xc = w.W.cuda(), w.Xc.cuda()
    m1 = P.prune(Wd, B.SP24_WANDA, 3, Xc=Xc)
    m2 = P.prune(Wd, B.SP24_WANDA, 2, Xc=Xc, mask_in=m1)
    r1, r2 = O.progressive(f64(w.W), O.WANDA, f64(w.Xc))
    assert np.array_equal(keep_of(m1, w.K), r1)
    assert np.array_equal(keep_of(m2, w.K), r2)


# (N, K, Mc): fused-norm path (BERT fc1), ragged K tail with a partial row
# tile, and the separate column-norm kernel (82 row tiles x 128 rows > 8192)
PROGRESSIVE_SHAPES = [(3072, 768, 128), (200, 136, 37), (10400, 256, 128)]


@pytest.mark.parametrize("mode", [B.SP24_WANDA, B.SP24_MAGNITUDE])
@pytest.mark.parametrize("nkm", PROGRESSIVE_SHAPES)
def test_prune_progressive_one_pass(mode, nkm):
    # one pass: mask1 (3 of 4), mask2 (2 of 4 on W * mask1), bf16 values and
    # metadata of mask2, bit for bit against the oracle's two-stage definition
    n, k, mc = nkm
    W = I.normal_bf16((n, k), 0.02, seed=61)
    Xc = I.normal_bf16((mc, k), 1.0, seed=62)
    xc = Xc.cuda() if mode == B.SP24_WANDA else None
    omode = O.WANDA if mode == B.SP24_WANDA else O.MAGNITUDE
    r1, r2 = O.progressive(f64(W), omode, f64(Xc) if mode == B.SP24_WANDA else None)
    compress = k % 16 == 0
    m1, m2, vals, meta = P.prune_progressive(W.cuda(), mode, xc, compress=compress)
    ok_status()
    assert np.array_equal(keep_of(m1, k), r1)
    assert np.array_equal(keep_of(m2, k), r2)
    if compress:
        rv, rm = O.compress(f64(W), r2)
        assert np.array_equal(f64(vals), rv)
        assert np.array_equal(canon_meta(meta, n, k, L.BF16), rm)
    # masks only, one output at a time
    m1b = torch.empty_like(m1)
    ws = torch.empty(max(B.sp24_prune_workspace_bytes(k, mode), 16), dtype=torch.uint8,
                     device="cuda")
    B.sp24_prune_progressive(W.cuda(), xc, mode, m1b, None, None, None, ws)
    assert torch.equal(m1b, m1)
    if mode == B.SP24_WANDA:   # the workspace holds the column norms afterwards
        assert np.array_equal(ws[: 8 * k].view(torch.float64).cpu().numpy(), O.column_norms(f64(Xc)))


def test_prune_progressive_then_int8_compress():
    # the progressive masks feed the INT8 path: scales over the 2:4 mask, int8
    # values and metadata bit for bit
    w = I.int8_long_tail(M=16)
    Wd = w.W.cuda()
    m1, m2, _, _ = P.prune_progressive(Wd, B.SP24_MAGNITUDE, None, compress=False)
    s_w = P.wscale(Wd, m2)
    vals, meta = P.compress(Wd, m2, B.SP24_INT8, s_w)
    ok_status()
    r1, r2 = O.progressive(f64(w.W), O.MAGNITUDE)
    assert np.array_equal(keep_of(m1, w.K), r1) and np.array_equal(keep_of(m2, w.K), r2)
    rs = O.channel_scales(f64(w.W), r2)
    assert np.array_equal(s_w.cpu().numpy(), rs)
    rv, rm = O.compress(O.quantize(f64(w.W), rs[:, None]), r2)
    assert np.array_equal(vals.cpu().numpy(), rv)
    assert np.array_equal(canon_meta(meta, w.N, w.K, L.INT8), rm)


def test_prune_llm_full():
    w = I.llm_proj(11008, 4096, 16)
    mask = P.prune(w.W.cuda(), B.SP24_MAGNITUDE, 2)
    assert np.array_equal(keep_of(mask, 4096), O.prune(f64(w.W), O.MAGNITUDE, 2))


# ------------------------------------------------------------------ a4
COMPRESS_SHAPES = [(64, 128), (200, 160), (3072, 768), (8, 32), (129, 288)]


@pytest.mark.parametrize("shape", COMPRESS_SHAPES)
def test_compress_bf16(shape):
    n, k = shape
    w = I.normal_bf16((n, k), 1.0, seed=3)
    wd = w.cuda()
    mask = P.prune(wd, B.SP24_MAGNITUDE, 2)
    vals, meta = P.compress(wd, mask, B.SP24_BF16)
    keep = O.prune(f64(w), O.MAGNITUDE, 2)
    rv, rm = O.compress(f64(w), keep)
    assert np.array_equal(f64(vals), rv)
    assert np.array_equal(canon_meta(meta, n, k, L.BF16), rm)
    assert L.padding_is_valid(meta.cpu().numpy(), n, k, L.BF16)
    ok_status()


@pytest.mark.parametrize("shape", COMPRESS_SHAPES)
def test_compress_int8(shape):
    n, k = shape
    w = I.long_tail_bf16((n, k), 0.02, seed=4, tail_seed=7)
    wd = w.cuda()
    mask = P.prune(wd, B.SP24_MAGNITUDE, 2)
    s_w = P.wscale(wd, mask)
    vals, meta = P.compress(wd, mask, B.SP24_INT8, s_w)
    keep = O.prune(f64(w), O.MAGNITUDE, 2)
    rs = O.channel_scales(f64(w), keep)
    assert np.array_equal(s_w.cpu().numpy(), rs)
    wq = O.quantize(f64(w), rs[:, None])
    rv, rm = O.compress(wq, keep)
    assert np.array_equal(vals.cpu().numpy(), rv)
    assert np.array_equal(canon_meta(meta, n, k, L.INT8), rm)
    assert L.padding_is_valid(meta.cpu().numpy(), n, k, L.INT8)
    ok_status()


@pytest.mark.parametrize("case", [("int8_workload", 0.9999), ((130, 256), 0.5), ((1, 32), 0.9999),
                                  ((200, 4128), 0.9999), ((257, 1056), 0.9), ((64, 512), 1.0)])
def test_prune_compress_int8_one_pass(case):
    # the one-pass INT8 weight conversion against the three kernels it
    # replaces (every byte, metadata padding included) and the oracle
    shape, cov = case
    if shape == "int8_workload":
        w = I.int8_long_tail().W                      # 4096 x 4096, 1 % long tail
    else:
        w = I.long_tail_bf16(shape, 0.02, seed=5, tail_seed=8)
    n, k = w.shape
    wd = w.cuda()
    vals, meta, s_w, mask = P.prune_compress_int8(wd, cov, want_mask=True)
    ok_status()
    m3 = P.prune(wd, B.SP24_MAGNITUDE, 2)
    s3 = P.wscale(wd, m3, cov)
    v3, t3 = P.compress(wd, m3, B.SP24_INT8, s3)
    assert torch.equal(mask, m3) and torch.equal(s_w, s3)
    assert torch.equal(vals, v3) and torch.equal(meta, t3)
    keep = O.prune(f64(w), O.MAGNITUDE, 2)
    rs = O.channel_scales(f64(w), keep, cov)
    assert np.array_equal(keep_of(mask, k), keep)
    assert np.array_equal(s_w.cpu().numpy(), rs)
    rv, rm = O.compress(O.quantize(f64(w), rs[:, None]), keep)
    assert np.array_equal(vals.cpu().numpy(), rv)
    assert np.array_equal(canon_meta(meta, n, k, L.INT8), rm)
    assert L.padding_is_valid(meta.cpu().numpy(), n, k, L.INT8)
    ok_status()


@pytest.mark.parametrize("dtype", [B.SP24_BF16, B.SP24_INT8])
@pytest.mark.parametrize("mode", [B.SP24_MAGNITUDE, B.SP24_WANDA])
def test_prune_compress_fused(mode, dtype):
    w = I.bert_fc1()
    Wd, Xc = w.W.cuda(), w.Xc.cuda()
    m1 = P.prune(Wd, mode, 3, Xc=Xc)
    norms = P.colnorm(Xc) if mode == B.SP24_WANDA else None
    s_w = None
    if dtype == B.SP24_INT8:
        s_w = P.wscale(Wd, P.prune(Wd, mode, 2, Xc=Xc, mask_in=m1))
    vals, meta, mask = P.prune_compress(Wd, mode, norms, m1, dtype, s_w, want_mask=True)
    omode = O.WANDA if mode == B.SP24_WANDA else O.MAGNITUDE
    r1 = O.prune(f64(w.W), omode, 3, xc=f64(w.Xc))
    keep = O.prune(f64(w.W), omode, 2, xc=f64(w.Xc), mask_in=r1)
    assert np.array_equal(keep_of(mask, w.K), keep)
    if dtype == B.SP24_BF16:
        rv, rm = O.compress(f64(w.W), keep)
        assert np.array_equal(f64(vals), rv)
    else:
        rs = O.channel_scales(f64(w.W), keep)
        rv, rm = O.compress(O.quantize(f64(w.W), rs[:, None]), keep)
        assert np.array_equal(vals.cpu().numpy(), rv)
    ldt = L.BF16 if dtype == B.SP24_BF16 else L.INT8
    assert np.array_equal(canon_meta(meta, w.N, w.K, ldt), rm)
    ok_status()


def test_compress_rejects_bad_pattern():
    w = I.normal_bf16((64, 128), 1.0, seed=1).cuda()
    mask = P.prune(w, B.SP24_MAGNITUDE, 2)
    ok_status()
    bad = mask.clone()
    bad[5, 3] = 0x7F          # groups keeping 3 and 4 positions
    P.compress(w, bad, B.SP24_BF16)
    assert B.sp24_device_status() == B.SP24_ERR_PATTERN
    ok_status()               # reading the status cleared it
    m3 = P.prune(w, B.SP24_MAGNITUDE, 3)
    P.compress(w, m3, B.SP24_BF16)
    assert B.sp24_device_status() == B.SP24_ERR_PATTERN


# ------------------------------------------------------------------ a5
def test_wscale_long_tail_full():
    w = I.int8_long_tail()
    wd = w.W.cuda()
    mask = P.prune(wd, B.SP24_MAGNITUDE, 2)
    keep = keep_of(mask, w.K)
    assert np.array_equal(P.wscale(wd, mask).cpu().numpy(), O.channel_scales(f64(w.W), keep))


@pytest.mark.parametrize("coverage", [0.9, 0.5, 1.0, 1e-9])
def test_wscale_ranks_below_max(coverage):
    w = I.normal_bf16((300, 4096), 0.02, seed=9)
    w[7] = 0.0                                   # zero row -> scale 1
    wd = w.cuda()
    for n_keep in (2, 3):
        mask = P.prune(wd, B.SP24_MAGNITUDE, n_keep)
        got = P.wscale(wd, mask, coverage).cpu().numpy()
        ref = O.channel_scales(f64(w), keep_of(mask, 4096), coverage)
        assert np.array_equal(got, ref)
        assert got[7] == 1.0


@pytest.mark.parametrize("count", [1, 17, 4096, 1000003])
def test_act_scale_and_quantize_small(count):
    x = I.normal_f32((count,), 1.0, seed=count)
    xd = x.cuda()
    s = P.act_scale(xd)
    rs = O.tensor_scale(x.numpy())
    assert s.item() == rs
    q = P.quantize(xd, s)
    assert np.array_equal(q.cpu().numpy(), O.quantize(x.numpy(), rs))


def _act_inputs(kind, count, seed):
    x = I.normal_f32((count,), 1.0, seed=seed).numpy()
    if kind == "ties":          # coarse values: thousands of equal keys at the quantile
        x = np.round(x * 4.0) / 4.0
    elif kind == "outlier_cols":  # a few "channels" of a 1024-wide matrix carry x50 outliers
        body = x[: (count // 1024) * 1024].reshape(-1, 1024)   # a view into x
        body[:, [3, 517, 1000]] *= 50.0
    elif kind == "zeros":       # mostly exact zeros (ReLU-like), a sparse positive tail
        x = np.where(x > 2.5, x, 0.0).astype(np.float32)
    elif kind == "constant":    # one key everywhere but 8 outliers: more equal candidates
        x = np.full(count, 0.75, dtype=np.float32)   # than the bracket list holds, so the
        x[np.arange(8) * (count // 8)] = 9.0          # exact radix fallback decides
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))


@pytest.mark.parametrize("kind", ["normal", "ties", "outlier_cols", "zeros", "constant"])
@pytest.mark.parametrize("coverage", [0.5, 0.9, 0.9999, 1.0])
def test_act_scale_large_coverages(kind, coverage):
    # >= 2^18 elements take the sampled-bracket path; central coverages, heavy
    # ties and column-structured outliers exercise its exact fallback
    x = _act_inputs(kind, (1 << 20) + 12, seed=77)
    s = P.act_scale(x.cuda(), coverage)
    assert s.item() == O.tensor_scale(x.numpy(), coverage)
    ok_status()


@pytest.mark.parametrize("scale", [0.25, 0.0123457, 3.0])
def test_quantize_half_integer_ties(scale):
    # quotients at, and one float step either side of, every half-integer up
    # to the clamp (rint: ties to even), plus values beyond the clamp
    s = np.float32(scale)
    halves = (np.arange(-140, 141, dtype=np.float64) + 0.5)
    x = (halves * np.float64(s)).astype(np.float32)
    near = np.concatenate([x, np.nextafter(x, np.float32(np.inf)),
                           np.nextafter(x, np.float32(-np.inf)),
                           np.array([1e30, -1e30, 0.0, -0.0], dtype=np.float32)])
    xd = torch.from_numpy(near).cuda()
    sd = torch.tensor([s, 0, 0, 0], dtype=torch.float32, device="cuda")[:1]
    q = P.quantize(xd, sd)
    assert np.array_equal(q.cpu().numpy(), O.quantize(near, s))


def test_act_scale_and_quantize_int8_workload():
    w = I.int8_long_tail()
    xd = w.X.cuda()
    s = P.act_scale(xd)
    rs = O.tensor_scale(w.X.numpy())
    assert s.item() == rs
    q = P.quantize(xd, s)
    rows = np.arange(0, w.M, 97)
    assert np.array_equal(q.cpu().numpy()[rows], O.quantize(w.X.numpy()[rows], rs))


# ------------------------------------------------------------------ a6 bf16
def _bf16_pipeline(W, X, mode=B.SP24_MAGNITUDE, Xc=None):
    Wd = W.cuda()
    mask = P.prune(Wd, mode, 2, Xc=None if Xc is None else Xc.cuda())
    vals, meta = P.compress(Wd, mask, B.SP24_BF16)
    y = P.gemm(X.cuda(), vals, meta, W.shape[0])
    return mask, vals, meta, y


def _bf16_ref(W, X, rows=None, mode=O.MAGNITUDE, Xc=None):
    keep = O.prune(f64(W), mode, 2, xc=None if Xc is None else f64(Xc))
    vals, meta = O.compress(f64(W), keep)
    x = f64(X) if rows is None else f64(X[rows])
    return O.gemm(x, vals, meta, W.shape[1])


GEMM_SHAPES = [
    # (M, N, K): several tiles, ragged tails in every dimension, minimal sizes
    (16, 64, 128), (77, 72, 144), (1, 8, 16), (130, 136, 272), (300, 256, 512),
    (33, 384, 1024), (64, 128, 256), (5, 11008, 256), (129, 4096, 384),
    # persistent path (>= 2 tiles per SM, or a single K block), ragged M, N, K
    (2500, 2056, 400), (300, 256, 128), (4099, 1032, 784),
    # persistent path with N < 128 (store box narrower than a tile)
    (300, 24, 128), (1000, 40, 96),
]


@pytest.mark.parametrize("mnk", GEMM_SHAPES)
def test_gemm_bf16_shapes(mnk):
    m, n, k = mnk
    W = I.normal_bf16((n, k), 1.0, seed=21)
    X = I.normal_bf16((m, k), 1.0, seed=22)
    _, _, _, y = _bf16_pipeline(W, X)
    yr, ar = _bf16_ref(W, X)
    assert_bf16_close(y, yr, ar)
    ok_status()


def test_gemm_bf16_tiny_config():
    w = I.tiny()
    _, _, _, y = _bf16_pipeline(w.W, w.X)
    assert_bf16_close(y, *_bf16_ref(w.W, w.X))


def test_gemm_bf16_bert_full():
    w = I.bert_fc1()
    Wd, Xc = w.W.cuda(), w.Xc.cuda()
    m1 = P.prune(Wd, B.SP24_WANDA, 3, Xc=Xc)
    m2 = P.prune(Wd, B.SP24_WANDA, 2, Xc=Xc, mask_in=m1)
    vals, meta = P.compress(Wd, m2, B.SP24_BF16)
    y = P.gemm(w.X.cuda(), vals, meta, w.N)
    keep = O.progressive(f64(w.W), O.WANDA, f64(w.Xc))[1]
    rv, rm = O.compress(f64(w.W), keep)
    assert_bf16_close(y, *O.gemm(f64(w.X), rv, rm, w.K))


@pytest.mark.parametrize("nk", I.LLM_SHAPES)
@pytest.mark.parametrize("m", I.LLM_M)
def test_gemm_bf16_llm(nk, m):
    n, k = nk
    w = I.llm_proj(n, k, m)
    mask, vals, meta, y = _bf16_pipeline(w.W, w.X)
    # every output element against the float64 product (and the mask and
    # metadata bit for bit)
    keep = O.prune(f64(w.W), O.MAGNITUDE, 2)
    assert np.array_equal(keep_of(mask, k), keep)
    rv, rm = O.compress(f64(w.W), keep)
    assert np.array_equal(canon_meta(meta, n, k, L.BF16), rm)
    assert_bf16_close(y, *O.gemm(f64(w.X), rv, rm, k))


def test_gemm_bf16_conv1x1_full():
    w = I.conv1x1()
    _, _, _, y = _bf16_pipeline(w.W, w.X)
    assert_bf16_close(y, *_bf16_ref(w.W, w.X))


@pytest.mark.parametrize("n", [1024, 2048, 4096, 8192])
def test_gemm_bf16_square(n):
    w = I.square(n)
    _, _, _, y = _bf16_pipeline(w.W, w.X)
    assert_bf16_close(y, *_bf16_ref(w.W, w.X))


@pytest.mark.parametrize("n", [16384])
def test_gemm_bf16_square_sampled_large(n):
    # the largest configured size: the whole pipeline runs on the GPU;
    # sampled weight rows (pruning is row-independent) are pruned by the
    # oracle, their masks compared bit for bit, and the outputs of sampled
    # tokens x those channels checked against the float64 product
    w = I.square(n)
    mask, _, _, y = _bf16_pipeline(w.W, w.X)
    ok_status()
    cols = np.unique(np.r_[0:24, n - 24:n, 777:n:1999])
    rows = np.unique(np.r_[0:16, n - 16:n, 100:n:2011])
    Wc = w.W[torch.from_numpy(cols)]
    keep = O.prune(f64(Wc), O.MAGNITUDE, 2)
    assert np.array_equal(keep_of(mask[torch.from_numpy(cols).cuda()], n), keep)
    vals, meta = O.compress(f64(Wc), keep)
    yr, ar = O.gemm(f64(w.X[torch.from_numpy(rows)]), vals, meta, n)
    got = y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()]
    assert_bf16_close(got, yr, ar)


def test_gemm_bf16_deterministic_split():
    for n, k in [(4096, 11008), (11008, 4096)]:     # split-K over a cluster (the second
        w = I.llm_proj(n, k, 16)                    # with CTAs sharing SMs)
        _, vals, meta, y1 = _bf16_pipeline(w.W, w.X)
        y2 = P.gemm(w.X.cuda(), vals, meta, w.N)
        assert torch.equal(y1, y2)


def test_compressed_weight_file_round_trip(tmp_path):
    # compress once, save, load back onto the device: the GEMM on the loaded
    # weight gives the same bits (bf16) and the same accumulators (int8)
    from structured_sparse_gemm_sp24_b200 import artifact as A
    w = I.llm_proj(1024, 2048, 64)
    Wd, Xd = w.W.cuda(), w.X.cuda()
    vals, meta = P.prune_compress(Wd)
    A.save_compressed(str(tmp_path / "w.sp24"), vals, meta, w.N, w.K, B.SP24_BF16)
    cw = A.load_compressed(str(tmp_path / "w.sp24"), "cuda")
    assert torch.equal(P.gemm(Xd, cw.vals, cw.meta, cw.n), P.gemm(Xd, vals, meta, w.N))
    v8, m8, s_w = P.prune_compress_int8(Wd)
    A.save_compressed(str(tmp_path / "w8.sp24"), v8, m8, w.N, w.K, B.SP24_INT8, s_w)
    c8 = A.load_compressed(str(tmp_path / "w8.sp24"), "cuda")
    xf = I.normal_f32((64, w.K), 1.0, seed=9).cuda()
    s_x = P.act_scale(xf)
    xq = P.quantize(xf, s_x)
    a = P.gemm(xq, c8.vals, c8.meta, c8.n, B.SP24_INT8, s_x, c8.s_w, B.SP24_OUT_INT32)
    b = P.gemm(xq, v8, m8, w.N, B.SP24_INT8, s_x, s_w, B.SP24_OUT_INT32)
    assert torch.equal(a, b)
    ok_status()


def test_gemm_empty_is_noop():
    W = I.normal_bf16((64, 128), 1.0, seed=1).cuda()
    mask = P.prune(W, B.SP24_MAGNITUDE, 2)
    vals, meta = P.compress(W, mask)
    y = P.gemm(torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"), vals, meta, 64)
    assert y.shape == (0, 64)
    ok_status()


# ------------------------------------------------------------------ a7 int8
def _int8_pipeline(W, X32, out_kind, s_y=None):
    Wd = W.cuda()
    mask = P.prune(Wd, B.SP24_MAGNITUDE, 2)
    s_w = P.wscale(Wd, mask)
    vals, meta = P.compress(Wd, mask, B.SP24_INT8, s_w)
    xd = X32.cuda()
    s_x = P.act_scale(xd)
    xq = P.quantize(xd, s_x)
    sy = None if s_y is None else torch.tensor([s_y], dtype=torch.float32, device="cuda")
    y = P.gemm(xq, vals, meta, W.shape[0], B.SP24_INT8, s_x, s_w, out_kind, sy)
    return y, s_x.item(), s_w.cpu().numpy()


def _int8_ref(W, X32, rows=None):
    keep = O.prune(f64(W), O.MAGNITUDE, 2)
    s_w = O.channel_scales(f64(W), keep)
    vq, meta = O.compress(O.quantize(f64(W), s_w[:, None]), keep)
    s_x = O.tensor_scale(X32.numpy())
    x = X32.numpy() if rows is None else X32.numpy()[rows]
    acc = O.gemm_int8_acc(O.quantize(x, s_x), vq, meta, W.shape[1])
    return acc, s_x, s_w


INT8_SHAPES = [(16, 64, 128), (77, 72, 160), (1, 8, 32), (130, 136, 288), (300, 256, 512),
               (16, 11008, 4096), (128, 4096, 1024),
               # persistent path, ragged M, N, K
               (2500, 2056, 416), (300, 256, 224), (300, 40, 224), (300, 48, 224)]


@pytest.mark.parametrize("mnk", INT8_SHAPES)
def test_gemm_int8_shapes(mnk):
    m, n, k = mnk
    W = I.long_tail_bf16((n, k), 0.02, seed=31, tail_seed=34)
    X = I.normal_f32((m, k), 1.0, seed=32)
    acc, s_x, s_w = _int8_ref(W, X)
    y32, gx, gw = _int8_pipeline(W, X, B.SP24_OUT_INT32)
    assert gx == s_x and np.array_equal(gw, s_w)
    assert np.array_equal(y32.cpu().numpy(), acc)
    ybf, _, _ = _int8_pipeline(W, X, B.SP24_OUT_BF16)
    ref_bits = O.dequant_bf16(acc, s_x, s_w)
    assert np.array_equal(ybf.view(torch.int16).cpu().numpy().view(np.uint16), ref_bits)
    if n % 16:
        # int8 rows of N bytes must stay 16-byte aligned
        with pytest.raises(B.Sp24Error) as e:
            _int8_pipeline(W, X, B.SP24_OUT_INT8, s_y=0.05)
        assert e.value.status == B.SP24_ERR_ALIGN
    else:
        y8, _, _ = _int8_pipeline(W, X, B.SP24_OUT_INT8, s_y=0.05)
        assert np.array_equal(y8.cpu().numpy(), O.requant_int8(acc, s_x, s_w, np.float32(0.05)))
    ok_status()


def test_gemm_int8_full_config():
    # every one of the 8192 x 4096 outputs, bit for bit.  The oracle's int64
    # product (gemm_int8_acc) is too slow at this size, so the accumulators
    # are formed as a float64 product of the oracle's int8 operands: every
    # partial sum is an integer below 2^31 in magnitude, exact in float64.
    # The two agree exactly on a slice of rows (checked here), then the full
    # float64 product is the reference.
    w = I.int8_long_tail()
    keep = O.prune(f64(w.W), O.MAGNITUDE, 2)
    s_w = O.channel_scales(f64(w.W), keep)
    vq, meta = O.compress(O.quantize(f64(w.W), s_w[:, None]), keep)
    s_x = O.tensor_scale(w.X.numpy())
    xq = O.quantize(w.X.numpy(), s_x)
    wd = O.decompress(vq, meta, w.K).astype(np.float64)
    acc_f = xq.astype(np.float64) @ wd.T
    assert np.abs(acc_f).max() < 2.0 ** 31
    acc = acc_f.astype(np.int64)
    assert np.array_equal(acc[:64], O.gemm_int8_acc(xq[:64], vq, meta, w.K))
    ybf, gx, gw = _int8_pipeline(w.W, w.X, B.SP24_OUT_BF16)
    assert gx == s_x and np.array_equal(gw, s_w)
    got = ybf.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.dequant_bf16(acc, s_x, s_w))
    y32, _, _ = _int8_pipeline(w.W, w.X, B.SP24_OUT_INT32)
    assert np.array_equal(y32.cpu().numpy(), acc)
    ok_status()


# ------------------------------------------------ large-problem kernel variants
IMPL_SHAPES = [(2500, 2056, 400), (300, 256, 128), (130, 520, 96), (4099, 1032, 784),
               (200, 64, 128), (3000, 1800, 1296)]


@pytest.fixture
def gemm_impl(request, monkeypatch):
    monkeypatch.setenv("SP24_GEMM_IMPL", request.param)
    return request.param


@pytest.mark.parametrize("gemm_impl", ["single", "pair128", "pair192", "pair224", "pair240", "pair256"], indirect=True)
@pytest.mark.parametrize("mnk", IMPL_SHAPES)
def test_gemm_bf16_impls(gemm_impl, mnk):
    m, n, k = mnk
    W = I.normal_bf16((n, k), 1.0, seed=41)
    X = I.normal_bf16((m, k), 1.0, seed=42)
    _, _, _, y = _bf16_pipeline(W, X)
    assert_bf16_close(y, *_bf16_ref(W, X))
    ok_status()


@pytest.mark.parametrize("gemm_impl", ["single", "pair128", "pair192", "pair224", "pair240", "pair256"], indirect=True)
@pytest.mark.parametrize("out_kind", [B.SP24_OUT_INT32, B.SP24_OUT_BF16, B.SP24_OUT_INT8])
@pytest.mark.parametrize("mnk", [(2500, 2064, 416), (130, 528, 96 + 32), (3000, 1808, 1280)])
def test_gemm_int8_impls(gemm_impl, out_kind, mnk):
    m, n, k = mnk
    W = I.long_tail_bf16((n, k), 0.02, seed=51, tail_seed=54)
    X = I.normal_f32((m, k), 1.0, seed=52)
    acc, s_x, s_w = _int8_ref(W, X)
    y, _, _ = _int8_pipeline(W, X, out_kind, s_y=0.05)
    if out_kind == B.SP24_OUT_INT32:
        assert np.array_equal(y.cpu().numpy(), acc)
    elif out_kind == B.SP24_OUT_BF16:
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, O.dequant_bf16(acc, s_x, s_w))
    else:
        assert np.array_equal(y.cpu().numpy(), O.requant_int8(acc, s_x, s_w, np.float32(0.05)))
    ok_status()


@pytest.mark.parametrize("split", ["1", "2", "3", "4", "5", "6", "7", "8"])
@pytest.mark.parametrize("mnk", [(16, 392, 1024), (40, 264, 2048 + 128), (128, 136, 1536)])
def test_gemm_splitk_forced(split, mnk, monkeypatch):
    # every K split of the split-K kernel (the plan picks few of them)
    monkeypatch.setenv("SP24_GEMM_IMPL", "splitk")
    monkeypatch.setenv("SP24_SPLITK", split)
    m, n, k = mnk
    plan = B.sp24_gemm_plan(m, n, k, B.SP24_BF16)
    assert plan["kernel"] == "splitk" and plan["split_k"] == int(split)
    W = I.normal_bf16((n, k), 1.0, seed=61)
    X = I.normal_bf16((m, k), 1.0, seed=62)
    _, _, _, y = _bf16_pipeline(W, X)
    assert_bf16_close(y, *_bf16_ref(W, X))
    acc, s_x, s_w = _int8_ref(I.long_tail_bf16((n, k), 0.02, seed=63, tail_seed=64),
                              I.normal_f32((m, k), 1.0, seed=65))
    yi, _, _ = _int8_pipeline(I.long_tail_bf16((n, k), 0.02, seed=63, tail_seed=64),
                              I.normal_f32((m, k), 1.0, seed=65), B.SP24_OUT_INT32)
    assert np.array_equal(yi.cpu().numpy(), acc)
    ok_status()


# --------------------------------------------- split-K with CTAs sharing SMs
@pytest.mark.parametrize("case", [(16, 11008, 4096, None), (64, 11008, 4096, None),
                                  (40, 11008, 2048 + 96, None),
                                  # forced odd splits: uneven token ownership in the
                                  # cluster reduction (43/43/42 and 4/3/3/3/3 tokens)
                                  (128, 11008, 4096, "3"), (100, 11008, 1536, "3"),
                                  (16, 11008, 4096, "5")])
def test_gemm_splitk_small_ring(case, monkeypatch):
    # more split CTAs than SMs (several per SM on the small ring): bf16 within
    # the bound, int8 accumulators exact
    m, n, k, forced = case
    monkeypatch.delenv("SP24_GEMM_IMPL", raising=False)
    if forced:
        monkeypatch.setenv("SP24_SPLITK", forced)
    else:
        monkeypatch.delenv("SP24_SPLITK", raising=False)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = B.sp24_gemm_plan(m, n, k, B.SP24_BF16)
    assert plan["kernel"] == "splitk" and plan["split_k"] > 1 and plan["ctas"] > sms
    W = I.normal_bf16((n, k), 1.0, seed=66)
    X = I.normal_bf16((m, k), 1.0, seed=67)
    Wd = W.cuda()
    vals, meta = P.compress(Wd, P.prune(Wd, B.SP24_MAGNITUDE, 2), B.SP24_BF16)
    y = P.gemm(X.cuda(), vals, meta, n)
    ok_status()
    assert_bf16_close(y, *_bf16_ref(W, X))
    Wi = I.long_tail_bf16((n, k), 0.02, seed=68, tail_seed=69)
    Xi = I.normal_f32((m, k), 1.0, seed=70)
    acc, _, _ = _int8_ref(Wi, Xi)
    Wid = Wi.cuda()
    mask = P.prune(Wid, B.SP24_MAGNITUDE, 2)
    gw = P.wscale(Wid, mask)
    vq, mq = P.compress(Wid, mask, B.SP24_INT8, gw)
    xd = Xi.cuda()
    gx = P.act_scale(xd)
    y32 = P.gemm(P.quantize(xd, gx), vq, mq, n, B.SP24_INT8, gx, gw, B.SP24_OUT_INT32)
    ok_status()
    assert np.array_equal(y32.cpu().numpy(), acc)


# ------------------------------------------------------ Sparse-QAT fake quant
@pytest.mark.parametrize("case", ["int8_workload", "ragged_3of4"])
def test_fake_quant_matches_oracle(case):
    if case == "int8_workload":
        W = I.int8_long_tail().W                     # 4096 x 4096, 1 % long tail
        n_keep = 2
    else:
        W = I.normal_bf16((130, 264), 0.02, seed=81)
        n_keep = 3
    Wd = W.cuda()
    mask = P.prune(Wd, B.SP24_MAGNITUDE, n_keep)
    s_w = P.wscale(Wd, mask)
    got = P.fake_quant(Wd, mask, s_w)
    ok_status()
    keep = O.prune(f64(W), O.MAGNITUDE, n_keep)
    ref = O.fake_quant(f64(W), keep, O.channel_scales(f64(W), keep))
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), ref)


# ------------------------------------------------------------ failure path
def test_bounded_wait_reports_timeout_and_context_survives():
    assert B.sp24_device_status() == B.SP24_OK
    B.sp24_selftest_wait_timeout(20_000_000)          # 20 ms, nothing arrives
    assert B.sp24_device_status() == B.SP24_ERR_TIMEOUT
    assert B.sp24_device_status() == B.SP24_OK         # read and cleared
    w = I.normal_bf16((64, 128), 1.0, seed=3)        # the library still works
    mask = P.prune(w.cuda(), B.SP24_MAGNITUDE, 2)
    assert np.array_equal(keep_of(mask, 128), O.prune(f64(w), O.MAGNITUDE, 2))
    ok_status()
    with pytest.raises(B.Sp24Error):
        B.sp24_selftest_wait_timeout(0)


_CONCURRENT_FIRST_CALLS = r"""
import sys, threading, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from oracle import sp24_oracle as O
from structured_sparse_gemm_sp24_b200 import inputs as I, pipeline as P, sp24 as B
torch.cuda.set_device(0)
B.lib()
shapes = [(2500, 2056, 400), (16, 392, 1024), (300, 24, 128), (4099, 1032, 784)]
data, out, err = [], [None] * 4, []
for i, (m, n, k) in enumerate(shapes):
    W = I.normal_bf16((n, k), 1.0, seed=100 + i)
    X = I.normal_bf16((m, k), 1.0, seed=200 + i)
    Wd = W.cuda()
    mask = P.prune(Wd, B.SP24_MAGNITUDE, 2)
    vals, meta = P.compress(Wd, mask, B.SP24_BF16)
    data.append((W, X, X.cuda(), vals, meta, n))
torch.cuda.synchronize()
go = threading.Barrier(4)
def run(i):
    try:
        W, X, Xd, vals, meta, n = data[i]
        st = torch.cuda.Stream()
        with torch.cuda.stream(st):
            go.wait()          # first GEMM launches of the process, all at once
            y = P.gemm(Xd, vals, meta, n)
        st.synchronize()
        out[i] = y
    except Exception as e:
        err.append(repr(e))
ts = [threading.Thread(target=run, args=(i,)) for i in range(4)]
[t.start() for t in ts]; [t.join() for t in ts]
assert not err, err
assert B.sp24_device_status() == B.SP24_OK
for i, (W, X, _, _, _, n) in enumerate(data):
    keep = O.prune(W.double().numpy(), O.MAGNITUDE, 2)
    v, mt = O.compress(W.double().numpy(), keep)
    yr, ar = O.gemm(X.double().numpy(), v, mt, W.shape[1])
    d = np.abs(out[i].double().cpu().numpy() - yr)
    assert (d <= 8e-3 * ar + 1e-30).all(), i
print("ok")
"""


def test_concurrent_first_calls_from_host_threads():
    # a fresh process, so the per-device kernel attributes and plan caches are
    # set up by four threads racing on their first GEMM launches
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _CONCURRENT_FIRST_CALLS, root],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stderr[-2000:]


# ------------------------------------------------------------ launch plans
def test_gemm_plan_families(monkeypatch):
    monkeypatch.delenv("SP24_GEMM_IMPL", raising=False)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    small = B.sp24_gemm_plan(16, 11008, 4096, B.SP24_BF16)
    assert small["kernel"] == "splitk" and small["tile_tokens"] == 16
    assert small["split_k"] >= 1 and small["cluster"] == small["split_k"]
    big = B.sp24_gemm_plan(8192, 8192, 8192, B.SP24_BF16)
    assert big["kernel"].startswith("pair") and big["cluster"] == 2
    # a persistent pair grid never exceeds the resident pairs (<= SMs / 2)
    assert big["ctas"] % 2 == 0 and 2 <= big["ctas"] <= sms
    conv = B.sp24_gemm_plan(200704, 64, 256, B.SP24_BF16)
    assert conv["kernel"] == "single" and conv["ctas"] == sms
    # less than one wave of 128 x 128 tiles (86 for N = 11008): split-K
    assert B.sp24_gemm_plan(128, 11008, 4096, B.SP24_BF16)["kernel"] == "splitk"
    # 16 tokens, 86 row tiles of 32 stages: split so that several CTAs share
    # each SM (the exact split depends on how many clusters the GPCs hold)
    dec = B.sp24_gemm_plan(16, 11008, 4096, B.SP24_BF16)
    assert dec["split_k"] > 1 and dec["ctas"] == 86 * dec["split_k"] > sms
    assert dec["cluster"] == dec["split_k"]
    # 32 row tiles of 86 stages: split 4 fills the SMs once
    dec2 = B.sp24_gemm_plan(16, 4096, 11008, B.SP24_BF16)
    assert dec2["split_k"] == 4 and dec2["ctas"] == 128
    # the one-accumulator 256-token pair tile for the INT8 workload shape
    assert B.sp24_gemm_plan(8192, 4096, 4096, B.SP24_INT8)["kernel"] == "pair256"
    monkeypatch.setenv("SP24_GEMM_IMPL", "pair240")
    forced = B.sp24_gemm_plan(4096, 3072, 768, B.SP24_BF16)
    assert forced["kernel"] == "pair240" and forced["tile_tokens"] == 240
    assert forced["tile_channels"] == 256
    with pytest.raises(B.Sp24Error):
        B.sp24_gemm_plan(0, 64, 64, B.SP24_BF16)
