"""GPU parity of the 3x3 convolution path ([Orin ch.7] 2.2 A.3, 2.1): the
im2col gather through the C ABI is bit-exact against the oracle's im2col,
and the sparse convolution (prune + compress of W[Cout][3][3][C] as
[Cout][9C], gather, sparse GEMM) matches the oracle's direct convolution of
the pruned weights: bf16 within |dy| <= 8e-3 * sum|x w|, int8 (int32
accumulator) bit-exact."""
import numpy as np
import pytest
import torch

from oracle import sp24_oracle as O
from structured_sparse_gemm_sp24_b200 import inputs as I
from structured_sparse_gemm_sp24_b200 import pipeline as P
from structured_sparse_gemm_sp24_b200 import sp24 as B

pytestmark = pytest.mark.gpu
TOL = 8e-3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    B.lib()
    assert B.sp24_device_status() == B.SP24_OK


def f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


@pytest.mark.parametrize("b,h,w,c,dtype", [
    (2, 5, 7, 8, torch.bfloat16), (1, 1, 1, 16, torch.int8), (3, 4, 9, 64, torch.bfloat16),
    (2, 6, 5, 32, torch.int8), (4, 28, 28, 128, torch.bfloat16), (1, 2, 1, 24, torch.bfloat16)])
def test_im2col_bit_exact(b, h, w, c, dtype):
    g = torch.Generator().manual_seed(b * 1000 + h * 100 + w * 10 + c)
    if dtype == torch.int8:
        x = torch.randint(-127, 128, (b, h, w, c), generator=g, dtype=torch.int8)
        bits = x.numpy()
    else:
        x = torch.randn((b, h, w, c), generator=g).to(dtype)
        bits = x.view(torch.int16).numpy()
    a = P.im2col3x3(x.cuda())
    assert B.sp24_device_status() == B.SP24_OK
    got = a.cpu()
    got = got.numpy() if dtype == torch.int8 else got.view(torch.int16).numpy()
    assert np.array_equal(got, O.im2col3x3(bits))


def test_im2col_rejects_unaligned_channels():
    x = torch.zeros((1, 4, 4, 12), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.Sp24Error) as e:
        P.im2col3x3(x)
    assert e.value.status == B.SP24_ERR_ALIGN


def _sparse_conv_bf16(b, h, w, c, cout, seed):
    w4 = I.normal_bf16((cout, 3, 3, c), 0.05, seed)
    x = I.normal_bf16((b, h, w, c), 1.0, seed + 1)
    wflat = w4.view(cout, 9 * c)
    vals, meta, mask = P.prune_compress(wflat.cuda(), B.SP24_MAGNITUDE, want_mask=True)
    y = P.conv3x3(x.cuda(), vals, meta, cout)
    assert B.sp24_device_status() == B.SP24_OK
    keep = O.prune(f64(wflat), O.MAGNITUDE, 2)
    assert np.array_equal(O.unpack_mask(mask.cpu().numpy(), 9 * c), keep)
    wm4 = np.where(keep, f64(wflat), 0.0).reshape(cout, 3, 3, c)
    return x, wm4, y


@pytest.mark.parametrize("b,h,w,c,cout", [(2, 9, 11, 64, 64), (1, 5, 3, 32, 16),
                                         (4, 28, 28, 128, 128), (1, 14, 14, 256, 256)])
def test_sparse_conv3x3_bf16_matches_oracle(b, h, w, c, cout):
    x, wm4, y = _sparse_conv_bf16(b, h, w, c, cout, seed=b + h + c)
    xo = f64(x)
    y_ref = O.conv3x3_nhwc(xo, wm4)
    a_ref = O.conv3x3_nhwc(np.abs(xo), np.abs(wm4))
    d = np.abs(f64(y) - y_ref)
    assert (d <= TOL * a_ref).all(), float((d / np.maximum(a_ref, 1e-30)).max())


def test_sparse_conv3x3_int8_bit_exact():
    b, h, w, c, cout = 2, 10, 13, 64, 64
    w4 = I.long_tail_bf16((cout, 3, 3, c), 0.02, seed=41, tail_seed=42)
    x = I.normal_f32((b, h, w, c), 1.0, seed=43)
    wflat = w4.view(cout, 9 * c)
    wd = wflat.cuda()
    mask = P.prune(wd, B.SP24_MAGNITUDE, 2)
    s_w = P.wscale(wd, mask)
    vals, meta = P.compress(wd, mask, B.SP24_INT8, s_w)
    xd = x.cuda()
    s_x = P.act_scale(xd)
    xq = P.quantize(xd, s_x)
    y32 = P.conv3x3(xq, vals, meta, cout, dtype=B.SP24_INT8, s_x=s_x, s_w=s_w,
                    out_kind=B.SP24_OUT_INT32)
    assert B.sp24_device_status() == B.SP24_OK
    keep = O.prune(f64(wflat), O.MAGNITUDE, 2)
    rs = O.channel_scales(f64(wflat), keep)
    rv, rm = O.compress(O.quantize(f64(wflat), rs[:, None]), keep)
    sx = O.tensor_scale(x.numpy().astype(np.float64))
    assert s_x.item() == sx and np.array_equal(s_w.cpu().numpy(), rs)
    xq_o = O.quantize(x.numpy(), sx)
    acc = O.gemm_int8_acc(O.im2col3x3(xq_o), rv, rm, 9 * c)
    assert np.array_equal(y32.cpu().numpy().reshape(-1, cout), acc)


def test_conv3x3_large_batch_timing_and_parity():
    # ResNet stage-2 3x3 convolution (128 -> 128 channels, 28 x 28) at batch
    # 32: explicit gather + GEMM against the implicit GEMM, both checked on
    # every output against the oracle's direct convolution
    b, h, w, c, cout = 32, 28, 28, 128, 128
    w4 = I.normal_bf16((cout, 3, 3, c), 0.05, 51)
    x = I.normal_bf16((b, h, w, c), 1.0, 52)
    xd = x.cuda()
    vals, meta = P.prune_compress(w4.view(cout, 9 * c).cuda(), B.SP24_MAGNITUDE)
    a = torch.empty((b * h * w, 9 * c), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((b * h * w, cout), dtype=torch.bfloat16, device="cuda")
    yi = torch.empty((b, h, w, cout), dtype=torch.bfloat16, device="cuda")

    def implicit():
        B.sp24_conv3x3(xd, vals, meta, cout, B.SP24_BF16, None, None, B.SP24_OUT_BF16, None, yi)

    for _ in range(3):
        B.sp24_im2col3x3(xd, a)
        P.gemm(a, vals, meta, cout, out=y)
        implicit()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    reps = 20
    ev[0].record()
    for _ in range(reps):
        B.sp24_im2col3x3(xd, a)
    ev[1].record()
    for _ in range(reps):
        P.gemm(a, vals, meta, cout, out=y)
    ev[2].record()
    for _ in range(reps):
        implicit()
    ev[3].record()
    torch.cuda.synchronize()
    assert B.sp24_device_status() == B.SP24_OK
    t_i = ev[0].elapsed_time(ev[1]) / reps * 1e3
    t_g = ev[1].elapsed_time(ev[2]) / reps * 1e3
    t_c = ev[2].elapsed_time(ev[3]) / reps * 1e3
    m, k = b * h * w, 9 * c
    print(f"\nconv3x3 {b}x{h}x{w} {c}->{cout}: im2col {t_i:.1f} us "
          f"({(m * c * 2 + m * k * 2) / t_i / 1e3:.0f} GB/s read+write), "
          f"sparse GEMM {t_g:.1f} us ({2 * m * cout * k / t_g / 1e6:.0f} TFLOP/s dense-equiv); "
          f"implicit GEMM {t_c:.1f} us ({2 * m * cout * k / t_c / 1e6:.0f} TFLOP/s)")
    keep = O.prune(f64(w4.view(cout, 9 * c)), O.MAGNITUDE, 2)
    wm4 = np.where(keep, f64(w4.view(cout, 9 * c)), 0.0).reshape(cout, 3, 3, c)
    xo = f64(x)
    y_ref = O.conv3x3_nhwc(xo, wm4).reshape(m, cout)
    a_ref = O.conv3x3_nhwc(np.abs(xo), np.abs(wm4)).reshape(m, cout)
    for got in (f64(y), f64(yi).reshape(m, cout)):
        assert (np.abs(got - y_ref) <= TOL * a_ref).all()


# ------------------------------------------------ implicit GEMM (sp24_conv3x3)
# (B, H, W, C, Cout): W = 16 / 32 (one image row per box, 256-token tiles),
# W = 28 (two rows per box, 224-token tiles), W = 56 with K = 9 * 64 = 4.5
# k-blocks (the last half k-block reads past K), a last tile past the final
# image (M = 192 < 256), and Cout not a multiple of the 256-channel pair tile
IMPLICIT_BF16 = [(2, 8, 16, 64, 64), (4, 28, 28, 128, 128), (2, 56, 56, 64, 64),
                 (3, 8, 8, 64, 256), (1, 16, 32, 128, 192),
                 # output channels that fill neither a 128-row nor a 256-row tile
                 (2, 8, 32, 64, 72), (1, 16, 16, 128, 200)]


@pytest.mark.parametrize("b,h,w,c,cout", IMPLICIT_BF16)
def test_implicit_conv3x3_bf16_matches_oracle(b, h, w, c, cout):
    w4 = I.normal_bf16((cout, 3, 3, c), 0.05, 71 + c)
    x = I.normal_bf16((b, h, w, c), 1.0, 72 + w)
    wflat = w4.view(cout, 9 * c)
    vals, meta = P.prune_compress(wflat.cuda(), B.SP24_MAGNITUDE)
    y = P.conv3x3(x.cuda(), vals, meta, cout, path="implicit")
    assert B.sp24_device_status() == B.SP24_OK
    keep = O.prune(f64(wflat), O.MAGNITUDE, 2)
    wm4 = np.where(keep, f64(wflat), 0.0).reshape(cout, 3, 3, c)
    xo = f64(x)
    y_ref = O.conv3x3_nhwc(xo, wm4)
    a_ref = O.conv3x3_nhwc(np.abs(xo), np.abs(wm4))
    d = np.abs(f64(y) - y_ref)
    assert (d <= TOL * a_ref).all(), float((d / np.maximum(a_ref, 1e-30)).max())


@pytest.mark.parametrize("b,h,w,c,cout", [(2, 10, 16, 128, 64), (1, 8, 32, 256, 128)])
def test_implicit_conv3x3_int8_bit_exact(b, h, w, c, cout):
    w4 = I.long_tail_bf16((cout, 3, 3, c), 0.02, seed=81, tail_seed=82)
    x = I.normal_f32((b, h, w, c), 1.0, seed=83)
    wflat = w4.view(cout, 9 * c)
    wd = wflat.cuda()
    mask = P.prune(wd, B.SP24_MAGNITUDE, 2)
    s_w = P.wscale(wd, mask)
    vals, meta = P.compress(wd, mask, B.SP24_INT8, s_w)
    xd = x.cuda()
    s_x = P.act_scale(xd)
    xq = P.quantize(xd, s_x)
    kw = dict(dtype=B.SP24_INT8, s_x=s_x, s_w=s_w, path="implicit")
    y32 = P.conv3x3(xq, vals, meta, cout, out_kind=B.SP24_OUT_INT32, **kw)
    ybf = P.conv3x3(xq, vals, meta, cout, out_kind=B.SP24_OUT_BF16, **kw)
    assert B.sp24_device_status() == B.SP24_OK
    keep = O.prune(f64(wflat), O.MAGNITUDE, 2)
    rs = O.channel_scales(f64(wflat), keep)
    rv, rm = O.compress(O.quantize(f64(wflat), rs[:, None]), keep)
    sx = O.tensor_scale(x.numpy().astype(np.float64))
    assert s_x.item() == sx and np.array_equal(s_w.cpu().numpy(), rs)
    a = O.im2col3x3(O.quantize(x.numpy(), sx))
    # float64 product of the int8 operands: every partial sum is an integer
    # below 2^31, exact; checked against the oracle's int64 product on a slice
    acc = (a.astype(np.float64) @ O.decompress(rv, rm, 9 * c).astype(np.float64).T).astype(np.int64)
    assert np.array_equal(acc[:32], O.gemm_int8_acc(a[:32], rv, rm, 9 * c))
    assert np.array_equal(y32.cpu().numpy().reshape(-1, cout), acc)
    got = ybf.reshape(-1, cout).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.dequant_bf16(acc, sx, rs))


def test_implicit_conv3x3_rejects_untiled_shapes():
    # 14 x 14 images: no r dividing 14 with 14 r % 8 == 0; C = 32 bf16 rows of
    # 64 bytes: a K-half would span two taps
    vals = torch.zeros((64, 9 * 64 // 2), dtype=torch.bfloat16, device="cuda")
    meta = torch.zeros(B.sp24_meta_bytes(64, 9 * 64), dtype=torch.uint8, device="cuda")
    x = torch.zeros((1, 14, 14, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.Sp24Error) as e:
        P.conv3x3(x, vals, meta, 64, path="implicit")
    assert e.value.status == B.SP24_ERR_UNSUPPORTED
    x32 = torch.zeros((1, 16, 16, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.Sp24Error) as e:
        P.conv3x3(x32, vals, meta, 64, path="implicit")
    assert e.value.status == B.SP24_ERR_ALIGN
    # the automatic path falls back to the explicit gather for such shapes
    y = P.conv3x3(x, vals, meta, 64)
    assert y.shape == (1, 14, 14, 64) and B.sp24_device_status() == B.SP24_OK


def test_implicit_conv3x3_int8_requantised_output():
    # int8 codes in, int8 codes out (requantised with s_y), single-SM tiles
    # with 4 boxes of 2 image rows per tile and a partial last tile
    b, h, w, c, cout = 3, 10, 16, 128, 32
    w4 = I.normal_bf16((cout, 3, 3, c), 0.02, 91)
    x = I.normal_f32((b, h, w, c), 1.0, 92)
    wflat = w4.view(cout, 9 * c).cuda()
    mask = P.prune(wflat, B.SP24_MAGNITUDE, 2)
    s_w = P.wscale(wflat, mask)
    vals, meta = P.compress(wflat, mask, B.SP24_INT8, s_w)
    xd = x.cuda()
    s_x = P.act_scale(xd)
    xq = P.quantize(xd, s_x)
    s_y = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    y8 = P.conv3x3(xq, vals, meta, cout, dtype=B.SP24_INT8, s_x=s_x, s_w=s_w,
                   out_kind=B.SP24_OUT_INT8, s_y=s_y, path="implicit")
    assert B.sp24_device_status() == B.SP24_OK
    wf = f64(w4.view(cout, 9 * c))
    keep = O.prune(wf, O.MAGNITUDE, 2)
    rs = O.channel_scales(wf, keep)
    rv, rm = O.compress(O.quantize(wf, rs[:, None]), keep)
    sx = O.tensor_scale(x.numpy().astype(np.float64))
    acc = O.gemm_int8_acc(O.im2col3x3(O.quantize(x.numpy(), sx)), rv, rm, 9 * c)
    ref = O.requant_int8(acc, sx, rs, np.float32(0.05))
    assert np.array_equal(y8.cpu().numpy().reshape(-1, cout), ref)
