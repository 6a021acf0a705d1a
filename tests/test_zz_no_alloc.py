"""GPU test of sp24_prune_wanda_noalloc, the Wanda prune for callers that must
not allocate device memory (engines and plugins with a fixed memory plan).

It must produce exactly the masks of sp24_prune (mode SP24_WANDA, with a
caller workspace) on the same inputs, over consecutive calls that reuse the
library's shared scratch array.  The file is collected last so that a run
stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import pytest
import torch

from structured_sparse_gemm_sp24_b200 import inputs as I
from structured_sparse_gemm_sp24_b200 import sp24 as B

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    B.lib()


def _with_workspace(W, Xc, n_keep, mask_in=None):
    N, K = W.shape
    out = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    ws = torch.empty(B.sp24_prune_workspace_bytes(K, B.SP24_WANDA), dtype=torch.uint8,
                     device=W.device)
    B.sp24_prune(W, Xc, B.SP24_WANDA, n_keep, mask_in, out, ws)
    return out


def _no_alloc(W, Xc, n_keep, mask_in=None):
    N, K = W.shape
    out = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    B.sp24_prune_wanda_noalloc(W, Xc, n_keep, mask_in, out)
    return out


def test_no_alloc_matches_workspace_prune_on_consecutive_calls():
    # call 1: BERT fc1 shapes, 3:4 stage
    w = I.bert_fc1()
    W1, Xc1 = w.W.cuda(), w.Xc.cuda()
    got1 = _no_alloc(W1, Xc1, 3)
    ref1 = _with_workspace(W1, Xc1, 3)
    # call 2 reuses the scratch array with a smaller K and a mask_in: a stale
    # norm from call 1 would change the result
    W2 = I.normal_bf16((333, 264), 0.02, seed=71).cuda()
    Xc2 = I.normal_bf16((37, 264), 1.0, seed=72).cuda()
    m1 = _with_workspace(W2, Xc2, 3)
    got2 = _no_alloc(W2, Xc2, 2, m1)
    ref2 = _with_workspace(W2, Xc2, 2, m1)
    # call 3: back to the first problem, 2:4 stage on top of its 3:4 mask
    got3 = _no_alloc(W1, Xc1, 2, ref1)
    ref3 = _with_workspace(W1, Xc1, 2, ref1)
    assert B.sp24_device_status() == B.SP24_OK
    assert torch.equal(got1, ref1)
    assert torch.equal(got2, ref2)
    assert torch.equal(got3, ref3)


def test_no_alloc_separate_norm_kernel_on_consecutive_calls():
    # Row tiles x calibration rows above 8192 make the library compute the
    # column norms with their own kernel, which writes them to the scratch
    # array, and the prune kernel then reads them back from it (the fused
    # path above keeps them on chip).  Call 1: 11008 rows (86 row tiles) x
    # 128 calibration rows.  Call 2: 1024 rows (8 row tiles) x 1100
    # calibration rows, smaller K, with a mask_in: norms left over from call 1
    # in the shared array would change its mask.
    Wa = I.normal_bf16((11008, 512), 0.02, seed=81).cuda()
    Xa = I.normal_bf16((128, 512), 1.0, seed=82).cuda()
    Wb = I.normal_bf16((1024, 264), 0.02, seed=83).cuda()
    Xb = I.normal_bf16((1100, 264), 1.0, seed=84).cuda()
    got_a = _no_alloc(Wa, Xa, 3)
    mb = _with_workspace(Wb, Xb, 3)
    got_b = _no_alloc(Wb, Xb, 2, mb)
    ref_a = _with_workspace(Wa, Xa, 3)
    ref_b = _with_workspace(Wb, Xb, 2, mb)
    # call 3 repeats call 1 after call 2 left other norms in the array
    got_a2 = _no_alloc(Wa, Xa, 3)
    assert B.sp24_device_status() == B.SP24_OK
    assert torch.equal(got_a, ref_a)
    assert torch.equal(got_b, ref_b)
    assert torch.equal(got_a2, ref_a)


def test_no_alloc_rejects_k_above_limit():
    big = B.SP24_NOALLOC_MAX_K + 8
    W = torch.empty((1, big), dtype=torch.bfloat16, device="cuda")
    Xc = torch.empty((1, big), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((1, big // 8), dtype=torch.uint8, device="cuda")
    with pytest.raises(B.Sp24Error) as e:
        B.sp24_prune_wanda_noalloc(W, Xc, 2, None, out)
    assert e.value.status == B.SP24_ERR_UNSUPPORTED
