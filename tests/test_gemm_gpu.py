"""GPU tests of the tcgen05/TMA weight-streaming GEMM (lt_gemm_rows).

Reference: the same bf16 (or fp32) operand values multiplied in fp64 on the
CPU.  bf16 operands are exact in both, so the only difference is the fp32
accumulation order: |err| <= ~K * 2^-24 * sum|x_k w_k|.  fp32 operands run as
split tf32 (hi*hi + hi*lo + lo*hi): each product is within ~2^-21 relative,
so |err| <= ~(2^-20 + K * 2^-24) * sum|x_k w_k|.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

SHAPES = [
    (6144, 2048), (2048, 2048), (11264, 2048), (2048, 5632),  # shared block, Ouro-shaped
    (15840, 5280), (5280, 5280),  # Huginn-shaped: 5280 is not a multiple of 64 (K and n_out tails)
    (300, 200), (128, 64), (129, 72),  # small and ragged
]


def _ref(w, x):
    return (x.double().cpu() @ w.double().cpu().T)


def _bound(w, x, unit):
    return (x.double().abs().cpu() @ w.double().abs().cpu().T) * unit + 1e-30


@pytest.mark.parametrize("n_out,k", SHAPES)
@pytest.mark.parametrize("ncols", [8, 16, 64])
def test_gemm_bf16_matches_fp64(n_out, k, ncols):
    from looped_transformer_self_b200.binding import gemm_rows
    g = torch.Generator().manual_seed(n_out * 7 + k + ncols)
    w = (torch.randn(n_out, k, generator=g) / k ** 0.5).bfloat16().cuda()
    x = torch.randn(ncols, k, generator=g).bfloat16().cuda()
    y = gemm_rows(w, x).double().cpu()
    err = (y - _ref(w, x)).abs()
    assert torch.all(err <= _bound(w, x, 4 * k * 2.0 ** -24)), float(err.max())


@pytest.mark.parametrize("n_out,k", [(384, 128), (1152, 128), (512, 128), (128, 384), (300, 200)])
def test_gemm_f32_split_tf32_matches_fp64(n_out, k):
    from looped_transformer_self_b200.binding import gemm_rows
    g = torch.Generator().manual_seed(n_out + k)
    w = (torch.randn(n_out, k, generator=g) / k ** 0.5).cuda()
    x = torch.randn(8, k, generator=g).cuda()
    y = gemm_rows(w, x).double().cpu()
    err = (y - _ref(w, x)).abs()
    assert torch.all(err <= _bound(w, x, 2.0 ** -20 + 4 * k * 2.0 ** -24)), float(err.max())


def test_gemm_rows_are_independent_and_deterministic():
    """A row's result is bit-identical whatever the other rows hold, and
    repeated calls are bit-identical (fixed-order split-K reduction)."""
    from looped_transformer_self_b200.binding import gemm_rows
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(6144, 2048, generator=g) / 45).bfloat16().cuda()
    x = torch.randn(16, 2048, generator=g).bfloat16().cuda()
    y1 = gemm_rows(w, x)
    y2 = gemm_rows(w, x)
    assert torch.equal(y1, y2)
    x2 = x.clone()
    x2[1:] = torch.randn(15, 2048, generator=g).bfloat16().cuda()
    x2[5] = x[0]
    y3 = gemm_rows(w, x2)
    assert torch.equal(y3[0], y1[0]) and torch.equal(y3[5], y1[0])
    xz = torch.zeros_like(x)
    xz[9] = x[0]
    assert torch.equal(gemm_rows(w, xz)[9], y1[0])


def test_gemm_returns_ok_status_word():
    """A normal call clears the scratch's error word, runs, finds the word
    still 0 after its synchronisation and returns LT_OK (a bounded wait that
    gave up would make it LT_ERR_DEVICE_CHECK; the give-up path itself is
    exercised by tests/test_selftest_gpu.py without a fault)."""
    import ctypes
    from looped_transformer_self_b200.binding import LT_BF16, lib
    w = torch.randn(2048, 2048).bfloat16().cuda()
    x = torch.randn(16, 2048).bfloat16().cuda()
    y = torch.empty(16, 2048, dtype=torch.float32, device="cuda")
    need = ctypes.c_size_t()
    assert lib().lt_gemm_scratch_bytes(LT_BF16, 2048, 2048, 16, ctypes.byref(need)) == 0
    scratch = torch.full((need.value,), 0xFF, dtype=torch.uint8, device="cuda")  # word != 0 before
    torch.cuda.synchronize()
    for _ in range(2):
        rc = lib().lt_gemm_rows(LT_BF16, w.data_ptr(), x.data_ptr(), y.data_ptr(), 2048, 2048, 16,
                                scratch.data_ptr(), need.value, torch.cuda.current_stream().cuda_stream)
        assert rc == 0
    assert int(scratch[:4].view(torch.int32).item()) == 0
