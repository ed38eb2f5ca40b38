"""The allocation-free GEMM entry point (lt_gemm_rows_noalloc).

It exists for callers that cannot allocate device memory (a CUDA graph or a
memory pool owns every allocation, a plug-in is handed a stream but no
allocator, another framework has reserved the device): its scratch is a static
array inside the library.  This file is collected last on purpose, so that a
run stopping at the first failure has already run every other test; it must
pass both alone in a fresh process and after the other tests.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _bound(w, x, k):
    return (x.double().abs().cpu() @ w.double().abs().cpu().T) * (4 * k * 2.0 ** -24) + 1e-30


@pytest.mark.parametrize("n_out,k,ncols", [(6144, 2048, 16), (2048, 5632, 16), (300, 200, 8),
                                           (49152, 2048, 16)])
def test_noalloc_matches_allocating_entry_on_two_calls(n_out, k, ncols):
    from looped_transformer_self_b200.binding import gemm_rows, gemm_rows_noalloc
    g = torch.Generator().manual_seed(n_out + k)
    w = (torch.randn(n_out, k, generator=g) / k ** 0.5).bfloat16().cuda()
    ref = gemm_rows(w, torch.randn(ncols, k, generator=g).bfloat16().cuda())  # warm the other path
    for call in range(2):  # two calls in a row share (and reuse) the static scratch
        x = torch.randn(ncols, k, generator=g).bfloat16().cuda()
        ref = gemm_rows(w, x).double().cpu()
        got = gemm_rows_noalloc(w, x).double().cpu()
        assert torch.all((got - ref).abs() <= _bound(w, x, k)), (call, float((got - ref).abs().max()))


def test_noalloc_returns_ok_status_on_two_calls():
    """Each call clears the library's static error word before its launch and
    reads it back after its synchronisation: a normal call returns LT_OK."""
    from looped_transformer_self_b200.binding import LT_BF16, lib
    w = torch.randn(2048, 2048).bfloat16().cuda()
    x = torch.randn(16, 2048).bfloat16().cuda()
    y = torch.empty(16, 2048, dtype=torch.float32, device="cuda")
    for _ in range(2):
        rc = lib().lt_gemm_rows_noalloc(LT_BF16, w.data_ptr(), x.data_ptr(), y.data_ptr(), 2048,
                                        2048, 16, torch.cuda.current_stream().cuda_stream)
        assert rc == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from looped_transformer_self_b200.binding import LoopedSpecError, gemm_rows_noalloc
    w = torch.zeros(49152, 2048, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(64, 2048, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(LoopedSpecError) as e:
        gemm_rows_noalloc(w, x)
    assert e.value.code == -3
