"""The allocation-free GEMM entry point (alodlm_gemm_bf16_noalloc).

Some callers cannot allocate device memory themselves: code whose device memory is owned
and budgeted by a host framework's pool, and latency-critical paths that must not pay for
cudaMalloc/cudaFree (which can synchronise the device).  For them the library offers a
variant of its stream-K GEMM whose scratch is a fixed array compiled into the library.
This test calls it through the C ABI twice in a row and checks each result against a
float64 product of the same bf16 inputs and against the workspace-taking entry point
(alodlm_gemm_bf16), within the GEMM tests' tolerance, with the call's own status word read
back as zero; it also checks that shapes beyond the array's limits are refused.  It runs
last so that a failure here leaves every other test already run, and it passes both alone
in a fresh process and after the rest of the suite.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 1e-5  # max |C - ref| / max |ref|, as in the GEMM tests


@pytest.mark.parametrize("M,N,K", [(32, 6144, 4096), (20, 1376, 880), (64, 4096, 12288), (1, 128, 64)])
def test_noalloc_gemm_matches_fp64_and_workspace_gemm_twice(M, N, K):
    import adaptively_looped_masked_b200 as alo
    g = torch.Generator(device="cuda").manual_seed(1000 + M + N + K)
    ws = torch.zeros(64 + 4096 + 16 * M * N + (8 << 20), dtype=torch.float32, device="cuda")
    for call in range(2):
        A = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
        W = torch.randn((N, K), device="cuda", generator=g).to(torch.bfloat16)
        ref64 = A.double() @ W.double().T
        with_ws = alo.gemm_bf16(A, W, workspace=ws)
        out = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        alo.gemm_bf16_noalloc(A, W, out, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, "the allocation-free call's own status word"
        assert int(ws[:1].view(torch.int32).item()) == 0, "the workspace call's status word"
        scale = ref64.abs().max().item()
        err64 = (out.double() - ref64).abs().max().item() / scale
        err_ws = (out - with_ws).abs().max().item() / scale
        assert err64 < TOL, (call, M, N, K, err64)
        assert err_ws < TOL, (call, M, N, K, err_ws)


def test_noalloc_gemm_refuses_shapes_beyond_its_scratch():
    import adaptively_looped_masked_b200 as alo
    A = torch.zeros((65, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((65, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(alo.AlodlmError) as e:
        alo.gemm_bf16_noalloc(A, W, out)
    assert e.value.code == -1 and "M <= 64" in str(e.value)
    A = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((32768 + 128, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((8, 32768 + 128), dtype=torch.float32, device="cuda")
    with pytest.raises(alo.AlodlmError) as e:
        alo.gemm_bf16_noalloc(A, W, out)
    assert e.value.code == -1
