"""lynx_linear_host: the layer on host-memory activations, row chunks copied in
and out while the kernels run.  Its Y equals lynx_linear's on device copies of
the same inputs, bit for bit, for one and for several chunks, on both paths."""
import numpy as np
import pytest
import torch

from activation_sparse_gemm_lynx_b200 import lynx, workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def bf16(bits, device=None):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t if device is None else t.to(device)


@pytest.mark.parametrize("M,K,N,skip,lora", [
    (300, 576, 264, False, True),     # one ragged chunk
    (4608, 512, 1024, False, True),   # six chunks of 768 rows
    (2500, 1024, 512, False, False),  # four chunks of 768 rows, the last 196, no LoRA
    (4100, 512, 768, True, True),     # dense path, six chunks of 768 rows, the last 260
])
def test_host_entry_matches_device_entry(M, K, N, skip, lora):
    assert torch.cuda.is_available(), "this test needs a GPU"
    torch.cuda.set_device(0)
    lynx.lynx_check_error()
    inp = workloads.make_linear_inputs(M, K, N, seed=[7, M, K, N], lora=lora)
    W, bias = bf16(inp["W"], DEV), bf16(inp["bias"], DEV)
    A = bf16(inp["A"], DEV) if lora else None
    B = bf16(inp["B"], DEV) if lora else None
    ref = lynx.lynx_linear(bf16(inp["X"], DEV), W, bias, A, B, skip_sparsify=skip)
    Xh = bf16(inp["X"]).pin_memory()
    Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    for _ in range(2):  # twice: the library's streams and events are reused
        Yh.zero_()
        lynx.lynx_linear_host(Xh, W, bias, A, B, skip_sparsify=skip, Y_host=Yh)
        torch.cuda.current_stream().synchronize()
        st, code = lynx.lynx_check_error()
        assert st == lynx.LYNX_OK, (st, code)
        assert torch.equal(Yh.view(torch.int16), ref.cpu().view(torch.int16))
