"""The tensor-level functions reject wrong dtypes, devices and shapes with
ValueError before anything is launched (the C ABI takes raw pointers and
could not see the sizes)."""

import pytest
import torch

import exact_attention_120_b200 as fa

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16, device=DEV)


def test_forward_rejects_bad_tensors():
    q, k, v = _bf(1, 2, 256, 64), _bf(1, 2, 256, 64), _bf(1, 2, 256, 64)
    with pytest.raises(ValueError):
        fa.attention_forward(q, k, _bf(1, 2, 255, 64))                  # v rows differ from k
    with pytest.raises(ValueError):
        fa.attention_forward(q, _bf(1, 3, 256, 64), _bf(1, 3, 256, 64))  # heads differ
    with pytest.raises(ValueError):
        fa.attention_forward(q, k, v, out=_bf(1, 2, 128, 64))           # out too small
    with pytest.raises(ValueError):
        fa.attention_forward(q, k, v, lse=torch.zeros((1, 2, 256), device=DEV, dtype=torch.float16))
    with pytest.raises(ValueError):
        fa.attention_forward(q, k, v, block_mask=torch.ones((1, 2, 1, 2), dtype=torch.uint8, device=DEV))
    with pytest.raises(ValueError):
        fa.attention_forward(q.cpu(), k, v)                              # host tensor
    with pytest.raises(ValueError):
        fa.attention_forward(q.transpose(2, 3), k, v)                    # not contiguous
    torch.cuda.synchronize()


def test_backward_rejects_bad_tensors():
    q, k, v = _bf(1, 2, 128, 64), _bf(1, 2, 128, 64), _bf(1, 2, 128, 64)
    o, lse = fa.attention_forward(q, k, v)
    do = _bf(1, 2, 128, 64)
    with pytest.raises(ValueError):
        fa.attention_backward(q, k, v, o, lse[:, :, :64].contiguous(), do)   # lse too short
    with pytest.raises(ValueError):
        fa.attention_backward(q, k, v, o, lse, _bf(1, 2, 128, 128))         # dout shape
    with pytest.raises(ValueError):
        fa.attention_backward(q, k, v, o, lse, do, workspace=torch.empty(8, dtype=torch.uint8))
    torch.cuda.synchronize()


def test_varlen_and_fp8_reject_bad_tensors():
    q = _bf(100, 2, 128)
    cu = torch.tensor([0, 60, 100], dtype=torch.int32, device=DEV)
    with pytest.raises(ValueError):
        fa.attention_forward_varlen(q, _bf(100, 2, 128), _bf(99, 2, 128), cu, cu, 60)
    with pytest.raises(ValueError):
        fa.attention_forward_varlen(q, q, q, cu, cu[:2].contiguous(), 60)
    with pytest.raises(ValueError):
        fa.attention_forward_varlen(q, q, q, cu.long(), cu, 60)
    with pytest.raises(ValueError):
        fa.attention_forward_varlen(q, q, q, cu, cu, 60, lse=torch.zeros((100, 2), device=DEV))
    q8 = torch.zeros((1, 1, 128, 128), dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        fa.attention_forward_fp8(q8, q8, torch.zeros((1, 1, 64, 128), dtype=torch.uint8, device=DEV),
                                 1.0, 1.0, 1.0)
    with pytest.raises(ValueError):
        fa.attention_forward_fp8(q8.to(torch.int8), q8, q8, 1.0, 1.0, 1.0)
    torch.cuda.synchronize()
