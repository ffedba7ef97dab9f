"""MoELayer.forward's input checks on the CPU: the library reads x and y_out
through their data pointers alone, so the wrapper refuses a tensor of the
wrong type, width, layout or device before any call (no GPU needed: the
library calls are replaced by recorders)."""
import pytest
import torch

from bit_dequant_expert_b200.layer import MoELayer, check_rows

H = 512


def test_check_rows_accepts_and_refuses():
    cpu = torch.device("cpu")
    check_rows(torch.zeros(3, H, dtype=torch.bfloat16), "x", H, cpu)
    with pytest.raises(TypeError):
        check_rows(torch.zeros(3, H, dtype=torch.float32), "x", H, cpu)
    with pytest.raises(TypeError):
        check_rows([[0.0] * H], "x", H, cpu)
    with pytest.raises(ValueError):
        check_rows(torch.zeros(3, H + 8, dtype=torch.bfloat16), "x", H, cpu)
    with pytest.raises(ValueError):
        check_rows(torch.zeros(H, dtype=torch.bfloat16), "x", H, cpu)
    with pytest.raises(ValueError):
        check_rows(torch.zeros(H, 3, dtype=torch.bfloat16).t(), "x", H, cpu)
    with pytest.raises(ValueError):
        check_rows(torch.zeros(3, H, dtype=torch.bfloat16), "x", H, torch.device("cuda"))


def _layer(calls):
    """A MoELayer with its buffers and library calls replaced by recorders."""
    L = object.__new__(MoELayer)
    L.H, L.max_tokens, L.device = H, 8, torch.device("cpu")
    L.mode, L.path, L.E = 0, 0, 256
    L.y = torch.zeros(8, H, dtype=torch.bfloat16)
    L.decode_fused = lambda x, T, *a, **k: calls.append(("fused", T)) or L.y[:T]
    L.route = lambda x, T, *a, **k: calls.append(("route", T))
    L.permute = lambda T, *a, **k: calls.append(("permute", T))
    L.expert_ffn = lambda x, T, *a, **k: calls.append(("ffn", T))
    L.combine = lambda T, *a, **k: calls.append(("combine", T))
    return L


def test_forward_checks_before_any_call():
    calls = []
    L = _layer(calls)
    x = torch.zeros(3, H, dtype=torch.bfloat16)
    L.forward(x)
    assert calls == [("fused", 3)]
    L.forward(x, y_out=torch.zeros(3, H, dtype=torch.bfloat16))
    calls.clear()
    L.forward(x, logits_in=torch.zeros(3, 256))          # given logits take the four calls
    assert [c[0] for c in calls] == ["route", "permute", "ffn", "combine"]
    calls.clear()
    for bad in (x.float(), torch.zeros(3, H - 8, dtype=torch.bfloat16), torch.zeros(H, 3, dtype=torch.bfloat16).t()):
        with pytest.raises((TypeError, ValueError)):
            L.forward(bad)
    with pytest.raises(ValueError):
        L.forward(torch.zeros(9, H, dtype=torch.bfloat16))           # more tokens than the buffers hold
    with pytest.raises(ValueError):
        L.forward(x, y_out=torch.zeros(2, H, dtype=torch.bfloat16))  # too few output rows
    with pytest.raises(TypeError):
        L.forward(x, y_out=torch.zeros(3, H, dtype=torch.float32))
    with pytest.raises(TypeError):
        L.forward(x, logit_bias=torch.zeros(256, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        L.forward(x, logit_bias=torch.zeros(2, 256), bias_stride=256)      # 3 tokens need 3 rows
    with pytest.raises(ValueError):
        L.forward(x, logit_bias=torch.zeros(256), bias_stride=-1)
    with pytest.raises(ValueError):
        L.forward(x, logits_in=torch.zeros(2, 256))
    assert calls == []
    L.forward(x, logit_bias=torch.zeros(256))                              # one row for every token
    L.forward(x, logit_bias=torch.zeros(3, 256), bias_stride=256)          # one row per token
    assert calls == [("fused", 3), ("fused", 3)]
