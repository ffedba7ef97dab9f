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
    L.mode, L.path, L.E, L.I = 0, 0, 256, 512
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


def test_check_weights():
    import numpy as np
    import gen
    from bit_dequant_expert_b200.layer import check_weights
    lay = gen.make_weights(gen.config(0))
    assert check_weights(lay) == (256, 512, 128)
    assert check_weights(gen.make_weights(gen.LayerSpec(T=1, H=1024, I=256))) == (256, 1024, 256)
    as_tensors = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16
                  else torch.from_numpy(v.view(np.int32)) for k, v in lay.items()}
    assert check_weights(as_tensors) == (256, 512, 128)
    bad = [("d_codes", lay["d_codes"][:, :-8]), ("gu_sb", lay["gu_sb"][:, :, :-1]),
           ("w_router", lay["w_router"][:-1]), ("d_sb", lay["d_sb"].astype(np.float32))]
    for name, arr in bad:
        with pytest.raises((ValueError, TypeError)):
            check_weights(dict(lay, **{name: arr}))
    with pytest.raises(ValueError):
        check_weights({k: v for k, v in lay.items() if k != "d_sb"})
    with pytest.raises(TypeError):
        check_weights(dict(lay, w_router=lay["w_router"].astype(np.float32)))
