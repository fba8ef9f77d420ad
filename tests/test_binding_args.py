"""The Python binding checks the tensors it turns into raw pointers: the library trusts
their sizes, so a wrong shape, dtype, layout or device is rejected on the host before any
entry point is called (runs without a GPU: the library is replaced by a recorder)."""

import pytest
import torch

from mixture_experts_layer_sort_b200.layer import MoELayer


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append(name)
            return 0
        return call


def _layer(E=8, k=2, H=256, I=512):
    lay = object.__new__(MoELayer)
    lay.lib = _Recorder()
    lay.E, lay.k, lay.H, lay.I, lay.dtype = E, k, H, I, 0
    lay.handle = None
    return lay


def _host(M, E=8, H=256):
    return (torch.zeros((M, H), dtype=torch.bfloat16), torch.zeros((M, E), dtype=torch.float32),
            torch.zeros((M, H), dtype=torch.bfloat16))


def test_host_forward_passes_well_formed_tensors():
    lay = _layer()
    for M in (0, 1, 5):
        lay.forward_host(*_host(M), stream=0)
    assert lay.lib.calls == ["moe_forward_host"] * 3


@pytest.mark.parametrize("what", ["x_dtype", "x_width", "x_strided", "logits_dtype", "logits_rows", "logits_width",
                                  "out_dtype", "out_rows", "x_3d"])
def test_host_forward_rejects_malformed_tensors(what):
    lay = _layer()
    x, logits, out = _host(4)
    if what == "x_dtype":
        x = x.float()
    elif what == "x_width":
        x = torch.zeros((4, 128), dtype=torch.bfloat16)
    elif what == "x_strided":
        x = torch.zeros((8, 256), dtype=torch.bfloat16)[::2]
    elif what == "logits_dtype":
        logits = logits.double()
    elif what == "logits_rows":
        logits = torch.zeros((3, 8), dtype=torch.float32)
    elif what == "logits_width":
        logits = torch.zeros((4, 16), dtype=torch.float32)
    elif what == "out_dtype":
        out = out.float()
    elif what == "out_rows":
        out = torch.zeros((5, 256), dtype=torch.bfloat16)
    elif what == "x_3d":
        x = torch.zeros((4, 1, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lay.forward_host(x, logits, out)
    assert lay.lib.calls == []


def test_device_entry_points_reject_host_tensors():
    lay = _layer()
    x, logits, out = _host(4)
    with pytest.raises(ValueError, match="device memory"):
        lay.forward(x, logits, out=out)
    with pytest.raises(ValueError, match="device memory"):
        lay.forward_noalloc(x, logits, out)
    assert lay.lib.calls == []


def test_inv_rope_rejects_malformed_tensors():
    from mixture_experts_layer_sort_b200.layer import inv_rope_fp8_quant
    x = torch.zeros((4, 2, 128), dtype=torch.bfloat16)
    pos = torch.zeros(4, dtype=torch.int32)
    tab = torch.zeros((16, 128), dtype=torch.float32)
    with pytest.raises(ValueError, match="x must be"):
        inv_rope_fp8_quant(x.float(), pos, tab)
    with pytest.raises(ValueError, match="positions must be"):
        inv_rope_fp8_quant(x, pos.long(), tab)
    with pytest.raises(ValueError, match="cos_sin must be"):
        inv_rope_fp8_quant(x, pos, torch.zeros((16, 64), dtype=torch.float32))
    with pytest.raises(ValueError, match="device memory"):    # well formed, but on the host
        inv_rope_fp8_quant(x, pos, tab)


def test_weight_loads_reject_malformed_tensors():
    lay = _layer()
    E, H, I = 8, 256, 512
    host = [torch.zeros(s, dtype=torch.bfloat16) for s in ((E, I, H), (E, I, H), (E, H, I))]
    with pytest.raises(ValueError, match="w_gate must be"):          # host memory
        lay.load_weights(*host)
    with pytest.raises(ValueError, match="w_gate must be"):
        lay.load_weights_mixed(*host, [True] * E)
    with pytest.raises(ValueError, match="w_gate must be"):          # the full tensors of 2 shards
        lay.load_weights_shard(*host, 0, 2)
    with pytest.raises(ValueError, match="w_gate must be"):          # codes are uint8
        lay.load_weights_fp8(*host, torch.ones(E, 3))
    assert lay.lib.calls == []
