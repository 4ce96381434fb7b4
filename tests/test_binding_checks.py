"""Argument checks of the Python binding, run on the host with stand-in
tensors: the kernels size every access from Q's descriptor, so an `out`,
K, V or conv_w that does not match Q must be refused before any launch."""
import pytest
import torch

import nystr_self_attention_segment_b200 as nys
from nystr_self_attention_segment_b200 import _check_operands


class Fake:
    """Just the attributes the checks read."""

    def __init__(self, shape=(2, 3, 128, 64), dtype=torch.bfloat16, cuda=True, device="cuda:0",
                 contiguous=True):
        self.shape = tuple(shape)
        self.dtype = dtype
        self.is_cuda = cuda
        self.device = torch.device(device)
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)


def conv(heads=3, k=33, **kw):
    kw.setdefault("dtype", torch.float32)
    return Fake(shape=(heads, k), **kw)


def test_matching_operands_pass():
    Q = Fake()
    _check_operands(Q, Fake(), Fake(), Fake(), conv())
    _check_operands(Q, Fake(), Fake(), Fake(), None)
    H = dict(cuda=False, device="cpu")
    _check_operands(Fake(**H), Fake(**H), Fake(**H), Fake(**H), conv(**H), on_cuda=False)


@pytest.mark.parametrize("bad", [
    dict(shape=(2, 3, 64, 64)),          # shorter sequence: the kernels would write past it
    dict(shape=(2, 3, 128, 32)),
    dict(dtype=torch.float32),
    dict(device="cuda:1"),
    dict(cuda=False, device="cpu"),
    dict(contiguous=False),
])
@pytest.mark.parametrize("which", ["K", "V", "out"])
def test_mismatched_operand_is_refused(bad, which):
    ops = {"K": Fake(), "V": Fake(), "out": Fake()}
    ops[which] = Fake(**bad)
    with pytest.raises(ValueError, match=which):
        _check_operands(Fake(), ops["K"], ops["V"], ops["out"], None)


@pytest.mark.parametrize("bad", [
    dict(heads=2),
    dict(dtype=torch.bfloat16),
    dict(device="cuda:1"),
    dict(cuda=False, device="cpu"),
    dict(contiguous=False),
])
def test_mismatched_conv_weights_are_refused(bad):
    with pytest.raises(ValueError, match="conv_w"):
        _check_operands(Fake(), Fake(), Fake(), Fake(), conv(**bad))


def test_host_entry_wants_host_operands():
    with pytest.raises(ValueError, match="CPU"):
        _check_operands(Fake(), Fake(), Fake(), Fake(), None, on_cuda=False)


def test_cpu_tensors_are_refused_by_the_device_entry():
    Q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        nys.nys_attn_forward(Q, Q, Q, 64)
