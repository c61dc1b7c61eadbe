"""CPU checks of the PyTorch custom ops' fake (shape) implementations: the
shapes and dtypes torch.compile sees must be those the library writes."""
import torch
from torch._subclasses.fake_tensor import FakeTensorMode

from grouped_gemm_route_b200 import moe as M
from grouped_gemm_route_b200 import torch_op as TO


def test_forward_and_backward_fakes_match_the_library_sizes():
    T, d, E, k, I = 300, 256, 8, 2, 128
    sizes, p_cap = M.saved_sizes(M.make_shape(T, d, E, k, I))
    with FakeTensorMode():
        x = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        lg = torch.empty(T, E, dtype=torch.float32, device="cuda")
        wgu = torch.empty(E, 2 * I, d, dtype=torch.bfloat16, device="cuda")
        wd = torch.empty(E, d, I, dtype=torch.bfloat16, device="cuda")
        outs = TO.moe_forward(x, lg, wgu, wd, k, M.MOE_BF16, 0.0)
        assert tuple(outs[0].shape) == (T, d) and outs[0].dtype == torch.bfloat16
        for name, t, nbytes in zip(M.SAVED_FIELDS, outs[1:], sizes):
            assert t.numel() * t.element_size() == nbytes, name
        assert outs[M.SAVED_FIELDS.index("perm") + 1].shape[0] == p_cap
        g = TO.moe_backward(outs[0], x, wgu, wd, *outs[1:], k, M.MOE_BF16, 0.0)
        assert [tuple(t.shape) for t in g] == [(T, d), (T, E), (E, 2 * I, d), (E, d, I), (T, k)]
        assert [t.dtype for t in g] == [torch.bfloat16, torch.float32, torch.bfloat16, torch.bfloat16,
                                        torch.float32]


def test_input_checks_reject_bad_dtypes_shapes_top_k_and_devices():
    import pytest
    T, d, E, I = 8, 256, 4, 128
    x = torch.empty(T, d, dtype=torch.bfloat16)
    lg = torch.empty(T, E, dtype=torch.float32)
    wgu = torch.empty(E, 2 * I, d, dtype=torch.bfloat16)
    wd = torch.empty(E, d, I, dtype=torch.bfloat16)
    TO._check_inputs(x, lg, wgu, wd, 2)  # a valid set passes
    with pytest.raises(TypeError):
        TO._check_inputs(x.float(), lg, wgu, wd, 2)
    with pytest.raises(TypeError):
        TO._check_inputs(x, lg.double(), wgu, wd, 2)
    with pytest.raises(ValueError):
        TO._check_inputs(x, lg[:, :3], wgu, wd, 2)
    with pytest.raises(ValueError):
        TO._check_inputs(x, lg, wgu, wd.transpose(1, 2), 2)
    for k in (0, E + 1):
        with pytest.raises(ValueError):
            TO._check_inputs(x, lg, wgu, wd, k)
    with pytest.raises(ValueError, match="one device"):
        TO._check_inputs(x, lg, wgu, wd.to("meta"), 2)
