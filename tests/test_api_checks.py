"""Host-side argument checks of the Python API (no GPU needed): a tensor of
the wrong dtype, shape or layout, or one in host memory, is refused before
any kernel sees its address."""
import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt


def test_check_tensor_refuses_each_kind_of_mismatch():
    shape = (1, 2, 64, 64)
    good = torch.zeros(shape, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="torch.Tensor"):
        dt.check_tensor([0], "Q", shape, (torch.bfloat16,))
    with pytest.raises(TypeError, match="dtype"):
        dt.check_tensor(good.float(), "Q", shape, (torch.bfloat16,))
    with pytest.raises(ValueError, match="shape"):
        dt.check_tensor(good[:, :1], "Q", shape, (torch.bfloat16,))
    with pytest.raises(ValueError, match="last dimension"):
        dt.check_tensor(torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16)[..., ::2], "Q", shape,
                        (torch.bfloat16,))
    with pytest.raises(ValueError, match="contiguous"):
        dt.check_tensor(torch.zeros((1, 64, 2), dtype=torch.float32).permute(0, 2, 1), "out_lse",
                        (1, 2, 64), (torch.float32,), contiguous=True)
    # right dtype, shape and layout, but in host memory
    with pytest.raises(ValueError, match="CUDA device"):
        dt.check_tensor(good, "Q", shape, (torch.bfloat16,))
    # strided views with a contiguous last dimension pass every check but the device
    view = torch.zeros((1, 64, 3, 2, 64), dtype=torch.bfloat16)[:, :, 0].permute(0, 2, 1, 3)
    with pytest.raises(ValueError, match="CUDA device"):
        dt.check_tensor(view, "Q", shape, (torch.bfloat16,))


def test_host_tensors_never_reach_the_library():
    g = dt.Geometry(1, 2, 64, 64, [0, 32, 64])
    host = torch.zeros(16, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dt.ditango_plan(g, None, None, 0, 1.0, 1, host, host, host, stream=0)


def test_state_cache_must_live_on_a_cuda_device():
    with pytest.raises(ValueError, match="CUDA device"):
        dt.PartitionedAttention(1, 2, 64, 64, [0, 32, 64], device="cpu")
