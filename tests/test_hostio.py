"""HostGroupedQuantizer argument checks that run before any device work."""
import pytest
import torch

import nvfp4_quantization_aware_b200 as Q


def test_rejects_unpinned_or_misshaped_inputs_and_bad_pass_orders():
    x = torch.zeros(4, 32, dtype=torch.bfloat16)  # not pinned
    with pytest.raises(ValueError):
        Q.HostGroupedQuantizer([x], "cpu")
    with pytest.raises(ValueError):
        Q.HostGroupedQuantizer([], "cpu")


def test_rejects_bad_pass_orders_widths_and_mixed_dtypes():
    # these checks need no device; a stand-in that reports itself pinned gets
    # past the pinning check on a machine without CUDA
    class Pinned(torch.Tensor):
        def is_pinned(self):
            return True

    x = torch.zeros(4, 32, dtype=torch.bfloat16).as_subclass(Pinned)
    with pytest.raises(ValueError):
        Q.HostGroupedQuantizer([x], "cpu", passes=(Q.FROZEN_ALL,))
    with pytest.raises(ValueError):
        Q.HostGroupedQuantizer([x], "cpu", passes=(Q.FROZEN_GLOBAL,))
    with pytest.raises(ValueError):
        Q.HostGroupedQuantizer([x], "cpu", passes=())
    y = torch.zeros(4, 33, dtype=torch.bfloat16).as_subclass(Pinned)
    with pytest.raises(ValueError):
        Q.HostGroupedQuantizer([y], "cpu")
    z = torch.zeros(4, 32, dtype=torch.float32).as_subclass(Pinned)
    with pytest.raises(ValueError):
        Q.HostGroupedQuantizer([x, z], "cpu")
