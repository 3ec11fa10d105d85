"""The Python binding refuses tensors too small for a call before anything reaches the
library (the C calls cannot see device buffer sizes). Runs without a GPU: the shape
checks come before the device checks."""
import pytest
import torch

import dispatch_combine_topk_b200 as mep


def z(*shape, dtype=torch.int32):
    return torch.zeros(shape, dtype=dtype)


def test_dispatch_and_combine_shapes():
    x = z(4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="pos must hold"):
        mep.mep_dispatch(x, z(7), 2, z(8, 8, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="recv must be"):
        mep.mep_dispatch(x, z(8), 2, z(8, 16, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="recv_scale"):
        mep.mep_dispatch(x, z(8), 2, z(8, 8, dtype=torch.int8), z(3, dtype=torch.float32), quant=1)
    out = z(4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="pos and gates"):
        mep.mep_combine(z(8, 8, dtype=torch.bfloat16), z(8), z(7, dtype=torch.float32), 2, out)
    with pytest.raises(ValueError, match="y must be"):
        mep.mep_combine(z(8, 4, dtype=torch.bfloat16), z(8), z(8, dtype=torch.float32), 2, out)
    with pytest.raises(ValueError, match="y_scale"):
        mep.mep_combine_int8(z(8, 8, dtype=torch.int8), z(2, dtype=torch.float32), z(8),
                             z(8, dtype=torch.float32), 2, out)
    with pytest.raises(ValueError, match="residual"):
        mep.mep_combine_add_rmsnorm(z(8, 8, dtype=torch.bfloat16), z(8), z(8, dtype=torch.float32), 2,
                                    z(4, 7, dtype=torch.bfloat16), z(8, dtype=torch.bfloat16), 1e-6, out,
                                    z(4, 8, dtype=torch.bfloat16), z(4, dtype=torch.float32))


def test_plan_mapping_and_dedup_shapes():
    pb = mep.PlanBuffers(z(16), z(4), z(3), z(2), z(2), z(2, 4), z(2, 5), z(8), z(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="keep"):
        mep.mep_plan(z(16), 2, 4, 4, 2, pb, mode=mep.MEP_PLAN_GROUPED, keys_per_rank=2,
                     keep=z(15, dtype=torch.uint8))
    small = mep.PlanBuffers(z(15), z(4), z(3), z(2), z(2), z(2, 4), z(2, 5), z(8), z(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="plan buffers"):
        mep.mep_plan(z(16), 2, 4, 4, 2, small)
    with pytest.raises(ValueError, match="hist"):
        mep.mep_histogram(z(16), 8, z(7))
    ids = z(4, 2)
    with pytest.raises(ValueError, match="expert_scales"):
        mep.mep_update_expert(ids, z(4, 3), z(4, 3, dtype=torch.float32), z(2, dtype=torch.float32), None, 0, 2,
                              0, z(4, 2), z(4, 2, dtype=torch.uint8))
    with pytest.raises(ValueError, match="active_mask"):
        mep.mep_update_expert(ids, z(4, 3), z(4, 2, dtype=torch.float32), z(2, dtype=torch.float32),
                              z(3, dtype=torch.uint8), 0, 2, 0, z(4, 2), z(4, 2, dtype=torch.uint8))
    with pytest.raises(ValueError, match="outputs"):
        mep.mep_update_expert(ids, z(4, 3), None, None, None, 0, 2, 0, z(4, 1), z(4, 2, dtype=torch.uint8))
    with pytest.raises(ValueError, match="world_size blocks"):
        mep.mep_update_expert_ranks(z(5, 2), z(4, 3), None, None, None, 2, 0, z(5, 2),
                                    z(5, 2, dtype=torch.uint8))
    db = mep.DedupBuffers(z(15), z(16), z(3), z(16), z(16), z(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="dedup buffers"):
        mep.mep_dedup_plan(z(16), z(3), 2, 4, 2, db)
    with pytest.raises(ValueError, match="int8 rows need"):
        mep.mep_expand(z(4, 8, dtype=torch.int8), z(6), z(6, 8, dtype=torch.int8))
    with pytest.raises(ValueError, match="same dtype"):
        mep.mep_expand(z(4, 8, dtype=torch.bfloat16), z(6), z(6, 8, dtype=torch.int8))


def test_weight_side_shapes():
    pb = mep.PlanBuffers(z(16), z(4), z(3), z(2), z(2), z(2, 4), z(2, 5), z(8), z(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="slot_expert"):
        mep.mep_prefetch_plan(pb, 2, 4, 2, z(3), z(2, 4))
    with pytest.raises(ValueError, match="rep_weight"):
        mep.mep_prefetch_plan(pb, 2, 4, 2, z(4), z(2, 3))
    with pytest.raises(ValueError, match="w_slots"):
        mep.mep_prefetch_weights(z(4, 6, dtype=torch.bfloat16), z(4), 2, 2, z(3, 6, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="grad_slots"):
        mep.mep_grad_reduce(z(4, 6, dtype=torch.float32), z(3, 6, dtype=torch.float32), z(4), 2, 2)
    with pytest.raises(ValueError, match="smooth"):
        mep.mep_dispatch_int8_smooth(z(4, 8, dtype=torch.bfloat16), z(8), z(8), 2, z(3, 7, dtype=torch.float32),
                                     z(8, 8, dtype=torch.int8), z(8, dtype=torch.float32))
