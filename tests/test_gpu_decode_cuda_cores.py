"""The decode parity suite again with the CUDA-core score product selected
(yocopp_set_decode_kernel(1)).  By default bf16 / head_dim 128 caches use the
tcgen05 score product (test_gpu_decode.py covers that); this module keeps the
packed-FMA kernel, which also serves fp32 and head_dim 64, under the same
parity bar on every shape."""
import pytest

import test_gpu_decode as base
import test_gpu_e2e as e2e

pytestmark = pytest.mark.gpu

y = base.y
orc = base.orc


@pytest.fixture(autouse=True)
def cuda_core_scores():
    import decode_attention_yocopp_b200 as yy
    yy.load()
    yy.yocopp_set_decode_kernel(yy.DECODE_CUDA_CORES)
    yield
    yy.yocopp_set_decode_kernel(yy.DECODE_DEFAULT)


test_cc_edge_lengths_contiguous = base.test_edge_lengths_contiguous
test_cc_edge_lengths_paged_block16 = base.test_edge_lengths_paged_block16
test_cc_config2_shape_contiguous = base.test_config2_shape_contiguous
test_cc_ragged_paged_block64 = base.test_ragged_paged_block64
test_cc_paged_block128_group2 = base.test_paged_block128_group2
test_cc_paged_block32_group1 = base.test_paged_block32_group1
test_cc_head_dim_64_bf16 = base.test_head_dim_64_bf16
test_cc_fp32_tiny_shape = base.test_fp32_tiny_shape
test_cc_peaked_softmax = base.test_peaked_softmax
test_cc_explicit_scale = base.test_explicit_scale
test_cc_planted_key = base.test_planted_key
test_cc_length_above_capacity = base.test_length_above_capacity_is_clamped_and_flagged
test_cc_unzeroed_workspace = base.test_unzeroed_workspace_is_reported
test_cc_e2e_b4_t4096 = e2e.test_b4_t4096_full
test_cc_e2e_full_size = e2e.test_full_size_sampled
