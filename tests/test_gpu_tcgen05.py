"""The grouped / multi-token decode on the tcgen05 consumer (pa_set_grouped_consumer):
one thread issues 5th-generation tensor-core MMAs (S = Q K^T and O += P V, S and
O in tensor memory, P in shared memory) for four softmax warps that split each
64-token unit; over FP8 / int8 codes two converter warps turn each unit into f16
tiles first. The same oracle parity (full-size configurations included),
bitwise invariants and bounded-wait behaviour as the default consumer, re-run
with this one selected (the test functions are those of the default consumer's
modules); shapes it does not take fall back to the default consumer."""
import pytest
import torch

import paged_kv_cache_335_b200 as pa
from paged_kv_cache_335_b200 import workloads as W
from tests import gpu_helpers as G
from tests.test_gpu_grouped import (test_bad_block_id_is_reported,  # noqa: F401
                                    test_cow_beam4_full_size,
                                    test_cow_small_full_pool,
                                    test_deterministic_repeat,
                                    test_long_shared_context_many_partitions,
                                    test_members_sharing_blocks_with_different_lengths,
                                    test_members_with_empty_contexts,
                                    test_placement_invariance_bitwise,
                                    test_shared_equals_private_bitwise,
                                    test_unshared_shape_sweep_edges)
from tests.test_gpu_multi import (test_parity_shape_sweep,  # noqa: F401
                                  test_token_result_independent_of_the_other_tokens,
                                  test_verification_full_size)
from tests.test_gpu_quant import test_q_magnitudes_outside_f16_range  # noqa: F401
from tests.test_gpu_quant_grouped import (test_full_size as test_codes_full_size,  # noqa: F401
                                          test_grouped_cow_parity,
                                          test_grouped_shared_equals_private_bitwise,
                                          test_grouped_unshared_edges, test_multi_parity)
from tests.test_gpu_scale_sign import test_negative_scale_codes  # noqa: F401
from tests.test_gpu_timeout import test_skipped_load_times_out_then_recovers  # noqa: F401

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(autouse=True)
def tcgen05_consumer():
    prev = pa.pa_set_grouped_consumer(pa.PA_GROUPED_TCGEN05)
    yield
    pa.pa_set_grouped_consumer(prev)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_selector_takes_the_tcgen05_path_over_codes(fmt):
    wl = W.quantized(W.cow_beam4(num_prompts=2, prompt_len=100, max_suffix=20, num_heads=16,
                                 num_kv_heads=2, head_dim=128), fmt)
    vals = W.make_values(wl, DEV)
    d = G.device_tensors(wl, vals)
    out = torch.empty_like(vals["q"])
    pa.pa_decode_grouped_quant(out, vals["q"], vals["k_cache"], vals["v_cache"], vals["k_scale"],
                               vals["v_scale"], d["tables"], d["ctx"], wl.scale, 4,
                               max_context_len=wl.max_context_len)
    pa.pa_sync_check()
    assert G.last_kernel() == pa.PA_KERNEL_GROUPED_TCGEN05


def test_selector_takes_the_tcgen05_path():
    wl = W.cow_beam4(num_prompts=2, prompt_len=100, max_suffix=20, num_heads=16, num_kv_heads=2,
                     head_dim=128)
    vals = W.make_values(wl, DEV)
    G.gpu_step(wl, vals, partition_size=0, group_size=4)
    pa.pa_sync_check()
    assert G.last_kernel() == pa.PA_KERNEL_GROUPED_TCGEN05
    with pytest.raises(pa.PAError):
        pa.pa_set_grouped_consumer(7)
