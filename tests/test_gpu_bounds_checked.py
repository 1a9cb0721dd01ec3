"""The bounds-checked build (libgated_delta_checked.so, the sanitizer
substitute): every index its kernels compute for a global access of their own
is compared with the extent of its buffer; a violation is counted and the
access skipped.  A selection of the GPU parity tests (the four timed workloads at full size
among them) runs through that build:
each must still match the oracle and leave the violation count at zero.
Covers every kernel: the planning kernel, the tensor-core prep and scan, the
fp32 path, the token-by-token kernel, the state copies."""
import importlib

import pytest

import gated_delta_rule_87_b200 as gdr

pytestmark = pytest.mark.gpu

CASES = [
    ("test_gpu_prefill", "test_kda_ragged_lengths", dict(io="bf16", T=130)),
    ("test_gpu_prefill", "test_kda_ragged_lengths", dict(io="f32", T=65)),
    ("test_gpu_prefill", "test_kda_head_sizes", dict(dk=64, dv=128)),
    ("test_gpu_prefill", "test_kda_dense_batch", {}),
    ("test_gpu_prefill", "test_kda_packed_with_empty_sequences", dict(io="bf16")),
    ("test_gpu_prefill", "test_kda_packed_with_empty_sequences", dict(io="f32")),
    ("test_gpu_prefill", "test_gdn_packed_sequences", {}),
    ("test_gpu_prefill", "test_gdn_dense_batch_ragged_tail", {}),
    ("test_gpu_prefill", "test_kda_steep_decays", dict(scale=1.5, order="erase_then_decay", mixed=True)),
    ("test_gpu_prefill", "test_kda_column_slice_widths", dict(nseq=20)),
    ("test_gpu_prefill", "test_split_prefill_carries_state", {}),
    ("test_gpu_decay_order", "test_variant_packed_with_empty_sequences", dict(io="bf16")),
    ("test_gpu_decode", "test_kda_decode_small", dict(io="bf16", dk=128, dv=64)),
    ("test_gpu_decode", "test_gdn_decode_shared_heads", dict(io="f32")),
    ("test_gpu_recurrent", "test_kda_tokens_per_sequence", dict(order="erase_then_decay", io="bf16", T=7)),
    ("test_gpu_recurrent", "test_state_pool_slots_and_padding", dict(order="decay_then_erase")),
    ("test_gpu_recurrent", "test_slot_past_pool_end_is_padding", {}),
    ("test_gpu_state_pool", "test_prefill_updates_pool_in_place", dict(io="bf16", gate="channel")),
    ("test_gpu_state_pool", "test_gather_scatter_are_exact_copies", {}),
    ("test_gpu_state_pool", "test_empty_prefill_leaves_pool_unchanged", {}),
    # the timed workloads at full size
    ("test_gpu_prefill", "test_kda_prefill_full_workload", {}),
    ("test_gpu_prefill", "test_kda_varlen_full_workload_sampled_heads", {}),
    ("test_gpu_prefill", "test_gdn_long_full_workload_sampled_heads", {}),
    ("test_gpu_decode", "test_kda_decode_full_size_sampled", {}),
    ("test_gpu_host_stream", "test_streamed_prefill_equals_device_call",
     dict(io="bf16", B=2, T=1000, pieces=3)),
]


@pytest.mark.parametrize("mod,fn,kw", CASES, ids=[f"{f}-{'-'.join(map(str, k.values()))}"
                                                  for _, f, k in CASES])
def test_checked_build_matches_oracle_with_no_violation(mod, fn, kw):
    test = getattr(importlib.import_module(mod), fn)
    with gdr.use_library(gdr.checked_library_path):
        assert gdr.bounds_checked()
        gdr.bounds_violations()  # start from zero
        test(**kw)
        assert gdr.bounds_violations() == 0
    assert not gdr.bounds_checked()  # back on the normal build
