"""Host-side logic of bench.py that needs no GPU: which fused kernels a workload's line names
(the library's launch rules: persistent forward for head-major launches without key lengths,
more tile pairs than SMs and at most 32 key blocks per tile, causal or not; persistent backward
only without the causal mask and for at most 16 query steps per unit)."""
import bench
import workloads

SMS = 148


def names(B, H, N, d, causal, pad=None, H_kv=None):
    w = workloads.custom(B, H, N, d, causal, seed=1, pad_range=pad, H_kv=H_kv)
    return bench.main_kernels(w, SMS)


def test_default_workload_runs_the_persistent_forward_and_per_unit_backward():
    assert names(4, 16, 4096, 128, False) == ("fa_fwd_persist_kernel", "fa_bwd_kernel")


def test_short_non_causal_runs_both_persistent_kernels():
    assert names(16, 16, 1024, 128, False) == ("fa_fwd_persist_kernel", "fa_bwd_persist_kernel")
    assert names(8, 32, 2048, 64, False) == ("fa_fwd_persist_kernel", "fa_bwd_persist_kernel")


def test_causal_runs_the_persistent_forward_and_per_unit_backward():
    assert names(32, 16, 512, 128, True) == ("fa_fwd_persist_kernel", "fa_bwd_kernel")
    assert names(4, 16, 4096, 128, True) == ("fa_fwd_persist_kernel", "fa_bwd_kernel")


def test_long_sequences_and_key_lengths_run_one_cta_per_unit():
    assert names(2, 16, 8192, 128, False) == ("fa_fwd_kernel", "fa_bwd_kernel")
    assert names(16, 16, 1024, 128, False, pad=(512, 1024)) == ("fa_fwd_kernel", "fa_bwd_kernel")


def test_few_units_run_one_cta_per_unit():
    # 2 * 16 * ceil(1024 / 256) = 128 tile pairs and 2 * 16 * 8 = 256 key blocks
    assert names(2, 16, 1024, 128, False) == ("fa_fwd_kernel", "fa_bwd_persist_kernel")
    assert names(1, 8, 1024, 128, False) == ("fa_fwd_kernel", "fa_bwd_kernel")


def test_grouped_heads_count_query_steps_over_the_group():
    # H / H_kv = 4 query heads per key block: 4 * 8 = 32 steps, above the persistent limit
    assert names(16, 32, 1024, 128, False, H_kv=8)[1] == "fa_bwd_kernel"
    assert names(16, 32, 512, 128, False, H_kv=8)[1] == "fa_bwd_persist_kernel"
