"""The bench's kernel-launch claims (`gpu_launches`) against the launch lists
ncu recorded for the same workloads (summaries under profiles/): one d20
forward is 147 kernels, 231 with every product in e4m3."""
import bench


def test_forward_kernel_counts_match_the_launch_lists():
    L = 20
    # trace entries of one forward with targets and loss (nc_forward_traced)
    plain = 3 + 7 * L + 1 + 3
    assert bench.kernels_per_step(plain, L, 0, 0) == 147
    fp8_all = plain + 4 * L + 1  # four activation quantisations per layer, one before the LM head
    assert bench.kernels_per_step(fp8_all, L, 3, 0) == 231
    fp8_block = plain + 4 * L
    # block only: 120 e4m3 weights (two amax + quantise batches) and the 16-bit lm_head cast
    assert bench.kernels_per_step(fp8_block, L, 1, 0) == fp8_block + 4


def test_unfused_activation_quantisations_add_an_amax_launch():
    L = 4
    base = 3 + 7 * L + 1 + 3 + 4 * L + 1
    fused = bench.kernels_per_step(base, L, 3, 0)
    assert bench.kernels_per_step(base, L, 3, 4) == fused + L      # x0 mixing in every first norm
    assert bench.kernels_per_step(base, L, 3, 8) == fused + 2      # backout: one first norm + the final norm
    assert bench.kernels_per_step(base, L, 1, 8) == bench.kernels_per_step(base, L, 1, 0) + 1



def test_training_extras_kernel_counts():
    """The further terms' backward kernels of one training micro-step, item by
    item for four layers with tables on layers 1 and 3 (the trace records none
    of them)."""
    L, n_ve = 4, 2
    backout_dot = 1
    ve_bwd = n_ve
    lambda_dots, mixes, final_mix = L, L, 1  # the middle block's mix also carries the backout term
    smear = 2  # per-token pass, then the gate's weight gradient
    assert bench.train_extra_kernels(L, n_ve, 15) == backout_dot + ve_bwd + lambda_dots + mixes + final_mix + smear
    assert bench.train_extra_kernels(L, n_ve, 0) == 0
    assert bench.train_extra_kernels(L, n_ve, 8) == 2  # backout alone: its dot and one mix
    assert bench.train_extra_kernels(L, n_ve, 2) == n_ve


def test_training_claim_matches_the_recorded_launch_list():
    """One d20 training step with every term: 492 trace entries (the 40
    residual copies launch no kernel, the 20 attention backwards three kernels
    each) plus the terms' untraced backward kernels are the 546 library kernels
    ncu recorded for one step (profiles/launches_d20_train_extras_b8.md)."""
    L, n_ve = 20, 10
    entries = 12 + 24 * L
    assert entries - 2 * L + 2 * L == 492
    assert entries + bench.train_extra_kernels(L, n_ve, 15) == 546
