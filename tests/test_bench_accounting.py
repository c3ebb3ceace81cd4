"""bench.py's measurement definitions on the CPU: the algorithmic bytes of a step (the roofline
numerator) and the count of kernel launches it claims, against values computed from the
workload's shapes."""
import bench
from workload import configs, inputs


def test_step_bytes_of_the_128k_workload():
    wl = configs.cfg2()
    per_token = wl.Hkv * 128 * 2 * 2                 # K and V, bf16, all KV heads
    assert per_token == 4096
    t = 131073
    local = 4 * 2052 * per_token * 36                 # |S^L| = 4 sinks + 2048 window
    full = t * per_token * 36                         # one flagged sequence, every layer
    head = 34_623_489 * 4                             # fp32 recall head at D = 4096
    assert inputs.head_param_count(wl.D) == 34_623_489
    assert bench.step_bytes(wl, [t] * 4, [0, 0, 1, 0]) == local + full + head
    assert bench.step_bytes(wl, [t] * 4, [0] * 4) == local + head
    # the local part is the 36 x 4 x 8.40 MB of the expected step
    assert abs(local / 1e6 - 36 * 4 * 8.405) < 1.0   # MB


def test_step_bytes_short_context_reads_every_position():
    wl = configs.cfg2()
    # t <= 2052: the local set is every position, and equals the full set
    assert bench.step_bytes(wl, [100] * 4, [1, 0, 0, 0]) == (
        4 * 100 * 4096 * 36 + 100 * 4096 * 36 + inputs.head_param_count(wl.D) * 4)


def test_launch_counts():
    wl = configs.cfg2()
    assert bench.head_launches(wl) == 1
    assert bench.head_launches(configs.cfg3()) == 6
    # 36 local launches, the hidden-state glue, the head, set-condition, commit
    assert bench.kernel_launches(wl, False) == 36 + 1 + 1 + 1 + 1
    # plus 36 full-set launches and the retry's hidden-state glue when the IF node fires
    assert bench.kernel_launches(wl, True) == 40 + 36 + 1


def test_step_bytes_of_the_hybrid_stack_count_the_state_each_pass_moves():
    wl = configs.cfg4()
    per_seq = 18 * (16 * 128 * 128 + 4 * 2048) * 4            # 18 recurrent layers, fp32
    assert bench.hybrid_state_bytes(wl) == per_seq
    t = 65537
    kv = wl.Hkv * 128 * 2 * 2
    local = 8 * 2052 * kv * 6 + 8 * 2 * per_seq               # every sequence: read + write
    full = 2 * (t * kv * 6 + 2 * per_seq)                     # two flagged sequences
    head = inputs.head_param_count(wl.D) * 4
    flags = [1, 0, 0, 1, 0, 0, 0, 0]
    assert bench.step_bytes(wl, [t] * 8, flags) == local + full + head
    # fp8 pages: 264 bytes per token and KV head
    assert bench.step_bytes(configs.cfg2(), [100] * 4, [0] * 4, "fp8") == (
        4 * 100 * 8 * 264 * 36 + inputs.head_param_count(4096) * 4)
    # a hybrid step launches no snapshot or restore kernels
    assert bench.kernel_launches(wl, True) == bench.kernel_launches(wl, False) + 24 + 1
