"""Host-side arithmetic of bench.py (no GPU): the algorithmic byte and FLOP
counts the roofline divides by, checked against closed forms written out by
hand for the workloads' shapes, and the whole-job throughput rule."""

import bench
from delta_rule_linear_gdn_b200.inputs import workload

TOK = 32768            # the headline prefill: one sequence of 32768 tokens
HQK, HV, D = 16, 48, 128


def test_prefill_bytes_headline_and_gate_layouts():
    w = workload("prefill_t32768")
    qk = TOK * HQK * D * 2 * 2          # q and k, bf16
    v = TOK * HV * D * 2                # v, bf16
    o = TOK * HV * D * 2                # o, bf16
    st = HV * D * D * 4                 # S_T, fp32 (S0 = 0 is not read)
    gates_v = TOK * HV * D * 4 * 3      # alpha, b, w per value head, fp32
    assert bench.prefill_bytes(w) == qk + v + o + st + gates_v == 3_492_806_656
    # bf16 logits: half the gate bytes
    assert bench.prefill_bytes(w, gate_bytes=2) == qk + v + o + st + gates_v // 2
    # alpha and b per QK head (16 instead of 48), w per value head
    gates_qk = TOK * (2 * HQK + HV) * D * 4
    assert bench.prefill_bytes(w, qk_gates=True) == qk + v + o + st + gates_qk == 2_419_064_832


def test_prefill_flops_closed_form():
    # 6 d^2 + 5 C d per token and value head (C = 64)
    w = workload("prefill_t32768")
    assert bench.prefill_flops(w) == TOK * HV * (6 * D * D + 5 * 64 * D) == 219_043_332_096


def test_decode_bytes_closed_form():
    w = workload("decode_b256")
    state = 256 * HV * D * D * 4 * 2                         # read and written once
    io = 256 * HQK * D * 2 * 2 + 256 * HV * D * 2 + 256 * HV * D * 4 * 3 + 256 * HV * D * 2
    assert bench.decode_bytes(w) == state + io


def test_weak_scaling_value_and_config_note():
    # every rank processes its own sequence: N ranks, the slowest rank's time
    assert bench.weak_value(32768, 4, 2.0) == 32768 * 4 / 2e-3
    note = bench.config_dict(workload("prefill_t32768"))["l2"]
    assert "3.49 GB" in note and "126 MB" in note


def test_tied_gate_bytes_and_backward_flops():
    w = workload("prefill_t32768")
    qk, v, o, st = TOK * HQK * D * 2 * 2, TOK * HV * D * 2, TOK * HV * D * 2, HV * D * D * 4
    # KDA: alpha per channel, beta one scalar per (token, value head)
    assert bench.prefill_bytes(w, gate_mode="kda") == qk + v + o + st + TOK * HV * (D + 1) * 4
    # Gated DeltaNet: alpha and beta scalars
    assert bench.prefill_bytes(w, gate_mode="gdn") == qk + v + o + st + TOK * HV * 2 * 4
    # backward: 18 d^2 per token and value head (B=8, T=8192)
    bw = workload("conv_prefill_b8_t8192")
    assert bench.bwd_flops(bw) == 8 * 8192 * HV * 18 * D * D


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    """`roofline.traffic` comes from an ncu capture of particular kernel
    sources: it is reported while the sources hash to the captured ones and
    is null once they change (or when no capture is recorded)."""
    sha = bench.kernel_sources_sha1()
    assert len(sha) == 40 and sha == bench.kernel_sources_sha1()   # stable over reads
    monkeypatch.setitem(bench.TRAFFIC, "sha1", sha)
    monkeypatch.setitem(bench.TRAFFIC, "bytes_per_call", 123456)
    assert bench.measured_traffic() == 123456
    monkeypatch.setitem(bench.TRAFFIC, "sha1", "0" * 40)
    assert bench.measured_traffic() is None
    monkeypatch.setitem(bench.TRAFFIC, "sha1", None)
    assert bench.measured_traffic() is None
