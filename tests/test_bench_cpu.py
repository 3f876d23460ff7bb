"""Host-side pieces of bench.py: the code-only source hash that decides
whether recorded DRAM traffic still applies, and the end-to-end staging
layout (views into one contiguous slab per direction)."""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_code_only_ignores_comments_and_whitespace():
    a = "int x = 1; // note\n/* block\n comment */ float y = 2.0f;\n"
    b = "int  x = 1;\n\n  float y = 2.0f; // other note\n"
    assert bench._code_only(a) == bench._code_only(b)


def test_code_only_keeps_code_and_literals():
    assert bench._code_only("int x = 1;") != bench._code_only("int x = 2;")
    s = 'asm("add.rn.f32 %0, %1; // not a comment"); char c = \'/\';'
    out = bench._code_only(s)
    assert '"add.rn.f32 %0, %1; // not a comment"' in out and "'/'" in out


def test_source_hash_is_stable():
    assert bench.kernel_source_hash() == bench.kernel_source_hash()
    assert len(bench.kernel_source_hash()) == 16


def test_e2e_staging_views_alias_one_slab():
    call = bench.workload_calls("decode")[0]
    b = bench.CallBuffers(call, torch.device("cpu"))
    kind, in_pad, out_pad, in_bytes, out_bytes = bench._e2e_sizes(b)
    before = [t.clone() for t in b.inputs()]
    din = torch.empty(in_pad, dtype=torch.uint8)
    dout = torch.empty(out_pad, dtype=torch.uint8)
    assert bench._carve_into(b, bench._E2E_IN[kind], din, 0) == in_pad
    assert bench._carve_into(b, bench._E2E_OUT[kind], dout, 0) == out_pad
    base = din.data_ptr()
    for t, t0 in zip(b.inputs(), before):
        assert base <= t.data_ptr() < base + in_pad and (t.data_ptr() - base) % 256 == 0
        assert torch.equal(t, t0)
    for t in b.outputs():
        assert dout.data_ptr() <= t.data_ptr() < dout.data_ptr() + out_pad
    assert in_bytes == sum(t.numel() * t.element_size() for t in b.inputs())
    assert out_bytes == sum(t.numel() * t.element_size() for t in b.outputs())


def test_oracle_sample_threads_cover_every_row():
    """Threaded oracle timing splits each call's rows into blocks; the bytes
    counted are those of the whole sample either way."""
    calls = bench.workload_calls("tiny")
    _, n1, b1 = bench.oracle_sample(calls, 0.0, max_steps=1, threads=1)
    _, n3, b3 = bench.oracle_sample(calls, 0.0, max_steps=1, threads=3)
    assert n1 == n3 == 1 and b1 == b3 == bench.call_bytes(calls[0])
    cpu = bench.host_cpu()
    assert cpu["nproc"] >= 1


def test_oracle_rows_are_independent():
    """What threading over row blocks relies on: the oracle's rows do not
    depend on each other, so blocks computed separately equal the whole."""
    import numpy as np
    import oracle
    from tensor_allreduce_residual_ar_b200 import workloads as wl
    inp = wl.make_norm_inputs(wl.TINY, 16, H=256)
    parts = [wl.bits(p) for p in inp.partials]
    res = wl.bits(inp.residual)
    whole = oracle.ar_add_rmsnorm(parts, res, wl.bits(inp.weight), inp.eps, False, 0)["y"]
    blocks = [oracle.ar_add_rmsnorm([p[a:b] for p in parts], res[a:b], wl.bits(inp.weight),
                                    inp.eps, False, 0)["y"] for a, b in ((0, 5), (5, 11), (11, 16))]
    assert np.array_equal(whole, np.concatenate(blocks))


def test_sweep_summary_fields():
    sweep = {"prefill": [{"T": 8192, "dtype": "bf16", "us": 104.0, "frac_of_peak": 0.98,
                          "frac_of_8TBps": 0.8, "plan": 9}],
             "decode": [{"T": 1, "dtype": "bf16", "us": 2.5, "frac_of_peak": 0.01,
                         "frac_of_8TBps": 0.01, "plan": 4},
                        {"T": 80, "dtype": "bf16", "us": 4.2, "frac_of_peak": 0.3,
                         "frac_of_8TBps": 0.27, "plan": 4}]}
    s = bench.sweep_summary(sweep)
    assert s["prefill_T8192"] == [104.0, 0.98, 0.8, 9]
    assert s["decode_us_min_max"] == [2.5, 4.2] and s["decode_T80_bf16"][0] == 4.2


def test_tp_crossover():
    rows = [[1, 8192, 5.0, 7.0, 12.0], [80, 8192, 8.0, 9.0, 14.0], [256, 8192, 20.0, 15.0, 18.0],
            [8192, 4096, None, 300.0, 280.0]]
    c = bench.tp_crossover(rows)
    assert c == {"twoshot_beats_oneshot_from_T": 256, "nccl_beats_fused_from_T": 8192}
    assert bench.tp_crossover(rows[:2]) == {"twoshot_beats_oneshot_from_T": None,
                                            "nccl_beats_fused_from_T": None}


def test_workload_calls_take_other_token_counts():
    import bench
    base = bench.workload_calls("qk")
    assert [c[2] for c in base] == [1, 64, 2048]
    assert [c[2] for c in bench.workload_calls("qk", [4096, 8192])] == [4096, 8192]
    dec = bench.workload_calls("decode", [3])
    assert [(c[2], c[3]) for c in dec] == [(3, "bf16"), (3, "fp16")]


def test_reference_arm_line():
    """The reference arm (the CPU oracle on the host cores) prints its JSON
    line with the same metric and unit, no GPU involved."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "3", "--warmup", "3"],
                       cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s" and d["steps"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
