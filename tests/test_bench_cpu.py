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
