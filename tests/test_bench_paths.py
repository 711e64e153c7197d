"""bench.py's host logic that names the path a forward takes and counts this
library's launches in it (no GPU): AUTO as include/coli_moe.h states it (the
fused kernel up to 64 tokens where it applies, the two-pass path for 65 to 1024
tokens, the GEMV path below 48 tokens and the GEMM path otherwise)."""
import dataclasses

import pytest

import bench
import synth


@pytest.mark.parametrize("T,want", [(1, "fused"), (3, "fused"), (64, "fused"), (65, "twopass"),
                                    (512, "twopass"), (1024, "twopass"), (1025, "gemm"),
                                    (2048, "gemm")])
def test_auto_on_glm_shapes(T, want):
    assert bench.resolve_path(synth.GLM_PREFILL, T, "auto") == want


def test_auto_where_the_s8_paths_do_not_apply():
    odd = dataclasses.replace(synth.TINY, H=384)          # H not a multiple of 256
    assert bench.resolve_path(odd, 4, "auto") == "gemv"
    assert bench.resolve_path(odd, 200, "auto") == "gemm"
    narrow = dataclasses.replace(synth.TINY, I=128)       # I not a multiple of 256
    assert bench.resolve_path(narrow, 200, "auto") == "gemm"
    assert bench.resolve_path(synth.GLM_PREFILL, 512, "auto", bits=8) == "gemm"
    assert bench.resolve_path(synth.GLM_PREFILL, 512, "gemv") == "gemv"   # asked for


@pytest.mark.parametrize("T,path,want", [
    (1, "auto", 3),         # router, fused kernel, combine
    (512, "auto", 8),       # router, top-k, union, x records, 2 passes, h records, combine
    (512, "gemm", 9),       # router + fp16 operand, top-k, union, gather, 2 GEMMs, h, combine
    (3, "gemv", 4),         # router, top-k + union, 2 GEMVs
    (20, "gemv", 5),        # T * E > 4096: top-k and union apart
])
def test_launch_counts(T, path, want):
    fused = bench.resolve_path(synth.GLM_PREFILL, T, path) == "fused"
    assert bench.launches_per_layer(synth.GLM_PREFILL, T, path, fused) == want
