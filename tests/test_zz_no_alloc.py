"""hga_forward_prefill_noalloc: the prefill path on the library's fixed device
scratch, for callers that cannot allocate device memory at call time (their
memory belongs to another allocator or a fixed arena, or they are handed only
input and output buffers).

Checked through the C ABI against the ordinary hga_forward(HGA_PREFILL) on
two calls in a row with different shapes and seeds (the second call runs on
the scratch the first one left behind).  This file is collected last so a
run that stops at the first failure has run every other test first; it also
passes on its own in a fresh process.
"""
import pytest
import torch

from tests.parity import TOL, row_rel_err
from workloads import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu

QWEN = WORKLOADS["qwen3_30b_a3b_bf16_prefill_32k"]
TINY = WORKLOADS["tiny_f32_prefill_1k"]


def _hp(hga, w):
    return hga.HGAParams(C=w.C, g_s=w.g_s, F=w.F, L=w.L, K_c=w.K_c, K_g=w.K_g,
                         rope_theta=w.theta)


@pytest.mark.parametrize("cases", [
    ((QWEN.replace(T=2048), 1), (QWEN.replace(T=64 * 13 + 21), 2)),
    ((TINY, 3), (TINY.replace(T=700, Hq=4, Hkv=2), 4)),
])
def test_noalloc_matches_forward_twice(gpu_lib, cases):
    dev = torch.device("cuda")
    for w, seed in cases:
        q, k, v, pos, _ = make_prefill_inputs(w, seed=seed, device=dev)
        hp = _hp(gpu_lib, w)
        ref = gpu_lib.hga_forward_prefill(q, k, v, pos, hp, want_lse=True)
        out = torch.empty_like(q)
        lse = torch.empty(w.B, w.Hq, w.T, device=dev, dtype=torch.float32)
        gpu_lib.hga_forward_prefill_noalloc(q, k, v, pos, hp, out, lse=lse)
        torch.cuda.synchronize()
        tol = TOL[w.dtype]
        assert row_rel_err(out.float().cpu().numpy(), ref["out"].float().cpu().numpy()) <= tol
        assert (lse - ref["lse"]).abs().max().item() <= tol * max(1.0, ref["lse"].abs().max().item())
        # the same kernels on the same inputs: the results are also bit-identical
        assert torch.equal(out, ref["out"]) and torch.equal(lse, ref["lse"])


def test_noalloc_rejects_oversized_shapes(gpu_lib):
    w = QWEN.replace(T=32768)
    dev = torch.device("cuda")
    q = torch.zeros(1, w.T, w.Hq, w.D, dtype=torch.bfloat16, device=dev)
    k = torch.zeros(1, w.T, w.Hkv, w.D, dtype=torch.bfloat16, device=dev)
    pos = torch.zeros(1, w.T, dtype=torch.int32, device=dev)
    with pytest.raises(gpu_lib.HGAError, match="workspace"):
        gpu_lib.hga_forward_prefill_noalloc(q, k, k, pos, _hp(gpu_lib, w), torch.empty_like(q))
