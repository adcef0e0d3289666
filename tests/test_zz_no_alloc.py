"""csa2_attend_noalloc -- attention for callers that cannot allocate device
memory (a framework that owns all device memory and exposes no allocator to
plugins, or a serving loop that must not allocate while it runs).  It keeps
its split partials in a fixed array inside the library instead of a caller
workspace.  Here it must reproduce csa2_attend's output, within the parity
tolerance, on two calls in a row (the shared array keeps the previous call's
contents, which must not leak into the next), and refuse sizes over its
limit.  This file is collected last on purpose."""
import pytest
import torch

import synth
from parity_util import ATOL, RTOL

pytestmark = pytest.mark.gpu


def test_noalloc_attend_matches_workspace_attend_twice():
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE, DeviceWorkload

    w = synth.workload(3, small=True)            # 2 requests x 64 heads, 8 layers, two top-k groups
    dw = DeviceWorkload(w, out_fp32=True)
    dw.step()                                    # reference outputs through csa2_attend + workspace
    torch.cuda.synchronize()
    for li in (1, 5):                            # two calls in a row: different queries and top-k groups
        q = dw.layers[li][0]
        topk = dw.topk[dw.layer_topk[li]]
        out = torch.full_like(dw.outs[li], float("nan"))
        assert csa2.csa2_attend_noalloc(dw.cache, q, topk, SOFTMAX_SCALE, out) == 0
        torch.cuda.synchronize()
        ref = dw.outs[li]
        assert torch.isfinite(out).all()
        assert ((out - ref).abs() <= ATOL + RTOL * ref.abs()).all(), f"layer {li}"
    assert csa2.csa2_get_device_error(dw.cache) == 0


def test_noalloc_attend_rejects_sizes_over_its_limit():
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE, DeviceWorkload

    w = synth.workload(4, small=True)            # 8 requests
    dw = DeviceWorkload(w, build=False)
    heads = csa2.ATTEND_NOALLOC_MAX_ROWS // w.batch + 1
    q = torch.zeros(w.batch, heads, 512, dtype=torch.bfloat16, device="cuda")
    topk = torch.full((w.batch, 512), -1, dtype=torch.int32, device="cuda")
    out = torch.zeros(w.batch, heads, 512, dtype=torch.float32, device="cuda")
    assert csa2.csa2_attend_noalloc(dw.cache, q, topk, SOFTMAX_SCALE, out) == 2
